// gemv_norm.cuh -- one-row GEMV fused with a partial RMSNorm (matmul_fused_partial_rmsnorm).
//
// y = x W^T with W [n, k] row-major.  The work is a single pass over W, so it is bound by
// HBM (or L2) bandwidth, not by the tensor cores, and by how many bytes are in flight in so
// short a kernel: a CTA takes R whole rows of W and bulk-copies them and x into shared
// memory at once (one cp.async.bulk per row, all counted on one mbarrier), then spreads each
// row's 16-byte chunks over all its threads; a thread reads its chunks of x once and reuses
// them for the R rows.  (Rows too long for shared memory take a register path that loads
// the chunks directly.)  Each row's dot product is reduced in float32 inside the CTA.
// Entries past n_normed are rounded and written at once; the entries to be normalised go to
// the caller's workspace in float32.  The last CTA to finish (a count in the workspace) reads
// them back, forms their sum of squares in a fixed order, writes x * rsqrt(mean + eps) *
// gamma and returns the count to zero.  No CTA waits for another.
#pragma once

#include "common.cuh"

namespace rs {

constexpr int kGemvThreads = 256;
constexpr int kGemvUnroll = 4;  // chunks of a row a thread loads per iteration

struct GemvParams {
  const void *x, *w;
  int64_t w_stride;  // elements between rows of W
  int32_t n, k, n_normed;
  const void *gamma;
  float eps;
  void *normed, *unnormed;
  uint32_t *count;  // workspace word 0: CTAs finished
  float *ws;        // workspace from byte 16: y of the entries to be normalised
  uint32_t *err;
  int32_t overlap;
  int32_t row_bytes;  // k * element size, padded to 16: a row's place in shared memory
  uint32_t stall_test_ns;  // > 0: the launch starts with a wait nothing completes (a test)
};

template <typename T>
__device__ __forceinline__ T to_elem(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 to_elem<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ __half to_elem<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ float to_elem<float>(float v) { return v; }

// the block-wide sum of v (every thread gets it), combined in a fixed order
__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < kGemvThreads / 32; ++i) t += red[i];
  return t;
}

template <typename T, int R, bool STAGED>
__global__ void __launch_bounds__(kGemvThreads)
    gemv_norm_kernel(const __grid_constant__ GemvParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int W = kGemvThreads / 32;
  extern __shared__ __align__(128) unsigned char smem[];  // STAGED: x | R rows of W
  __shared__ float red[R][W];
  __shared__ float red1[W];
  __shared__ int s_last;
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  __shared__ __align__(8) uint64_t s_never;  // no thread ever arrives here
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) grid_dep_launch_dependents();
  if (STAGED && tid == 0) {
    mbar_init(&bar, 1);
    mbar_init(&s_never, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  grid_dep_wait();  // x, W and gamma may come from the kernels before

  const int row0 = blockIdx.x * R;
  const int chunks = p.k / N;
  const T *x = reinterpret_cast<const T *>(p.x);
  const T *w = reinterpret_cast<const T *>(p.w);
  const int rows = min(R, p.n - row0);
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  if constexpr (STAGED) {
    __syncthreads();  // the barrier is initialised
    const uint32_t kb = (uint32_t)p.k * sizeof(T);
    // A test of the timeout path (stall_test_ns > 0): the loading thread first waits on a
    // barrier that no thread ever arrives at, for at most stall_test_ns; when that runs out
    // the CTA takes the path of a load wait that runs out.
    if (tid == 0 && p.stall_test_ns != 0 && !mbar_wait(&s_never, 0, &s_abort, p.stall_test_ns)) {
      s_abort = 1;
      raise(p.err, ROPE_DEVERR_TIMEOUT);
    }
    if (tid == 0 && kb > 0) {
      mbar_arrive_expect_tx(&bar, kb * (uint32_t)(rows + 1));
      bulk_g2s(smem, x, kb, &bar);
      for (int r = 0; r < rows; ++r)
        bulk_g2s(smem + (size_t)(r + 1) * p.row_bytes, w + (int64_t)(row0 + r) * p.w_stride,
                 kb, &bar);
    }
    bool ok = true;
    if (kb > 0 && !mbar_wait(&bar, 0, &s_abort)) {
      ok = false;
      if (lane == 0) raise(p.err, ROPE_DEVERR_TIMEOUT);
    }
    if (!__syncthreads_and(ok)) {
      // let the copies land before the CTA's shared memory goes away; count the CTA (the
      // last one returns the count to zero)
      if (tid == 0) {
        int never = 0;
        mbar_wait(&bar, 0, &never);
        if (p.n_normed > 0 && atomicAdd(p.count, 1u) == gridDim.x - 1u) atomicExch(p.count, 0u);
      }
      return;
    }
    for (int c = tid; c < chunks; c += kGemvThreads) {
      float xf[N];
      VT::widen(ld_shared_v4(smem + (size_t)c * 16), xf);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r < rows) {
          float wf[N];
          VT::widen(ld_shared_v4(smem + (size_t)(r + 1) * p.row_bytes + (size_t)c * 16), wf);
#pragma unroll
          for (int e = 0; e < N; ++e) acc[r] = fmaf(xf[e], wf[e], acc[r]);
        }
      }
    }
  } else {  // (braced: an unbraced statement here was compiled as if the rest of the
           // kernel belonged to the discarded branch)
    for (int c0 = tid; c0 < chunks; c0 += kGemvThreads * kGemvUnroll) {
      uint4 xv[kGemvUnroll], wv[kGemvUnroll][R];
#pragma unroll
      for (int u = 0; u < kGemvUnroll; ++u) {
        const int c = c0 + u * kGemvThreads;
        xv[u] = c < chunks ? ld_plain(x + (int64_t)c * N) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int r = 0; r < R; ++r)
          wv[u][r] = (c < chunks && row0 + r < p.n)
                         ? ld_stream(w + (int64_t)(row0 + r) * p.w_stride + (int64_t)c * N)
                         : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kGemvUnroll; ++u) {
        float xf[N];
        VT::widen(xv[u], xf);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float wf[N];
          VT::widen(wv[u][r], wf);
#pragma unroll
          for (int e = 0; e < N; ++e) acc[r] = fmaf(xf[e], wf[e], acc[r]);
        }
      }
    }
  }
  // the CTA's row sums: warps, then the warps' partials in a fixed order
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float v = acc[r];
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    if (lane == 0) red[r][warp] = v;
  }
  __syncthreads();
  if (tid < R && row0 + tid < p.n) {
    float y = 0.f;
    for (int i = 0; i < W; ++i) y += red[tid][i];
    const int row = row0 + tid;
    if (row < p.n_normed)
      p.ws[row] = y;
    else
      reinterpret_cast<T *>(p.unnormed)[row - p.n_normed] = to_elem<T>(y);
    __threadfence();  // the workspace entry is visible before this CTA is counted
  }
  if (p.n_normed == 0) return;
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.count, 1u) == gridDim.x - 1u;
  __syncthreads();
  if (!s_last) return;

  // the last CTA: every entry to be normalised is in the workspace.  A thread keeps the
  // entries it reads (and their gammas, read at the same time) for the output, so the
  // normalisation takes one round trip to the workspace; longer rows loop.
  __threadfence();
  constexpr int kKeep = 4;  // entries a thread keeps: n_normed <= 1024 in one pass
  const T *g = reinterpret_cast<const T *>(p.gamma);
  T *out = reinterpret_cast<T *>(p.normed);
  if (p.n_normed <= kKeep * kGemvThreads) {
    float v[kKeep], gv[kKeep];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kKeep; ++k) {
      const int i = tid + k * kGemvThreads;
      v[k] = i < p.n_normed ? __ldcg(p.ws + i) : 0.f;
      gv[k] = i < p.n_normed ? static_cast<float>(g[i]) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kKeep; ++k) ss = fmaf(v[k], v[k], ss);
    ss = block_sum(ss, red1);
    const float r = rsqrtf(ss / (float)p.n_normed + p.eps);
#pragma unroll
    for (int k = 0; k < kKeep; ++k) {
      const int i = tid + k * kGemvThreads;
      if (i < p.n_normed) out[i] = to_elem<T>(v[k] * r * gv[k]);
    }
  } else {
    float ss = 0.f;
    for (int i = tid; i < p.n_normed; i += kGemvThreads) {
      const float v = __ldcg(p.ws + i);
      ss = fmaf(v, v, ss);
    }
    ss = block_sum(ss, red1);
    const float r = rsqrtf(ss / (float)p.n_normed + p.eps);
    for (int i = tid; i < p.n_normed; i += kGemvThreads)
      out[i] = to_elem<T>(__ldcg(p.ws + i) * r * static_cast<float>(g[i]));
  }
  if (tid == 0) atomicExch(p.count, 0u);
}

}  // namespace rs
