// common.cuh -- parameter blocks and device helpers shared by the prologue kernels.
#pragma once

#include "../../include/rope_store.h"
#include "device_utils.cuh"
#include "pipeline.cuh"

#include <cuda_runtime.h>
#include <stdint.h>

namespace rs {

// ----------------------------------------------------------------- parameter blocks --

struct PagedDev {
  void *k, *v;
  int64_t page_stride, layer_stride, slot_stride, head_stride;
  const uint32_t *page_table;
  int64_t pt_stride;
  const uint32_t *cache_lengths;
  uint32_t max_pages, page_size, num_pages, n_seqs;
};

struct RopeDev {
  const void *table;
  int32_t dtype;  // 0 bf16, 1 f16, 2 f32
  uint32_t max_seq_len;
  int32_t R, off, interleaved;
};

__device__ __forceinline__ void raise(uint32_t *err, uint32_t bits) {
  if (err != nullptr && bits != 0u) atomicOr(err, bits);
}

// Launch-overlap modes (rope_overlap_t): 0 plain launch; 1 programmatic dependent launch,
// every global access after the predecessors completed; 2 the same, but descriptor arrays
// (offsets, cache lengths, page and lookup tables, gammas) are read before that.
constexpr int kOverlapOff = 0;
constexpr int kOverlapPdl = 1;
constexpr int kOverlapEarlyMeta = 2;

// Token schedule of the staged kernels when the caller gives a workspace: a CTA first takes
// its static share of the tokens, all but about kDynTail of them, then claims the rest
// kDynChunk tokens at a time from a counter, so that CTAs that get more bandwidth take
// more of the tail.
constexpr int kDynTail = 4;
constexpr int kDynChunk = 2;
constexpr int kMaxStaticTokens = 32;

// Tokens a CTA takes statically: all of its share without a workspace.
__device__ __forceinline__ int static_tokens(int T, int n_local, bool dyn) {
  if (!dyn) return n_local;
  const int per = T / (int)gridDim.x;
  return per > kDynTail ? min(per - kDynTail, kMaxStaticTokens) : 0;
}

// End of a CTA in a launch with a workspace (sched[0] the claim counter, sched[1] CTAs
// finished): the last CTA to finish returns both words to zero for the next launch.
// Called once per CTA, after the CTA's last claim.
__device__ __forceinline__ void sched_release(uint32_t *sched) {
  __threadfence();
  if (atomicAdd(sched + 1, 1u) == gridDim.x - 1u) {
    atomicExch(sched, 0u);
    atomicExch(sched + 1, 0u);
    __threadfence();
  }
}

// sequence b with offs[b] <= row < offs[b+1] (offs a valid partition, row < offs[batch])
__device__ __forceinline__ int find_seq(const uint32_t *offs, int batch, uint32_t row) {
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offs[mid] <= row)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

// Page-table translation of (seq, pos); returns 0 or the ROPE_DEVERR_* bit.
__device__ __forceinline__ uint32_t translate(const PagedDev &c, uint32_t layer, uint64_t seq,
                                              uint64_t pos, int64_t *base) {
  const uint64_t col = pos / c.page_size;
  if (col >= c.max_pages) return ROPE_DEVERR_PAGE_INDEX;
  const uint32_t page = __ldg(c.page_table + (int64_t)seq * c.pt_stride + (int64_t)col);
  if (page >= c.num_pages) return ROPE_DEVERR_PAGE_ID;
  *base = (int64_t)page * c.page_stride + (int64_t)layer * c.layer_stride +
          (int64_t)(pos % c.page_size) * c.slot_stride;
  return 0;
}

// Copy input_row_offsets to shared memory (when `staged`) and check that it partitions
// [0, T): first entry 0, never decreasing, last entry T.  Returns false if it does not.
__device__ __forceinline__ bool stage_offsets(const uint32_t *offs, int batch, int T,
                                              bool staged, uint32_t *s_offs) {
  int bad = 0;
  for (int i = threadIdx.x; i <= batch; i += blockDim.x) {
    const uint32_t o = __ldg(offs + i);
    if (staged) s_offs[i] = o;
    if (i == 0)
      bad |= (o != 0u);
    else
      bad |= (o < __ldg(offs + i - 1));
    if (i == batch) bad |= (o != (uint32_t)T);
  }
  return bad == 0;
}

// ------------------------------------------------------------------------------ RoPE --

// M consecutive freqs_cis values starting at element `base` of the row F (any address
// space), widened to float.  FDT: 0 bf16, 1 f16, 2 f32.  base * sizeof(element) is a
// multiple of the vector width used.
template <int FDT, int M>
__device__ __forceinline__ void load_freqs(const void *F, int base, float (&f)[M]) {
  if constexpr (FDT == 2) {
    const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(F) + base);
#pragma unroll
    for (int i = 0; i < M / 4; ++i) {
      const float4 v = p[i];
      f[4 * i] = v.x;
      f[4 * i + 1] = v.y;
      f[4 * i + 2] = v.z;
      f[4 * i + 3] = v.w;
    }
  } else {
    const unsigned short *h = reinterpret_cast<const unsigned short *>(F) + base;
    uint32_t w[M / 2];
    if constexpr (M >= 8) {
#pragma unroll
      for (int i = 0; i < M / 8; ++i) {
        const uint4 v = reinterpret_cast<const uint4 *>(h)[i];
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
    } else {
      const uint2 v = *reinterpret_cast<const uint2 *>(h);
      w[0] = v.x;
      w[1] = v.y;
    }
#pragma unroll
    for (int i = 0; i < M / 2; ++i) {
      const unsigned short lo = (unsigned short)(w[i] & 0xffffu), hi = (unsigned short)(w[i] >> 16);
      if constexpr (FDT == 0) {
        f[2 * i] = __uint_as_float((uint32_t)lo << 16);
        f[2 * i + 1] = __uint_as_float((uint32_t)hi << 16);
      } else {
        f[2 * i] = __half2float(__ushort_as_half(lo));
        f[2 * i + 1] = __half2float(__ushort_as_half(hi));
      }
    }
  }
}

// RoPE of one lane's vector x = columns c0 .. c0+N-1 of its head row, c0 = li * N.  The
// rotated columns are [off, off + R); every lane vector is either wholly inside or wholly
// outside (the host checks the alignment).  All lanes of the warp must call this together:
// half-split partners (R/2 columns apart = R/(2N) lanes) come by shuffle.
template <int N, int FDT>
__device__ __forceinline__ void rope_vec_t(float (&x)[N], const void *F, const RopeDev &rp,
                                           int li, bool rotate) {
  const int c0 = li * N;
  const bool in_rope = c0 >= rp.off && c0 < rp.off + rp.R;
  if (rp.interleaved) {
    if (rotate && in_rope) {
      float f[N];
      load_freqs<FDT, N>(F, c0 - rp.off, f);
#pragma unroll
      for (int e = 0; e < N; e += 2) {
        const float a = x[e], b = x[e + 1], c = f[e], s = f[e + 1];
        x[e] = a * c - b * s;
        x[e + 1] = a * s + b * c;
      }
    }
  } else {
    const int half = rp.R >> 1;
    const int H = half / N;                 // lanes between partners
    const int rl = (c0 - rp.off) / N;       // lane index inside the rotated columns
    const bool first = in_rope && rl < H;
    const int partner = in_rope ? (first ? li + H : li - H) : li;
    const int src = (int)(threadIdx.x & 31) - li + partner;
    float y[N];
#pragma unroll
    for (int e = 0; e < N; ++e) y[e] = __shfl_sync(0xffffffffu, x[e], src);
    if (rotate && in_rope) {
      const int i0 = first ? (c0 - rp.off) : (c0 - rp.off - half);
      float f[2 * N];
      load_freqs<FDT, 2 * N>(F, 2 * i0, f);
#pragma unroll
      for (int e = 0; e < N; ++e) {
        const float c = f[2 * e], s = f[2 * e + 1];
        x[e] = first ? (x[e] * c - y[e] * s) : (y[e] * s + x[e] * c);
      }
    }
  }
}

template <int N>
__device__ __forceinline__ void rope_vec(float (&x)[N], const void *F, const RopeDev &rp,
                                         int li, bool rotate) {
  if (rp.dtype == 2)
    rope_vec_t<N, 2>(x, F, rp, li, rotate);
  else if (rp.dtype == 0)
    rope_vec_t<N, 0>(x, F, rp, li, rotate);
  else
    rope_vec_t<N, 1>(x, F, rp, li, rotate);
}

__device__ __forceinline__ bool lane_in_rope(const RopeDev &rp, int c0) {
  return c0 >= rp.off && c0 < rp.off + rp.R;
}

}  // namespace rs
