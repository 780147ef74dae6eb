// bshd.cuh -- BSHD continuous-batch RoPE with in-place K (qk_rope_bshd_continuous).
//
// Decode-shaped work (one or a few tokens per sequence) is latency-bound, so this kernel
// keeps the dependency chain short instead of staging: one CTA per token, every thread
// resolves the token's (valid, slot, position) itself from broadcast loads while its Q
// loads are already in flight; K rows and the freqs row are then loaded in one round trip,
// rotated, and stored.  No block-level barrier, no shared memory.  With launch overlap
// mode 2 the descriptor loads come first, before the wait for the preceding kernels, and
// the Q loads after it.
#pragma once

#include "common.cuh"

namespace rs {

constexpr int kBshdThreads = 256;

struct BshdParams {
  const void *q;
  void *out;
  int32_t B, S, n_q, n_kv;
  void *k;
  int64_t slot_stride, layer_stride, pos_stride, head_stride;
  const uint32_t *lookup, *cache_lengths, *valid;
  uint32_t num_slots, cache_max_seq, layer;
  RopeDev rope;
  uint32_t *err;
  int32_t f_row_bytes;
  int32_t overlap;  // launch-overlap mode (kOverlap*)
};

template <typename T, int D, int UQ, int UK>
__global__ void __launch_bounds__(kBshdThreads) bshd_rope_kernel(const __grid_constant__ BshdParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / N;
  constexpr int G = kBshdThreads / L;
  const int tid = threadIdx.x, li = tid % L, grp = tid / L;
  const int c0 = li * N;
  const bool in_rope = lane_in_rope(p.rope, c0);
  const int64_t n_tok = (int64_t)p.B * p.S;
  const bool early_meta = p.overlap == kOverlapEarlyMeta;
  if (tid == 0) grid_dep_launch_dependents();
  if (!early_meta) grid_dep_wait();
  for (int64_t tok = blockIdx.x; tok < n_tok; tok += gridDim.x) {
    const T *qrow = reinterpret_cast<const T *>(p.q) + tok * p.n_q * D;
    T *orow = reinterpret_cast<T *>(p.out) + tok * p.n_q * D;
    uint4 vq[UQ];
    if (!early_meta) {
#pragma unroll
      for (int u = 0; u < UQ; ++u) {
        const int h = grp + u * G;
        vq[u] = h < p.n_q ? ld_stream(qrow + (int64_t)h * D + c0) : make_uint4(0, 0, 0, 0);
      }
    }
    const int b = (int)(tok / p.S), s = (int)(tok % p.S);
    const bool valid = (uint32_t)s < __ldg(p.valid + b);
    const uint32_t slot = __ldg(p.lookup + b);
    const uint64_t pos = (uint64_t)__ldg(p.cache_lengths + b) + (uint32_t)s;
    uint32_t e = 0;
    if (valid) {
      if (slot >= p.num_slots)
        e = ROPE_DEVERR_BATCH;
      else if (pos >= p.rope.max_seq_len || pos >= p.cache_max_seq)
        e = ROPE_DEVERR_POSITION;
    }
    if (early_meta) {
      grid_dep_wait();  // returns at once after the first token
#pragma unroll
      for (int u = 0; u < UQ; ++u) {
        const int h = grp + u * G;
        vq[u] = h < p.n_q ? ld_stream(qrow + (int64_t)h * D + c0) : make_uint4(0, 0, 0, 0);
      }
    }
    if (tid == 0) raise(p.err, e);
    const bool ok = valid && e == 0;
    const void *F = reinterpret_cast<const unsigned char *>(p.rope.table) +
                    (ok ? (int64_t)pos * p.f_row_bytes : 0);
    T *krow = reinterpret_cast<T *>(p.k) +
              (ok ? (int64_t)slot * p.slot_stride + (int64_t)p.layer * p.layer_stride +
                        (int64_t)pos * p.pos_stride
                  : 0);
    uint4 vk[UK];
#pragma unroll
    for (int u = 0; u < UK; ++u) {
      const int h = grp + u * G;
      vk[u] = (ok && h < p.n_kv) ? ld_plain(krow + (int64_t)h * p.head_stride + c0)
                                 : make_uint4(0, 0, 0, 0);
    }
    // Q rows: rotated into output inside the valid length, copied beyond it
    for (int base = 0; base < p.n_q; base += G * UQ) {
      if (base > 0) {
#pragma unroll
        for (int u = 0; u < UQ; ++u) {
          const int h = base + grp + u * G;
          vq[u] = h < p.n_q ? ld_stream(qrow + (int64_t)h * D + c0) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < UQ; ++u) {
        const int h = base + grp + u * G;
        float x[N];
        VT::widen(vq[u], x);
        rope_vec<N>(x, F, p.rope, li, ok);
        if (h < p.n_q && (ok || !valid))
          st_plain(orow + (int64_t)h * D + c0, (ok && in_rope) ? VT::narrow(x) : vq[u]);
      }
    }
    // K rows: rotated in place
    if (ok) {
      for (int base = 0; base < p.n_kv; base += G * UK) {
        if (base > 0) {
#pragma unroll
          for (int u = 0; u < UK; ++u) {
            const int h = base + grp + u * G;
            vk[u] = h < p.n_kv ? ld_plain(krow + (int64_t)h * p.head_stride + c0)
                               : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int u = 0; u < UK; ++u) {
          const int h = base + grp + u * G;
          float x[N];
          VT::widen(vk[u], x);
          rope_vec<N>(x, F, p.rope, li, true);
          if (h < p.n_kv && in_rope) st_plain(krow + (int64_t)h * p.head_stride + c0, VT::narrow(x));
        }
      }
    }
  }
}

}  // namespace rs
