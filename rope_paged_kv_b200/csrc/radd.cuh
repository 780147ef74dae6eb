// radd.cuh -- in-place add of a [T, 2 * n_kv_heads * head_dim] tensor into the paged cache
// (kv_cache_radd).  Same producer / consumer staging as the banded store: the producer
// resolves each token's cache row (sequence + batch_offset, position, page translation) and
// bulk-copies the token's input row together with the K and V cache rows it will add into;
// the consumers add in float32, round once and store the rows back.
#pragma once

#include "banded.cuh"

namespace rs {

constexpr int kRaddConsumerWarps = 8;
constexpr int kRaddConsumers = 32 * kRaddConsumerWarps;
constexpr int kRaddThreads = kRaddConsumers + 32;  // + producer warp

struct RaddParams {
  const void *a;
  int64_t a_stride;
  int32_t T, n_kv, batch;
  PagedDev cache;
  const uint32_t *offs;
  uint32_t batch_offset, layer;
  uint32_t *err;
  int32_t S, stage_bytes, staged, kv_contig;  // kv_contig: a token's heads are adjacent
  int32_t bar_off, meta_off, offs_off;
};

struct RaddMeta {
  int64_t kv_base;
  int32_t ok, pad;
};

template <typename T, int D>
__global__ void __launch_bounds__(kRaddThreads, 1) radd_kernel(const __grid_constant__ RaddParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / N;
  constexpr int G = kRaddConsumers / L;
  constexpr int EB = (int)sizeof(T);
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *empty = full + p.S;
  RaddMeta *meta = reinterpret_cast<RaddMeta *>(smem + p.meta_off);
  uint32_t *s_offs = reinterpret_cast<uint32_t *>(smem + p.offs_off);
  uint32_t *s_cl = s_offs + (p.batch + 1);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kRaddConsumerWarps);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  const bool good = stage_offsets(p.offs, p.batch, p.T, p.staged, s_offs);
  if (p.staged)
    for (int i = tid; i < p.batch; i += kRaddThreads) {
      const uint64_t seq = (uint64_t)i + p.batch_offset;
      s_cl[i] = seq < p.cache.n_seqs ? __ldg(p.cache.cache_lengths + seq) : 0u;
    }
  if (!__syncthreads_and(good)) {
    if (tid == 0) raise(p.err, ROPE_DEVERR_ROW_OFFSETS);
    return;
  }
  const uint32_t *offs = p.staged ? s_offs : p.offs;
  const int n_local = (p.T - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  const int64_t hidden = (int64_t)p.n_kv * D;
  const uint32_t row_bytes = (uint32_t)(hidden * EB);  // one plane's heads of one token

  if (warp == 0) {
    int issued = 0;
    bool aborted = false;
    for (int c = 0; c < n_local && !aborted; c += 32) {
      RaddMeta m{};
      const int i = c + lane;
      if (i < n_local) {
        const uint32_t tok = blockIdx.x + (uint32_t)i * gridDim.x;
        const int b = find_seq(offs, p.batch, tok);
        const uint32_t t = tok - offs[b];
        const uint64_t seq = (uint64_t)b + p.batch_offset;
        uint32_t e = 0;
        if (seq >= p.cache.n_seqs) {
          e = ROPE_DEVERR_BATCH;
        } else {
          const uint32_t cl = p.staged ? s_cl[b] : __ldg(p.cache.cache_lengths + seq);
          e = translate(p.cache, p.layer, seq, (uint64_t)cl + t, &m.kv_base);
        }
        m.ok = (e == 0);
        raise(p.err, e);
      }
      const int cnt = min(32, n_local - c);
      for (int j = 0; j < cnt; ++j) {
        RaddMeta mj;
        mj.kv_base = __shfl_sync(0xffffffffu, m.kv_base, j);
        mj.ok = __shfl_sync(0xffffffffu, m.ok, j);
        const int ii = c + j;
        const int s = ii % p.S;
        if (lane == 0) {
          if (!mbar_wait(&empty[s], ((ii / p.S) & 1) ^ 1, &s_abort)) {
            aborted = true;
          } else {
            meta[s] = mj;
            mbar_arrive_expect_tx(&full[s], mj.ok ? 4u * row_bytes : 0u);
            if (mj.ok) {
              const uint32_t tok = blockIdx.x + (uint32_t)ii * gridDim.x;
              unsigned char *st = smem + (size_t)s * p.stage_bytes;
              bulk_g2s(st, reinterpret_cast<const unsigned char *>(p.a) + (int64_t)tok * p.a_stride * EB,
                       2u * row_bytes, &full[s]);
              const unsigned char *kb =
                  reinterpret_cast<const unsigned char *>(p.cache.k) + mj.kv_base * EB;
              const unsigned char *vb =
                  reinterpret_cast<const unsigned char *>(p.cache.v) + mj.kv_base * EB;
              if (p.kv_contig) {
                bulk_g2s(st + 2 * row_bytes, kb, row_bytes, &full[s]);
                bulk_g2s(st + 3 * row_bytes, vb, row_bytes, &full[s]);
              } else {
                for (int h = 0; h < p.n_kv; ++h) {
                  bulk_g2s(st + 2 * row_bytes + h * D * EB, kb + h * p.cache.head_stride * EB,
                           D * EB, &full[s]);
                  bulk_g2s(st + 3 * row_bytes + h * D * EB, vb + h * p.cache.head_stride * EB,
                           D * EB, &full[s]);
                }
              }
            }
            ++issued;
          }
        }
        aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
        if (aborted) break;
      }
    }
    if (aborted && lane == 0) {
      s_abort = 1;
      raise(p.err, ROPE_DEVERR_TIMEOUT);
      for (int ii = max(0, issued - p.S); ii < issued; ++ii) {
        int never = 0;
        mbar_wait(&full[ii % p.S], (ii / p.S) & 1, &never);
      }
    }
  } else {
    const int ctid = tid - 32;
    const int li = ctid % L, grp = ctid / L;
    const int rows = 2 * p.n_kv;
    for (int i = 0; i < n_local; ++i) {
      const int s = i % p.S;
      if (!mbar_wait(&full[s], (i / p.S) & 1, &s_abort)) {
        if (lane == 0) {
          s_abort = 1;
          raise(p.err, ROPE_DEVERR_TIMEOUT);
        }
        break;
      }
      const RaddMeta m = meta[s];
      if (m.ok) {
        const unsigned char *st = smem + (size_t)s * p.stage_bytes;
        for (int j = grp; j < rows; j += G) {
          const int plane = j >= p.n_kv ? 1 : 0, h = j - plane * p.n_kv;
          const int64_t e0 = (int64_t)plane * hidden + (int64_t)h * D + li * N;
          float xa[N], xc[N];
          VT::widen(ld_shared_v4(st + e0 * EB), xa);
          VT::widen(ld_shared_v4(st + 2 * row_bytes + e0 * EB), xc);
#pragma unroll
          for (int e = 0; e < N; ++e) xc[e] = xc[e] + xa[e];
          T *dst = reinterpret_cast<T *>(plane ? p.cache.v : p.cache.k) + m.kv_base +
                   (int64_t)h * p.cache.head_stride + li * N;
          st_plain(dst, VT::narrow(xc));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
}

}  // namespace rs
