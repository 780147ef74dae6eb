// banded.cuh -- the ragged paged store with optional per-head RMSNorm, for one or two
// bands (rope_split_store_paged_ragged, fused_qk_rmsnorm_rope_paged,
// fused_dual_qk_rmsnorm_rope_paged).
//
// Persistent CTAs, one ring of S shared-memory stages each; a token's row lives in one
// stage from load to store, and the bulk-copy (TMA) engine moves it both ways:
//   warp 0, producer:  for 32 tokens at a time each lane resolves one token (sequence by
//                      binary search over the staged input_row_offsets, position,
//                      page-table translation); then, token by token, it waits for a free
//                      stage, publishes the metadata and bulk-copies the token's Q | K | V
//                      head blocks of every band plus each band's freqs_cis row into it;
//   warps 2.., consumers: per token, the Q and K head rows are spread over lane groups of
//                      L = head_dim / vector lanes; each lane normalises (shuffle reduction
//                      over its group) and rotates its 16 bytes (a half-split partner's 16
//                      bytes are read from the stage) and writes them back in place;
//   warp 1, storer:    once the consumers are done with a token, bulk-copies the stage's Q
//                      block to q_out and its K and V blocks to the cache page, waits until
//                      the copies have read the stage, and hands the stage back.
// V rows never enter registers.  The row range of a token is the band concatenation
// [Q main | K main | V main | Q index | K index | (V index)].
#pragma once

#include "common.cuh"

namespace rs {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kPipeThreads = kConsumers + 64;  // + producer warp + storer warp

struct BandDev {
  const void *input;
  int64_t in_stride;
  int64_t q_col, k_col, v_col;
  int32_t n_q, n_kv, n_v;  // n_v = n_kv, or 0 for a K-only cache
  PagedDev cache;
  void *q_out;
  int64_t q_out_stride;
  const void *q_gamma, *k_gamma;
  float eps;
  // staging: the band's head blocks sit at stage offset `smem_off` as [Q | K | V]; nseg
  // bulk loads, segment i copies seg_bytes[i] from input column seg_col[i] to stage offset
  // seg_dst[i]; f_off: the band's freqs_cis row
  int32_t smem_off, f_off, tx_bytes, nseg;
  int64_t seg_col[3];
  int32_t seg_bytes[3], seg_dst[3];
  int32_t kv_contig;  // a slot's heads are adjacent in the cache (one store per plane)
};

struct BandedParams {
  BandDev band[2];
  int32_t n_bands;
  int32_t work0, work_total;  // Q + K head rows of band 0, of both bands
  const uint32_t *offs;
  int32_t batch, T;
  RopeDev rope;
  uint32_t layer;
  uint32_t *err;
  float weight_offset;
  // dynamic shared memory layout
  int32_t S, stage_bytes, f_row_bytes, staged, elem_bytes;
  int32_t bar_off, meta_off, gamma_off, offs_off, items_off;
};

// a consumer thread's head row of a token, packed: stage byte offset (18 bits), kind
// (0 Q, 1 K), band, active flag
constexpr uint32_t kItemOffMask = (1u << 18) - 1u;
constexpr int kItemKindShift = 27;
constexpr int kItemBandShift = 29;
constexpr uint32_t kItemAct = 1u << 30;

struct StageMeta {
  int64_t kv_base[2];
  int32_t pos[2];
  int32_t ok[2];
};

// This lane's (cos, sin) for a token from the staged freqs_cis row F (element type fdt).
// Interleaved: pair e/2 of the lane's vector uses F[fcol + e], F[fcol + e + 1]; fc[e] =
// fc[e+1] = cos and fs[e] = fs[e+1] = sin.  Half-split: element e uses pair (fcol/2 + e),
// fc[e] = cos and fs[e] = -sin for the first half (x*c - partner*s) or +sin for the second
// half (partner*s + x*c).
template <int N>
__device__ __forceinline__ void load_lane_freqs(const void *F, int fdt, bool inter, bool first,
                                                int fcol, float (&fc)[N], float (&fs)[N]) {
  if (inter) {
    float f[N];
    if (fdt == 2)
      load_freqs<2, N>(F, fcol, f);
    else if (fdt == 0)
      load_freqs<0, N>(F, fcol, f);
    else
      load_freqs<1, N>(F, fcol, f);
#pragma unroll
    for (int e = 0; e < N; e += 2) {
      fc[e] = fc[e + 1] = f[e];
      fs[e] = fs[e + 1] = f[e + 1];
    }
  } else {
    float f[2 * N];
    if (fdt == 2)
      load_freqs<2, 2 * N>(F, fcol, f);
    else if (fdt == 0)
      load_freqs<0, 2 * N>(F, fcol, f);
    else
      load_freqs<1, 2 * N>(F, fcol, f);
#pragma unroll
    for (int e = 0; e < N; ++e) {
      fc[e] = f[2 * e];
      fs[e] = first ? -f[2 * e + 1] : f[2 * e + 1];
    }
  }
}

template <typename T, int D, bool NORM>
__global__ void __launch_bounds__(kPipeThreads, 2)
    banded_store_kernel(const __grid_constant__ BandedParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / N;                 // lanes per head row
  constexpr int G = kConsumers / L;        // head rows per consumer pass
  constexpr int EB = (int)sizeof(T);
  static_assert(L <= 32 && 32 % L == 0, "a head row must fit in one warp");

  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *done = full + p.S;
  uint64_t *empty = done + p.S;
  StageMeta *meta = reinterpret_cast<StageMeta *>(smem + p.meta_off);
  float *s_gamma = reinterpret_cast<float *>(smem + p.gamma_off);
  uint32_t *s_offs = reinterpret_cast<uint32_t *>(smem + p.offs_off);
  uint32_t *s_cl = s_offs + (p.batch + 1);
  uint32_t *s_items = reinterpret_cast<uint32_t *>(smem + p.items_off);
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], kConsumerWarps);
      mbar_init(&empty[s], 1);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  const bool good = stage_offsets(p.offs, p.batch, p.T, p.staged, s_offs);
  if (p.staged)
    for (int i = tid; i < p.n_bands * p.batch; i += kPipeThreads) {
      const int bd = i >= p.batch ? 1 : 0;
      s_cl[i] = __ldg((bd ? p.band[1] : p.band[0]).cache.cache_lengths + (i - bd * p.batch));
    }
  if constexpr (NORM)
    for (int i = tid; i < 2 * p.n_bands * D; i += kPipeThreads) {
      const int which = i / D, d = i % D;  // 0 q main, 1 k main, 2 q index, 3 k index
      const BandDev &bd = (which >> 1) ? p.band[1] : p.band[0];
      const T *g = reinterpret_cast<const T *>((which & 1) ? bd.k_gamma : bd.q_gamma);
      s_gamma[i] = static_cast<float>(g[d]) + p.weight_offset;
    }
  if (!__syncthreads_and(good)) {
    if (tid == 0) raise(p.err, ROPE_DEVERR_ROW_OFFSETS);
    return;
  }
  const uint32_t *offs = p.staged ? s_offs : p.offs;
  const int n_local = (p.T - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  unsigned char *stages = smem;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer --
    int issued = 0;
    bool aborted = false;
    for (int c = 0; c < n_local && !aborted; c += 32) {
      StageMeta m{};
      const int i = c + lane;
      if (i < n_local) {
        const uint32_t tok = blockIdx.x + (uint32_t)i * gridDim.x;
        const int b = find_seq(offs, p.batch, tok);
        const uint32_t t = tok - offs[b];
        uint32_t e_all = 0;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (k >= p.n_bands) break;
          const BandDev &bd = k ? p.band[1] : p.band[0];
          const uint32_t cl = p.staged ? s_cl[k * p.batch + b] : __ldg(bd.cache.cache_lengths + b);
          const uint64_t pos = (uint64_t)cl + t;
          int64_t base = 0;
          const uint32_t e = pos >= p.rope.max_seq_len
                                 ? ROPE_DEVERR_POSITION
                                 : translate(bd.cache, p.layer, (uint64_t)b, pos, &base);
          m.ok[k] = (e == 0);
          m.kv_base[k] = base;
          m.pos[k] = (int32_t)(e == 0 ? pos : 0);
          e_all |= e;
        }
        raise(p.err, e_all);
      }
      const int cnt = min(32, n_local - c);
      for (int j = 0; j < cnt; ++j) {
        StageMeta mj;
        mj.kv_base[0] = __shfl_sync(0xffffffffu, m.kv_base[0], j);
        mj.kv_base[1] = __shfl_sync(0xffffffffu, m.kv_base[1], j);
        mj.pos[0] = __shfl_sync(0xffffffffu, m.pos[0], j);
        mj.pos[1] = __shfl_sync(0xffffffffu, m.pos[1], j);
        mj.ok[0] = __shfl_sync(0xffffffffu, m.ok[0], j);
        mj.ok[1] = __shfl_sync(0xffffffffu, m.ok[1], j);
        const int ii = c + j;
        const int s = ii % p.S;
        if (lane == 0) {
          if (!mbar_wait(&empty[s], ((ii / p.S) & 1) ^ 1, &s_abort)) {
            aborted = true;
          } else {
            meta[s] = mj;
            const uint32_t tok = blockIdx.x + (uint32_t)ii * gridDim.x;
            uint32_t tx = 0;
#pragma unroll
            for (int k = 0; k < 2; ++k)
              if (k < p.n_bands && mj.ok[k])
                tx += (uint32_t)((k ? p.band[1] : p.band[0]).tx_bytes + p.f_row_bytes);
            mbar_arrive_expect_tx(&full[s], tx);
            unsigned char *st = stages + (size_t)s * p.stage_bytes;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              if (k >= p.n_bands || !mj.ok[k]) continue;
              const BandDev &bd = k ? p.band[1] : p.band[0];
              const unsigned char *row =
                  reinterpret_cast<const unsigned char *>(bd.input) + (int64_t)tok * bd.in_stride * EB;
              for (int q = 0; q < bd.nseg; ++q)
                bulk_g2s(st + bd.seg_dst[q], row + bd.seg_col[q] * EB, (uint32_t)bd.seg_bytes[q],
                         &full[s]);
              if (p.f_row_bytes)
                bulk_g2s(st + bd.f_off,
                         reinterpret_cast<const unsigned char *>(p.rope.table) +
                             (int64_t)mj.pos[k] * p.f_row_bytes,
                         (uint32_t)p.f_row_bytes, &full[s]);
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
      // let the loads already issued land before the CTA's shared memory goes away
      for (int ii = max(0, issued - p.S); ii < issued; ++ii) {
        int never = 0;
        mbar_wait(&full[ii % p.S], (ii / p.S) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------------- storer --
    if (lane == 0) {
      for (int i = 0; i < n_local; ++i) {
        const int s = i % p.S;
        if (!mbar_wait(&done[s], (i / p.S) & 1, &s_abort)) {
          s_abort = 1;
          raise(p.err, ROPE_DEVERR_TIMEOUT);
          break;
        }
        const uint32_t tok = blockIdx.x + (uint32_t)i * gridDim.x;
        const unsigned char *st = stages + (size_t)s * p.stage_bytes;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (k >= p.n_bands || !meta[s].ok[k]) continue;
          const BandDev &bd = k ? p.band[1] : p.band[0];
          const unsigned char *blk = st + bd.smem_off;
          const uint32_t qb = (uint32_t)(bd.n_q * D * EB), kb = (uint32_t)(bd.n_kv * D * EB);
          if (qb)
            bulk_s2g(reinterpret_cast<unsigned char *>(bd.q_out) +
                         (int64_t)tok * bd.q_out_stride * EB,
                     blk, qb);
          const int64_t base = meta[s].kv_base[k];
          for (int plane = 0; plane < (bd.n_v ? 2 : 1); ++plane) {
            unsigned char *dst = reinterpret_cast<unsigned char *>(plane ? bd.cache.v : bd.cache.k) +
                                 base * EB;
            const unsigned char *src = blk + qb + plane * kb;
            if (bd.kv_contig) {
              if (kb) bulk_s2g(dst, src, kb);
            } else {
              for (int h = 0; h < bd.n_kv; ++h)
                bulk_s2g(dst + (int64_t)h * bd.cache.head_stride * EB, src + h * D * EB,
                         (uint32_t)(D * EB));
            }
          }
        }
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(&empty[s]);
      }
      bulk_wait<0>();
    }
  } else {
    // ------------------------------------------------------------------ consumers --
    const int ctid = tid - 64;
    const int li = ctid % L, grp = ctid / L;
    const int c0 = li * N;
    const unsigned gmask = (L == 32) ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));
    const RopeDev &rp = p.rope;
    const bool in_rope = lane_in_rope(rp, c0);
    const bool inter = rp.interleaved != 0;
    const int half = rp.R >> 1;
    const bool first = !inter && in_rope && (c0 - rp.off) < half;
    // element distance to the half-split partner vector, and this lane's first table column
    const int pdelta = (inter || !in_rope) ? 0 : (first ? half : -half);
    const int fcol = inter ? (c0 - rp.off) : 2 * (first ? (c0 - rp.off) : (c0 - rp.off - half));
    const bool busy = NORM || in_rope;  // lanes with nothing to do leave their bytes in place
    // the lanes of this group that write back (partners must have read first)
    const unsigned smask = gmask & __ballot_sync(0xffffffffu, busy);
    // this thread's head rows of a token, decoded once into shared memory
    const int n_items = (p.work_total + G - 1) / G;
    uint32_t *item = s_items + ctid;  // slot u at item[u * kConsumers]
    for (int u = 0; u < n_items; ++u) {
      const int j = grp + u * G;
      uint32_t w = 0;
      if (j < p.work_total) {
        const int band = j >= p.work0 ? 1 : 0;
        const BandDev &bd = band ? p.band[1] : p.band[0];
        const int r = j - (band ? p.work0 : 0);  // Q heads then K heads: stage rows 0..
        const int kind = r >= bd.n_q ? 1 : 0;
        const uint32_t soff = (uint32_t)(bd.smem_off + (r * D + c0) * EB);
        w = kItemAct | (uint32_t)band << kItemBandShift | (uint32_t)kind << kItemKindShift | soff;
      }
      item[u * kConsumers] = w;
    }
    float fc[N], fs[N];  // this token's (cos, sin) for this lane, current band
    float g[N], gp[N];   // gamma + weight_offset of this lane's and its partner's columns
    for (int i = 0; i < n_local; ++i) {
      const int s = i % p.S;
      if (!mbar_wait(&full[s], (i / p.S) & 1, &s_abort)) {
        if (lane == 0) {
          s_abort = 1;
          raise(p.err, ROPE_DEVERR_TIMEOUT);
        }
        break;
      }
      unsigned char *st = stages + (size_t)s * p.stage_bytes;
      const int ok0 = meta[s].ok[0], ok1 = meta[s].ok[1];
      int f_band = -1, g_sel = -1;
#pragma unroll 1
      for (int u = 0; u < n_items; ++u) {
        const uint32_t w = item[u * kConsumers];
        if (!busy || !(w & kItemAct)) continue;
        const int band = (w >> kItemBandShift) & 1;
        if (!(band ? ok1 : ok0)) continue;
        const int kind = (w >> kItemKindShift) & 1;
        unsigned char *src = st + (w & kItemOffMask);
        float x[N], xp[N];
        VT::widen(ld_shared_v4(src), x);
        const bool pair_lane = pdelta != 0;
        if (pair_lane) VT::widen(ld_shared_v4(src + pdelta * EB), xp);
        if constexpr (NORM) {
          if (g_sel != band * 2 + kind) {
            g_sel = band * 2 + kind;
            const float4 *gr = reinterpret_cast<const float4 *>(s_gamma + g_sel * D + c0);
#pragma unroll
            for (int e = 0; e < N / 4; ++e) {
              const float4 v = gr[e];
              g[4 * e] = v.x;
              g[4 * e + 1] = v.y;
              g[4 * e + 2] = v.z;
              g[4 * e + 3] = v.w;
            }
            if (pair_lane) {
              const float4 *gq = reinterpret_cast<const float4 *>(s_gamma + g_sel * D + c0 + pdelta);
#pragma unroll
              for (int e = 0; e < N / 4; ++e) {
                const float4 v = gq[e];
                gp[4 * e] = v.x;
                gp[4 * e + 1] = v.y;
                gp[4 * e + 2] = v.z;
                gp[4 * e + 3] = v.w;
              }
            }
          }
          const BandDev &bd = band ? p.band[1] : p.band[0];
          float2 acc = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < N; e += 2)
            acc = __ffma2_rn(make_float2(x[e], x[e + 1]), make_float2(x[e], x[e + 1]), acc);
          float ss = acc.x + acc.y;
#pragma unroll
          for (int msk = L / 2; msk > 0; msk >>= 1) ss += __shfl_xor_sync(gmask, ss, msk);
          const float r = rsqrtf(ss * (1.0f / D) + bd.eps);
#pragma unroll
          for (int e = 0; e < N; e += 2) {
            const float2 rg = __fmul2_rn(make_float2(r, r), make_float2(g[e], g[e + 1]));
            const float2 y = __fmul2_rn(make_float2(x[e], x[e + 1]), rg);
            x[e] = y.x;
            x[e + 1] = y.y;
          }
          if (pair_lane) {
#pragma unroll
            for (int e = 0; e < N; e += 2) {
              const float2 rg = __fmul2_rn(make_float2(r, r), make_float2(gp[e], gp[e + 1]));
              const float2 y = __fmul2_rn(make_float2(xp[e], xp[e + 1]), rg);
              xp[e] = y.x;
              xp[e + 1] = y.y;
            }
          }
        }
        if (in_rope) {
          if (f_band != band) {
            f_band = band;
            load_lane_freqs<N>(st + (band ? p.band[1] : p.band[0]).f_off, rp.dtype, inter, first,
                               fcol, fc, fs);
          }
          if (inter) {
#pragma unroll
            for (int e = 0; e < N; e += 2) {
              const float a = x[e], b = x[e + 1];
              x[e] = fmaf(a, fc[e], -b * fs[e]);
              x[e + 1] = fmaf(a, fs[e], b * fc[e]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < N; e += 2) {
              const float2 y = __ffma2_rn(make_float2(xp[e], xp[e + 1]), make_float2(fs[e], fs[e + 1]),
                                          __fmul2_rn(make_float2(x[e], x[e + 1]),
                                                     make_float2(fc[e], fc[e + 1])));
              x[e] = y.x;
              x[e + 1] = y.y;
            }
          }
        }
        if (!inter) __syncwarp(smask);  // partners have read before anyone writes back
        st_shared_v4(src, VT::narrow(x));
      }
      fence_proxy_async_smem();  // the storer's bulk copies read what was written here
      __syncwarp();
      if (lane == 0) mbar_arrive(&done[s]);
    }
  }
}

}  // namespace rs
