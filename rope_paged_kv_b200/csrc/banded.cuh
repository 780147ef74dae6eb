// banded.cuh -- the ragged paged store with optional per-head RMSNorm, for one or two
// bands (rope_split_store_paged_ragged, fused_qk_rmsnorm_rope_paged,
// fused_dual_qk_rmsnorm_rope_paged).
//
// Persistent CTAs, one ring of S shared-memory stages each; a token's row lives in one
// stage from load to store, and the bulk-copy (TMA) engine moves it both ways:
//   warp 0, producer:  for up to 32 tokens at a time each lane resolves one token
//                      (sequence by binary search over the staged input_row_offsets,
//                      position, page-table translation); then, token by token, it waits
//                      for a free stage, publishes the metadata and bulk-copies the token's
//                      Q | K | V head blocks of every band plus each band's freqs_cis row
//                      into it.  Its tokens are a static strided share and, when the caller
//                      gives a workspace, chunks claimed from a counter after that (see
//                      static_tokens); a stop marker in the next stage ends the CTA;
//   warps 2.., consumers: per token, the Q and K head rows are spread over lane groups of
//                      L = head_dim / vector lanes; each lane normalises (shuffle reduction
//                      over its group) and rotates its 16 bytes (a half-split partner's 16
//                      bytes are read from the stage) and writes them back in place;
//   warp 1, storer:    once the consumers are done with a token, bulk-copies the stage's Q
//                      block to q_out and its K and V blocks to the cache page, waits until
//                      the copies have read the stage, and hands the stage back.
// V rows never enter registers, except for an FP8 cache.  The extended-output instantiation
// (EXT) writes some results to stage regions of their own instead of in place: Q rounded
// into another element type, and the E4M3 codes of K and V for an FP8 cache; the storer
// copies those regions out.  The row range of a token is the band concatenation
// [Q main | K main | V main | Q index | K index | (V index)].
#pragma once

#include "common.cuh"

#include <cuda_fp8.h>

namespace rs {

// A CTA is a producer warp, a storer warp and CW consumer warps; the storer keeps LAG
// bulk-store groups in flight before handing a stage back.  Three shapes are built: a light
// one (4 consumer warps, more CTAs per SM) for little work per token, and six or eight
// consumer warps for RMSNorm, many heads and FP8 caches.
template <int CW>
__host__ __device__ constexpr int pipe_threads() { return 32 * (CW + 2); }

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
  int32_t k_inplace;  // K heads come from the token's cache slot, not from the input
  // Q output in another element type: the consumers write the rotated Q rows, converted,
  // to a stage region at qo_off, from where the storer copies them
  int32_t q_conv, q_dtype, q_eb, qo_off;
  // FP8 (E4M3) cache: the consumers write K (rotated) and V rows as codes of value / scale
  // to stage regions at k8_off and v8_off, from where the storer copies them
  int32_t kv8, k8_off, v8_off;
  const float *k_scale, *v_scale;
};

// N float values written to shared memory as N E4M3 codes (nearest, ties to even,
// saturating at +-448)
template <int N>
__device__ __forceinline__ void st_shared_e4m3(unsigned char *p, const float (&x)[N]) {
  uint32_t w[N / 4];
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i], x[4 * i + 1]),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i + 2], x[4 * i + 3]),
                                                 __NV_SATFINITE, __NV_E4M3);
    w[i] = lo | (hi << 16);
  }
  if constexpr (N == 8) {
    st_shared_v2(p, w[0], w[1]);
  } else {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(smem_addr(p)), "r"(w[0]) : "memory");
  }
}

// N float values written to shared memory as N elements of type qd (0 bf16, 1 f16, 2 f32),
// rounded to nearest even
template <int N>
__device__ __forceinline__ void st_shared_elems(unsigned char *p, const float (&x)[N], int qd) {
  if (qd == 2) {
#pragma unroll
    for (int k = 0; k < N; k += 4)
      st_shared_v4(p + k * 4, make_uint4(__float_as_uint(x[k]), __float_as_uint(x[k + 1]),
                                         __float_as_uint(x[k + 2]), __float_as_uint(x[k + 3])));
    return;
  }
  uint32_t w[N / 2];
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    if (qd == 0) {
      __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t *>(&h);
    } else {
      __half2 h = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
  }
  if constexpr (N == 8) {
    st_shared_v4(p, make_uint4(w[0], w[1], w[2], w[3]));
  } else {
    st_shared_v2(p, w[0], w[1]);
  }
}

struct BandedParams {
  BandDev band[2];
  int32_t n_bands;
  int32_t overlap;   // launch-overlap mode (kOverlap*)
  uint32_t *sched;   // claim counter + finished CTAs, or nullptr for a static schedule
  int32_t work0, work_total;  // Q + K head rows of band 0, of both bands
  const uint32_t *offs;
  int32_t batch, T;
  RopeDev rope;
  uint32_t layer;
  uint32_t *err;
  float weight_offset;
  int32_t mbc;  // multiply_before_cast: 0 rounds the normalised value before the gamma multiply
  // dynamic shared memory layout
  int32_t S, stage_bytes, f_row_bytes, staged, elem_bytes;
  int32_t bar_off, meta_off, gamma_off, offs_off, items_off;
};

// a consumer thread's head row of a token, packed: stage byte offset (18 bits), kind (2 bits
// from bit 27: 0 Q, 1 K, 2 V; V rows are items only for an FP8 cache), band (bit 29),
// active flag (bit 30)
constexpr uint32_t kItemOffMask = (1u << 18) - 1u;
constexpr int kItemKindShift = 27;
constexpr int kItemBandShift = 29;
constexpr uint32_t kItemAct = 1u << 30;

struct StageMeta {
  int64_t kv_base[2];
  int32_t pos[2];
  int32_t ok[2];
  int32_t tok;   // the token held by the stage
  int32_t stop;  // no token: the CTA's work is done
};

// Load C consecutive 16-byte chunks at `p` (shared memory) into out[0..C).  The lanes of a
// head-row group read neighbouring C*16-byte runs; issuing chunk (k + rot) % C at step k,
// with rot = (lane-in-group / lanes-per-128B) % C, puts the 8 lanes of a quarter-warp on 8
// different 16-byte bank groups.  The rotation is undone with fixed selects.
template <int C>
__device__ __forceinline__ void lds_chunks(const unsigned char *p, int rot, uint4 (&out)[C]) {
  uint4 t[C];
#pragma unroll
  for (int k = 0; k < C; ++k) t[k] = ld_shared_v4(p + ((k + rot) % C) * 16);
  // t[k] holds chunk (k + rot) % C: rotate right by rot
#pragma unroll
  for (int k = 0; k < C; ++k) out[k] = t[k];
  if constexpr (C >= 2) {
    if (rot & 1) {
#pragma unroll
      for (int k = 0; k < C; ++k) out[(k + 1) % C] = t[k];
#pragma unroll
      for (int k = 0; k < C; ++k) t[k] = out[k];
    }
  }
  if constexpr (C >= 4) {
    if (rot & 2) {
#pragma unroll
      for (int k = 0; k < C; ++k) out[(k + 2) % C] = t[k];
    }
  }
}

// M consecutive table values (element type fdt) starting at element `col` of the shared
// row F, widened to float, read bank-conflict free across the lanes of a group (`gl` =
// lane index inside the group).
template <int M>
__device__ __forceinline__ void lds_freqs(const unsigned char *F, int fdt, int col, int gl,
                                          float (&f)[M]) {
  if (fdt == 2) {
    constexpr int C = M / 4;           // 16-byte chunks per lane
    constexpr int LP = 32 / M > 0 ? 32 / M : 1;  // lanes sharing one 128-byte line
    uint4 c[C];
    lds_chunks<C>(F + col * 4, (gl / LP) % C, c);
#pragma unroll
    for (int k = 0; k < C; ++k) {
      f[4 * k] = __uint_as_float(c[k].x);
      f[4 * k + 1] = __uint_as_float(c[k].y);
      f[4 * k + 2] = __uint_as_float(c[k].z);
      f[4 * k + 3] = __uint_as_float(c[k].w);
    }
  } else {
    constexpr int C = M / 8 > 0 ? M / 8 : 1;
    uint32_t w[C * 4];
    if constexpr (M >= 8) {
      constexpr int LP = 64 / M;
      uint4 c[C];
      lds_chunks<C>(F + col * 2, (gl / LP) % C, c);
#pragma unroll
      for (int k = 0; k < C; ++k) {
        w[4 * k] = c[k].x;
        w[4 * k + 1] = c[k].y;
        w[4 * k + 2] = c[k].z;
        w[4 * k + 3] = c[k].w;
      }
    } else {
      const uint2 v = *reinterpret_cast<const uint2 *>(F + col * 2);
      w[0] = v.x;
      w[1] = v.y;
    }
#pragma unroll
    for (int i = 0; i < M / 2; ++i) {
      const unsigned short lo = (unsigned short)(w[i] & 0xffffu), hi = (unsigned short)(w[i] >> 16);
      if (fdt == 0) {
        f[2 * i] = __uint_as_float((uint32_t)lo << 16);
        f[2 * i + 1] = __uint_as_float((uint32_t)hi << 16);
      } else {
        f[2 * i] = __half2float(__ushort_as_half(lo));
        f[2 * i + 1] = __half2float(__ushort_as_half(hi));
      }
    }
  }
}

#ifndef ROPE_LIGHT_MIN_CTAS
#define ROPE_LIGHT_MIN_CTAS 2
#endif
// resident CTAs per SM the register budget is sized for: the light shape (<= 4 consumer
// warps) and the six- and eight-warp ones
template <int CW>
__host__ __device__ constexpr int pipe_min_ctas() { return CW <= 4 ? ROPE_LIGHT_MIN_CTAS : 2; }

// EXT: built with the extended outputs (a Q output in another element type, FP8 cache rows)
template <typename T, int D, bool NORM, int CW, int LAG, bool EXT>
__global__ void __launch_bounds__(pipe_threads<CW>(), pipe_min_ctas<CW>())
    banded_store_kernel(const __grid_constant__ BandedParams p) {
  constexpr int kConsumerWarps = CW;
  constexpr int kConsumers = 32 * CW;
  constexpr int kPipeThreads = pipe_threads<CW>();
  constexpr int kStoreLag = LAG;
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / (2 * N);           // lanes per head row: each lane owns 2 vectors
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
  if (tid == 0) grid_dep_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], kConsumerWarps);
      mbar_init(&empty[s], 1);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  if (p.overlap != kOverlapEarlyMeta) grid_dep_wait();
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
    grid_dep_wait();
    if (tid == 0) {
      raise(p.err, ROPE_DEVERR_ROW_OFFSETS);
      if (p.sched != nullptr) sched_release(p.sched);
    }
    return;
  }
  const uint32_t *offs = p.staged ? s_offs : p.offs;
  const int n_local = (p.T - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  unsigned char *stages = smem;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer --
    const bool dyn = p.sched != nullptr;
    const int n_static = static_tokens(p.T, n_local, dyn);
    const int dyn0 = n_static * (int)gridDim.x;  // first claimed token
    int issued = 0;
    bool aborted = false;
    bool waited = p.overlap != kOverlapEarlyMeta;  // otherwise done at the top
    // This lane's token (tok < 0: none) resolved into m; returns its error bits, raised by
    // the caller once the predecessors are done (error words may be reset by one).
    auto resolve = [&](int tok, StageMeta &m) -> uint32_t {
      m = StageMeta{};
      m.tok = tok;
      if (tok < 0) return 0u;
      const int b = find_seq(offs, p.batch, (uint32_t)tok);
      const uint32_t t = (uint32_t)tok - offs[b];
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
      return e_all;
    };
    auto ensure_wait = [&]() {
      if (!waited) {
        grid_dep_wait();
        waited = true;
      }
    };
    // stage and load the tokens held by lanes 0..cnt-1 of m, in lane order
    auto issue = [&](const StageMeta &m, int cnt) {
      for (int j = 0; j < cnt && !aborted; ++j) {
        StageMeta mj;
        mj.kv_base[0] = __shfl_sync(0xffffffffu, m.kv_base[0], j);
        mj.kv_base[1] = __shfl_sync(0xffffffffu, m.kv_base[1], j);
        mj.pos[0] = __shfl_sync(0xffffffffu, m.pos[0], j);
        mj.pos[1] = __shfl_sync(0xffffffffu, m.pos[1], j);
        mj.ok[0] = __shfl_sync(0xffffffffu, m.ok[0], j);
        mj.ok[1] = __shfl_sync(0xffffffffu, m.ok[1], j);
        mj.tok = __shfl_sync(0xffffffffu, m.tok, j);
        mj.stop = 0;
        const int s = issued % p.S;
        if (lane == 0) {
          if (!mbar_wait(&empty[s], ((issued / p.S) & 1) ^ 1, &s_abort)) {
            aborted = true;
          } else {
            meta[s] = mj;
            const uint32_t tok = (uint32_t)mj.tok;
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
              if (bd.k_inplace && bd.n_kv > 0) {  // K from the slot it is updated in
                const unsigned char *kc =
                    reinterpret_cast<const unsigned char *>(bd.cache.k) + mj.kv_base[k] * EB;
                unsigned char *kd = st + bd.smem_off + bd.n_q * D * EB;
                if (bd.kv_contig)
                  bulk_g2s(kd, kc, (uint32_t)(bd.n_kv * D * EB), &full[s]);
                else
                  for (int h = 0; h < bd.n_kv; ++h)
                    bulk_g2s(kd + h * D * EB, kc + (int64_t)h * bd.cache.head_stride * EB,
                             (uint32_t)(D * EB), &full[s]);
              }
              if (p.f_row_bytes)
                bulk_g2s(st + bd.f_off,
                         reinterpret_cast<const unsigned char *>(p.rope.table) +
                             (int64_t)mj.pos[k] * p.f_row_bytes,
                         (uint32_t)p.f_row_bytes, &full[s]);
            }
          }
        }
        aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
        if (!aborted) ++issued;
      }
    };
    // the static share: tokens blockIdx.x + i * gridDim.x
    for (int c = 0; c < n_static && !aborted; c += 32) {
      StageMeta m;
      const int i = c + lane;
      const uint32_t e = resolve(i < n_static ? (int)blockIdx.x + i * (int)gridDim.x : -1, m);
      ensure_wait();
      raise(p.err, e);
      issue(m, min(32, n_static - c));
    }
    // the claimed tail: the next claim is issued before the current chunk is staged
    if (dyn) {
      ensure_wait();
      uint32_t next = 0;
      if (lane == 0) next = atomicAdd(p.sched, (uint32_t)kDynChunk);
      while (!aborted) {
        const int64_t first = dyn0 + (int64_t)__shfl_sync(0xffffffffu, next, 0);
        if (first >= p.T) break;
        const int cnt = (int)min((int64_t)kDynChunk, (int64_t)p.T - first);
        StageMeta m;
        const uint32_t e = resolve(lane < cnt ? (int)first + lane : -1, m);
        raise(p.err, e);
        if (lane == 0) next = atomicAdd(p.sched, (uint32_t)kDynChunk);
        issue(m, cnt);
      }
    }
    // stop marker: the next stage carries no token
    if (!aborted && lane == 0) {
      const int s = issued % p.S;
      if (!mbar_wait(&empty[s], ((issued / p.S) & 1) ^ 1, &s_abort)) {
        aborted = true;
      } else {
        meta[s].stop = 1;
        mbar_arrive(&full[s]);
      }
    }
    aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
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
      int n_done = 0;  // tokens stored
      for (int i = 0;; ++i) {
        const int s = i % p.S;
        if (!mbar_wait(&done[s], (i / p.S) & 1, &s_abort)) {
          s_abort = 1;
          raise(p.err, ROPE_DEVERR_TIMEOUT);
          break;
        }
        if (meta[s].stop) break;
        n_done = i + 1;
        const uint32_t tok = (uint32_t)meta[s].tok;
        const unsigned char *st = stages + (size_t)s * p.stage_bytes;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (k >= p.n_bands || !meta[s].ok[k]) continue;
          const BandDev &bd = k ? p.band[1] : p.band[0];
          const unsigned char *blk = st + bd.smem_off;
          const uint32_t qb = (uint32_t)(bd.n_q * D * EB), kb = (uint32_t)(bd.n_kv * D * EB);
          if (qb) {
            if (bd.q_conv)  // the converted rows
              bulk_s2g(reinterpret_cast<unsigned char *>(bd.q_out) +
                           (int64_t)tok * bd.q_out_stride * bd.q_eb,
                       st + bd.qo_off, (uint32_t)(bd.n_q * D * bd.q_eb));
            else
              bulk_s2g(reinterpret_cast<unsigned char *>(bd.q_out) +
                           (int64_t)tok * bd.q_out_stride * EB,
                       blk, qb);
          }
          const int64_t base = meta[s].kv_base[k];
          const int CE = (EXT && bd.kv8) ? 1 : EB;  // cache element bytes
          const uint32_t kcb = (uint32_t)(bd.n_kv * D * CE);
          for (int plane = 0; plane < (bd.n_v ? 2 : 1); ++plane) {
            unsigned char *dst = reinterpret_cast<unsigned char *>(plane ? bd.cache.v : bd.cache.k) +
                                 base * CE;
            const unsigned char *src = (EXT && bd.kv8) ? st + (plane ? bd.v8_off : bd.k8_off)
                                                       : blk + qb + plane * kb;
            if (bd.kv_contig) {
              if (kcb) bulk_s2g(dst, src, kcb);
            } else {
              for (int h = 0; h < bd.n_kv; ++h)
                bulk_s2g(dst + (int64_t)h * bd.cache.head_stride * CE, src + h * D * CE,
                         (uint32_t)(D * CE));
            }
          }
        }
        bulk_commit();
        // hand back the stage whose stores were issued kStoreLag tokens ago once they have
        // read it; up to kStoreLag newer groups may still be reading
        if (i >= kStoreLag) {
          bulk_wait_read<kStoreLag>();
          mbar_arrive(&empty[(i - kStoreLag) % p.S]);
        }
      }
      bulk_wait_read<0>();
      for (int i = max(0, n_done - kStoreLag); i < n_done; ++i) mbar_arrive(&empty[i % p.S]);
      bulk_wait<0>();
    }
  } else {
    // ------------------------------------------------------------------ consumers --
    // A head row is D / N 16-byte vectors; lane j of its group of L lanes owns two of them,
    // va and vb.  Half-split: the first R/(2N) lanes own a rotation pair each (vector
    // o/N + j and its partner R/(2N) vectors later), the other lanes own two unrotated
    // vectors.  Interleaved: lane j owns vectors j and j + L.
    const int ctid = tid - 64;
    const int li = ctid % L, grp = ctid / L;
    const unsigned gmask = (L == 32) ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));
    const RopeDev &rp = p.rope;
    const bool inter = rp.interleaved != 0;
    const int ov = rp.off / N, rv = rp.R / N;  // first rotated vector, rotated vectors
    int va, vb;
    bool rot_a, rot_b;
    if (inter) {
      va = li;
      vb = li + L;
      rot_a = va >= ov && va < ov + rv;
      rot_b = vb >= ov && vb < ov + rv;
    } else if (li < rv / 2) {
      va = ov + li;
      vb = ov + li + rv / 2;
      rot_a = rot_b = true;
    } else {
      // the k-th unrotated vector, k < (D/N - rv) / 2, and the one half of those later
      const int k = li - rv / 2, np = D / N - rv;
      const int ka = k, kb = k + np / 2;
      va = ka < ov ? ka : ka + rv;
      vb = kb < ov ? kb : kb + rv;
      rot_a = rot_b = false;
    }
    const bool busy = NORM || rot_a || rot_b;  // lanes with nothing to do leave bytes in place
    const int ca = va * N, cb = vb * N;         // first columns of the two vectors
    // table columns: interleaved, vector v uses F[v*N - off ..]; half-split pair uses
    // F[2 * (ca - off) ..] (cos, sin of pair ca - off + e)
    const int fa = inter ? ca - rp.off : 2 * (ca - rp.off);
    const int fb = cb - rp.off;
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
        const int kind = r < bd.n_q ? 0 : r < bd.n_q + bd.n_kv ? 1 : 2;
        const uint32_t soff = (uint32_t)(bd.smem_off + r * D * EB);
        w = kItemAct | (uint32_t)band << kItemBandShift | (uint32_t)kind << kItemKindShift | soff;
      }
      item[u * kConsumers] = w;
    }
    // per token: (cos, sin) of this lane's columns; per (band, kind): gamma + weight_offset
    float fca[N], fsa[N], fcb[N], fsb[N];
    float ga[N], gb[N];
    int g_sel = -1;
    float kinv0 = 1.f, kinv1 = 1.f, vinv0 = 1.f, vinv1 = 1.f;  // 1 / scale of FP8 planes
    for (int i = 0;; ++i) {
      const int s = i % p.S;
      if (!mbar_wait(&full[s], (i / p.S) & 1, &s_abort)) {
        if (lane == 0) {
          s_abort = 1;
          raise(p.err, ROPE_DEVERR_TIMEOUT);
        }
        break;
      }
      if (meta[s].stop) {  // hand the marker on to the storer
        __syncwarp();
        if (lane == 0) mbar_arrive(&done[s]);
        break;
      }
      if (EXT && i == 0) {  // after the producer's wait for the preceding kernels
        if (p.band[0].kv8) {
          kinv0 = 1.f / __ldg(p.band[0].k_scale);
          if (p.band[0].n_v) vinv0 = 1.f / __ldg(p.band[0].v_scale);
        }
        if (p.n_bands > 1 && p.band[1].kv8) {
          kinv1 = 1.f / __ldg(p.band[1].k_scale);
          if (p.band[1].n_v) vinv1 = 1.f / __ldg(p.band[1].v_scale);
        }
      }
      unsigned char *st = stages + (size_t)s * p.stage_bytes;
      const int ok0 = meta[s].ok[0], ok1 = meta[s].ok[1];
      int f_band = -1;
#pragma unroll 1
      for (int u = 0; u < n_items; ++u) {
        const uint32_t w = item[u * kConsumers];
        if (!(w & kItemAct)) continue;
        const int band = (w >> kItemBandShift) & 1;
        if (!(band ? ok1 : ok0)) continue;
        const int kind = (w >> kItemKindShift) & 3;
        const BandDev &bd = band ? p.band[1] : p.band[0];
        const bool conv = EXT && kind == 0 && bd.q_conv;  // every lane writes its Q
        const bool to8 = EXT && kind >= 1 && bd.kv8;       // and its K / V codes
        if (!busy && !conv && !to8) continue;
        if ((rot_a || rot_b) && f_band != band) {  // this token's table row for the band
          f_band = band;
          const unsigned char *F = st + bd.f_off;
          if (inter) {
            float f[N];
            if (rot_a) {
              lds_freqs<N>(F, rp.dtype, fa, li, f);
#pragma unroll
              for (int e = 0; e < N; e += 2) {
                fca[e] = fca[e + 1] = f[e];
                fsa[e] = fsa[e + 1] = f[e + 1];
              }
            }
            if (rot_b) {
              lds_freqs<N>(F, rp.dtype, fb, li, f);
#pragma unroll
              for (int e = 0; e < N; e += 2) {
                fcb[e] = fcb[e + 1] = f[e];
                fsb[e] = fsb[e + 1] = f[e + 1];
              }
            }
          } else {
            float f[2 * N];
            lds_freqs<2 * N>(F, rp.dtype, fa, li, f);
#pragma unroll
            for (int e = 0; e < N; ++e) {
              fca[e] = f[2 * e];
              fsa[e] = f[2 * e + 1];
            }
          }
        }
        unsigned char *row = st + (w & kItemOffMask);
        float xa[N], xb[N];
        VT::widen(ld_shared_v4(row + ca * EB), xa);
        VT::widen(ld_shared_v4(row + cb * EB), xb);
        // the row's first element within the band's [Q | K | V] block
        const int re = (int)(((w & kItemOffMask) - (uint32_t)bd.smem_off) / EB);
        if (EXT && kind == 2) {  // a V row of an FP8 cache: scaled and encoded, nothing else
          const float inv = band ? vinv1 : vinv0;
#pragma unroll
          for (int e = 0; e < N; ++e) {
            xa[e] *= inv;
            xb[e] *= inv;
          }
          unsigned char *vrow = st + bd.v8_off + (re - (bd.n_q + bd.n_kv) * D);
          st_shared_e4m3<N>(vrow + ca, xa);
          st_shared_e4m3<N>(vrow + cb, xb);
          continue;
        }
        if constexpr (NORM) {
          if (g_sel != band * 2 + kind) {  // gamma does not depend on the token: kept
            g_sel = band * 2 + kind;
            const unsigned char *gr = reinterpret_cast<const unsigned char *>(s_gamma + g_sel * D);
            lds_freqs<N>(gr, 2, ca, li, ga);
            lds_freqs<N>(gr, 2, cb, li, gb);
          }
          float2 acc = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < N; e += 2) {
            acc = __ffma2_rn(make_float2(xa[e], xa[e + 1]), make_float2(xa[e], xa[e + 1]), acc);
            acc = __ffma2_rn(make_float2(xb[e], xb[e + 1]), make_float2(xb[e], xb[e + 1]), acc);
          }
          float ss = acc.x + acc.y;
#pragma unroll
          for (int msk = L / 2; msk > 0; msk >>= 1) ss += __shfl_xor_sync(gmask, ss, msk);
          const float r = rsqrtf(ss * (1.0f / D) + bd.eps);
          const float2 rr = make_float2(r, r);
          if (p.mbc) {
#pragma unroll
            for (int e = 0; e < N; e += 2) {
              const float2 ya = __fmul2_rn(make_float2(xa[e], xa[e + 1]),
                                           __fmul2_rn(rr, make_float2(ga[e], ga[e + 1])));
              const float2 yb = __fmul2_rn(make_float2(xb[e], xb[e + 1]),
                                           __fmul2_rn(rr, make_float2(gb[e], gb[e + 1])));
              xa[e] = ya.x; xa[e + 1] = ya.y;
              xb[e] = yb.x; xb[e + 1] = yb.y;
            }
          } else {  // the normalised value is rounded to the element type, then scaled
#pragma unroll
            for (int e = 0; e < N; ++e) {
              xa[e] *= r;
              xb[e] *= r;
            }
            VT::widen(VT::narrow(xa), xa);
            VT::widen(VT::narrow(xb), xb);
#pragma unroll
            for (int e = 0; e < N; ++e) {
              xa[e] *= ga[e];
              xb[e] *= gb[e];
            }
          }
        }
        if (inter) {
          if (rot_a) {
#pragma unroll
            for (int e = 0; e < N; e += 2) {
              const float a = xa[e], b = xa[e + 1];
              xa[e] = fmaf(a, fca[e], -b * fsa[e]);
              xa[e + 1] = fmaf(a, fsa[e], b * fca[e]);
            }
          }
          if (rot_b) {
#pragma unroll
            for (int e = 0; e < N; e += 2) {
              const float a = xb[e], b = xb[e + 1];
              xb[e] = fmaf(a, fcb[e], -b * fsb[e]);
              xb[e + 1] = fmaf(a, fsb[e], b * fcb[e]);
            }
          }
        } else if (rot_a) {
          // (a, b) -> (a c - b s, a s + b c), pair e of vector va with pair e of vector vb
#pragma unroll
          for (int e = 0; e < N; e += 2) {
            const float2 a = make_float2(xa[e], xa[e + 1]), b = make_float2(xb[e], xb[e + 1]);
            const float2 c = make_float2(fca[e], fca[e + 1]), sn = make_float2(fsa[e], fsa[e + 1]);
            const float2 ya = __ffma2_rn(b, make_float2(-sn.x, -sn.y), __fmul2_rn(a, c));
            const float2 yb = __ffma2_rn(a, sn, __fmul2_rn(b, c));
            xa[e] = ya.x; xa[e + 1] = ya.y;
            xb[e] = yb.x; xb[e + 1] = yb.y;
          }
        }
        if (conv) {
          unsigned char *qrow = st + bd.qo_off + (size_t)re * bd.q_eb;
          st_shared_elems<N>(qrow + ca * bd.q_eb, xa, bd.q_dtype);
          st_shared_elems<N>(qrow + cb * bd.q_eb, xb, bd.q_dtype);
        } else if (to8) {  // a K row of an FP8 cache
          const float inv = band ? kinv1 : kinv0;
#pragma unroll
          for (int e = 0; e < N; ++e) {
            xa[e] *= inv;
            xb[e] *= inv;
          }
          unsigned char *krow = st + bd.k8_off + (re - bd.n_q * D);
          st_shared_e4m3<N>(krow + ca, xa);
          st_shared_e4m3<N>(krow + cb, xb);
        } else {
          if (NORM || rot_a) st_shared_v4(row + ca * EB, VT::narrow(xa));
          if (NORM || rot_b) st_shared_v4(row + cb * EB, VT::narrow(xb));
        }
      }
      fence_proxy_async_smem();  // the storer's bulk copies read what was written here
      __syncwarp();
      if (lane == 0) mbar_arrive(&done[s]);
    }
  }
  if (p.sched != nullptr) {
    __syncthreads();  // every claim of this CTA is made
    if (tid == 0) sched_release(p.sched);
  }
}

}  // namespace rs
