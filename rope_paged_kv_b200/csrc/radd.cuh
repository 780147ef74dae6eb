// radd.cuh -- in-place add of a [T, 2 * n_kv_heads * head_dim] tensor into the paged cache
// (kv_cache_radd).  Same producer / consumer staging and token schedule as the banded
// store: the producer resolves each token's cache row (sequence + batch_offset, position,
// page translation) and bulk-copies the token's input row together with the K and V cache
// rows it will add into; the consumers add in float32, round once and write the sums over
// the staged cache rows; the storer warp bulk-copies those rows back to the cache.
#pragma once

#include "banded.cuh"

namespace rs {

// CW consumer warps + the producer and storer warps
template <int CW>
__host__ __device__ constexpr int radd_threads() { return 32 * (CW + 2); }

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
  int32_t overlap;  // launch-overlap mode (kOverlap*)
  uint32_t stall_test_ns;  // > 0: the launch starts with a wait nothing completes (a test)
  uint32_t *sched;  // claim counter + finished CTAs, or nullptr for a static schedule
};

struct RaddMeta {
  int64_t kv_base;
  int32_t ok, tok, stop, pad;
};

template <typename T, int D, int CW, int LAG>
__global__ void __launch_bounds__(radd_threads<CW>(), 1) radd_kernel(const __grid_constant__ RaddParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / N;
  constexpr int kConsumers = 32 * CW;
  constexpr int kThreads = radd_threads<CW>();
  constexpr int G = kConsumers / L;
  constexpr int EB = (int)sizeof(T);
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *done = full + p.S;
  uint64_t *empty = done + p.S;
  RaddMeta *meta = reinterpret_cast<RaddMeta *>(smem + p.meta_off);
  uint32_t *s_offs = reinterpret_cast<uint32_t *>(smem + p.offs_off);
  uint32_t *s_cl = s_offs + (p.batch + 1);
  __shared__ int s_abort;
  __shared__ __align__(8) uint64_t s_never;  // no thread ever arrives here

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) grid_dep_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], CW);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&s_never, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (p.overlap != kOverlapEarlyMeta) grid_dep_wait();
  const bool good = stage_offsets(p.offs, p.batch, p.T, p.staged, s_offs);
  if (p.staged)
    for (int i = tid; i < p.batch; i += kThreads) {
      const uint64_t seq = (uint64_t)i + p.batch_offset;
      s_cl[i] = seq < p.cache.n_seqs ? __ldg(p.cache.cache_lengths + seq) : 0u;
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
  const int64_t hidden = (int64_t)p.n_kv * D;
  const uint32_t row_bytes = (uint32_t)(hidden * EB);  // one plane's heads of one token

  if (p.stall_test_ns != 0 && warp >= 2) {
    // A test of the timeout path (stall_test_ns > 0): the consumers wait on a barrier that
    // no thread ever arrives at, for at most stall_test_ns; when the wait runs out they do
    // what a pipeline wait that runs out makes them do.
    if (!mbar_wait(&s_never, 0, &s_abort, p.stall_test_ns) && lane == 0) {
      s_abort = 1;
      raise(p.err, ROPE_DEVERR_TIMEOUT);
    }
  } else if (warp == 0) {
    const bool dyn = p.sched != nullptr;
    const int n_static = static_tokens(p.T, n_local, dyn);
    const int dyn0 = n_static * (int)gridDim.x;  // first claimed token
    int issued = 0;
    bool aborted = false;
    bool waited = p.overlap != kOverlapEarlyMeta;
    auto resolve = [&](int tok, RaddMeta &m) -> uint32_t {
      m = RaddMeta{};
      m.tok = tok;
      if (tok < 0) return 0u;
      const int b = find_seq(offs, p.batch, (uint32_t)tok);
      const uint32_t t = (uint32_t)tok - offs[b];
      const uint64_t seq = (uint64_t)b + p.batch_offset;
      uint32_t e = 0;
      if (seq >= p.cache.n_seqs) {
        e = ROPE_DEVERR_BATCH;
      } else {
        const uint32_t cl = p.staged ? s_cl[b] : __ldg(p.cache.cache_lengths + seq);
        e = translate(p.cache, p.layer, seq, (uint64_t)cl + t, &m.kv_base);
      }
      m.ok = (e == 0);
      return e;
    };
    auto ensure_wait = [&]() {
      if (!waited) {
        grid_dep_wait();
        waited = true;
      }
    };
    auto issue = [&](const RaddMeta &m, int cnt) {
      for (int j = 0; j < cnt && !aborted; ++j) {
        RaddMeta mj{};
        mj.kv_base = __shfl_sync(0xffffffffu, m.kv_base, j);
        mj.ok = __shfl_sync(0xffffffffu, m.ok, j);
        mj.tok = __shfl_sync(0xffffffffu, m.tok, j);
        const int s = issued % p.S;
        if (lane == 0) {
          if (!mbar_wait(&empty[s], ((issued / p.S) & 1) ^ 1, &s_abort)) {
            aborted = true;
          } else {
            meta[s] = mj;
            mbar_arrive_expect_tx(&full[s], mj.ok ? 4u * row_bytes : 0u);
            if (mj.ok) {
              unsigned char *st = smem + (size_t)s * p.stage_bytes;
              bulk_g2s(st, reinterpret_cast<const unsigned char *>(p.a) + (int64_t)mj.tok * p.a_stride * EB,
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
          }
        }
        aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
        if (!aborted) ++issued;
      }
    };
    for (int c = 0; c < n_static && !aborted; c += 32) {
      RaddMeta m;
      const int i = c + lane;
      const uint32_t e = resolve(i < n_static ? (int)blockIdx.x + i * (int)gridDim.x : -1, m);
      ensure_wait();
      raise(p.err, e);
      issue(m, min(32, n_static - c));
    }
    if (dyn) {
      ensure_wait();
      uint32_t next = 0;
      if (lane == 0) next = atomicAdd(p.sched, (uint32_t)kDynChunk);
      while (!aborted) {
        const int64_t first = dyn0 + (int64_t)__shfl_sync(0xffffffffu, next, 0);
        if (first >= p.T) break;
        const int cnt = (int)min((int64_t)kDynChunk, (int64_t)p.T - first);
        RaddMeta m;
        const uint32_t e = resolve(lane < cnt ? (int)first + lane : -1, m);
        raise(p.err, e);
        if (lane == 0) next = atomicAdd(p.sched, (uint32_t)kDynChunk);
        issue(m, cnt);
      }
    }
    bool marked = false;  // the stop marker went into stage issued % S
    if (!aborted && lane == 0) {  // stop marker
      const int s = issued % p.S;
      if (!mbar_wait(&empty[s], ((issued / p.S) & 1) ^ 1, &s_abort)) {
        aborted = true;
      } else {
        meta[s].stop = 1;
        mbar_arrive(&full[s]);
        marked = true;
      }
    }
    aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
    if (lane == 0) {
      if (aborted) {
        s_abort = 1;
        raise(p.err, ROPE_DEVERR_TIMEOUT);
      }
      // let the loads issued land before the CTA's shared memory goes away (the last S;
      // after the stop marker, not token issued - S, stored before its stage was reused)
      for (int ii = max(0, issued - p.S + (marked ? 1 : 0)); ii < issued; ++ii) {
        int never = 0;
        mbar_wait(&full[ii % p.S], (ii / p.S) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // storer: the summed K and V rows back to the cache, LAG bulk groups kept in flight
    if (lane == 0) {
      int n_done = 0;
      for (int i = 0;; ++i) {
        const int s = i % p.S;
        if (!mbar_wait(&done[s], (i / p.S) & 1, &s_abort)) {
          s_abort = 1;
          raise(p.err, ROPE_DEVERR_TIMEOUT);
          break;
        }
        if (meta[s].stop) break;
        n_done = i + 1;
        if (meta[s].ok) {
          const unsigned char *st = smem + (size_t)s * p.stage_bytes;
          const int64_t base = meta[s].kv_base;
          for (int plane = 0; plane < 2; ++plane) {
            unsigned char *dst =
                reinterpret_cast<unsigned char *>(plane ? p.cache.v : p.cache.k) + base * EB;
            const unsigned char *src = st + (2 + plane) * row_bytes;
            if (p.kv_contig) {
              bulk_s2g(dst, src, row_bytes);
            } else {
              for (int h = 0; h < p.n_kv; ++h)
                bulk_s2g(dst + (int64_t)h * p.cache.head_stride * EB, src + h * D * EB,
                         (uint32_t)(D * EB));
            }
          }
        }
        bulk_commit();
        if (i >= LAG) {
          bulk_wait_read<LAG>();
          mbar_arrive(&empty[(i - LAG) % p.S]);
        }
      }
      bulk_wait_read<0>();
      for (int i = max(0, n_done - LAG); i < n_done; ++i) mbar_arrive(&empty[i % p.S]);
      bulk_wait<0>();
    }
  } else {
    const int ctid = tid - 64;
    const int li = ctid % L, grp = ctid / L;
    const int rows = 2 * p.n_kv;
    for (int i = 0;; ++i) {
      const int s = i % p.S;
      if (!mbar_wait(&full[s], (i / p.S) & 1, &s_abort)) {
        if (lane == 0) {
          s_abort = 1;
          raise(p.err, ROPE_DEVERR_TIMEOUT);
        }
        break;
      }
      const RaddMeta m = meta[s];
      if (!m.stop && m.ok) {
        unsigned char *st = smem + (size_t)s * p.stage_bytes;
        for (int j = grp; j < rows; j += G) {
          const int plane = j >= p.n_kv ? 1 : 0, h = j - plane * p.n_kv;
          const int64_t e0 = (int64_t)plane * hidden + (int64_t)h * D + li * N;
          float xa[N], xc[N];
          VT::widen(ld_shared_v4(st + e0 * EB), xa);
          VT::widen(ld_shared_v4(st + 2 * row_bytes + e0 * EB), xc);
#pragma unroll
          for (int e = 0; e < N; ++e) xc[e] = xc[e] + xa[e];
          st_shared_v4(st + 2 * row_bytes + e0 * EB, VT::narrow(xc));
        }
        fence_proxy_async_smem();  // the storer's bulk copies read the sums
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&done[s]);  // the stop marker is handed on too
      if (m.stop) break;
    }
  }
  if (p.sched != nullptr) {
    __syncthreads();  // every claim of this CTA is made
    if (tid == 0) sched_release(p.sched);
  }
}

}  // namespace rs
