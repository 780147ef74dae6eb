// rope_store.cu -- sm_100a kernels and the C ABI of rope_store.h.
//
// Design (memory-bound path, no tensor cores):
//   * persistent grid: one CTA of 256 threads per resident slot (SM count x occupancy); each
//     CTA walks tokens with a grid stride;
//   * a token's row is split into head rows of head_dim elements; a head row is handled by
//     L = head_dim / (16-byte vector width) lanes (16 lanes for bf16 head_dim 128), so a CTA
//     keeps 256 / L head rows in flight per pass, U passes unrolled into registers;
//   * per token, warp 0 resolves the sequence (binary search over input_row_offsets staged
//     in shared memory), the position, the page-table translation and stages the freqs_cis
//     row in shared memory, while the other warps' 16-byte streaming loads of the row are
//     already in flight;
//   * RMSNorm: sum of squares reduced with xor-shuffles inside the head row's lanes;
//   * RoPE: interleaved pairs sit inside one lane's vector; half-split partners are
//     rope_dim/2 columns apart, i.e. rope_dim / (2 * vector width) lanes, fetched with one
//     shuffle per element;
//   * stores: 16-byte vectors; K/V rows of a token are contiguous runs in the cache page.
#include "../../include/rope_store.h"
#include "device_utils.cuh"

#include <cuda_runtime.h>

#include <type_traits>

namespace rs {

constexpr int kThreads = 256;
constexpr int kSmemSeqs = 1024;  // batches up to this size stage offsets / lengths in smem

// ---------------------------------------------------------------- device parameters --

struct PagedDev {
  void *k, *v;
  int64_t page_stride, layer_stride, slot_stride, head_stride;
  const uint32_t *page_table;
  int64_t pt_stride;
  const uint32_t *cache_lengths;
  uint32_t max_pages, page_size, num_pages, n_seqs;
};

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
};

struct RopeDev {
  const void *table;
  int32_t dtype;  // 0 bf16, 1 f16, 2 f32
  uint32_t max_seq_len;
  int32_t R, off, interleaved;
};

struct BandedParams {
  BandDev band[2];
  int32_t n_bands, rows0, rows_total;
  const uint32_t *offs;
  int32_t batch, T;
  RopeDev rope;
  uint32_t layer;
  uint32_t *err;
  float weight_offset;
};

struct TokMeta {
  int64_t kv_base[2];
  int32_t ok[2];
};

__device__ __forceinline__ void raise(uint32_t *err, uint32_t bits) {
  if (err != nullptr) atomicOr(err, bits);
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
__device__ __forceinline__ uint32_t translate(const PagedDev &c, uint32_t layer, int seq,
                                              uint64_t pos, int64_t *base) {
  const uint64_t col = pos / c.page_size;
  if (col >= c.max_pages) return ROPE_DEVERR_PAGE_INDEX;
  const uint32_t page = __ldg(c.page_table + (int64_t)seq * c.pt_stride + (int64_t)col);
  if (page >= c.num_pages) return ROPE_DEVERR_PAGE_ID;
  *base = (int64_t)page * c.page_stride + (int64_t)layer * c.layer_stride +
          (int64_t)(pos % c.page_size) * c.slot_stride;
  return 0;
}

// Stage input_row_offsets (and per-band cache lengths) and check that the offsets
// partition [0, T).  Returns true when the CTA may proceed.
__device__ __forceinline__ bool stage_offsets(const uint32_t *offs, int batch, int T,
                                              bool staged, uint32_t *s_offs) {
  int bad = 0;
  for (int i = threadIdx.x; i <= batch; i += kThreads) {
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

// RoPE of one lane's vector x (columns c0 .. c0+N-1 of its head row).  All lanes of the
// warp must call this together (half-split partners come by shuffle).
template <int N, int L>
__device__ __forceinline__ void rope_vec(float (&x)[N], const float *F, const RopeDev &rp,
                                         int li, bool rotate) {
  const int c0 = li * N;
  const bool in_rope = c0 >= rp.off && c0 < rp.off + rp.R;
  if (rp.interleaved) {
    if (rotate && in_rope) {
      const float *f = F + (c0 - rp.off);
#pragma unroll
      for (int e = 0; e < N; e += 2) {
        const float a = x[e], b = x[e + 1], c = f[e], s = f[e + 1];
        x[e] = a * c - b * s;
        x[e + 1] = a * s + b * c;
      }
    }
  } else {
    const int half = rp.R >> 1;
    const int H = half / N;                  // lanes between partners
    const int rl = (c0 - rp.off) / N;        // lane index inside the rotated columns
    const bool first = in_rope && rl < H;
    const int partner = in_rope ? (first ? li + H : li - H) : li;
    const int src = (int)(threadIdx.x & 31) - li + partner;
    float y[N];
#pragma unroll
    for (int e = 0; e < N; ++e) y[e] = __shfl_sync(0xffffffffu, x[e], src);
    if (rotate && in_rope) {
      const int i0 = first ? (c0 - rp.off) : (c0 - rp.off - half);
      const float *f = F + 2 * i0;
#pragma unroll
      for (int e = 0; e < N; ++e) {
        const float c = f[2 * e], s = f[2 * e + 1];
        x[e] = first ? (x[e] * c - y[e] * s) : (y[e] * s + x[e] * c);
      }
    }
  }
}

// ------------------------------------------------ banded ragged store (K1, K2, K3) --

struct Item {
  int band, kind, head;  // kind: 0 Q, 1 K, 2 V
  bool act;
};

__device__ __forceinline__ Item decode_item(const BandedParams &p, int j) {
  Item it;
  it.act = j < p.rows_total;
  it.band = (j >= p.rows0) ? 1 : 0;
  int r = j - (it.band ? p.rows0 : 0);
  const BandDev &bd = it.band ? p.band[1] : p.band[0];
  if (r < bd.n_q) {
    it.kind = 0;
  } else if (r < bd.n_q + bd.n_kv) {
    it.kind = 1;
    r -= bd.n_q;
  } else {
    it.kind = 2;
    r -= bd.n_q + bd.n_kv;
  }
  it.head = r;
  return it;
}

template <typename T, int D, bool NORM, int U>
__global__ void __launch_bounds__(kThreads)
    banded_store_kernel(const __grid_constant__ BandedParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / N;
  constexpr int G = kThreads / L;
  static_assert(L <= 32 && 32 % L == 0, "a head row must fit in one warp");

  extern __shared__ uint32_t s_dyn[];
  __shared__ float s_freq[2][2][D];
  __shared__ float s_gamma[NORM ? 4 : 1][NORM ? D : 1];
  __shared__ TokMeta s_meta[2];

  const int tid = threadIdx.x;
  const int li = tid % L, grp = tid / L;
  const bool staged = p.batch <= kSmemSeqs;
  uint32_t *s_offs = s_dyn;
  uint32_t *s_cl = s_dyn + (p.batch + 1);

  bool good = stage_offsets(p.offs, p.batch, p.T, staged, s_offs);
  if (staged)
    for (int i = tid; i < p.n_bands * p.batch; i += kThreads) {
      const int bd = i >= p.batch ? 1 : 0;
      s_cl[i] = __ldg((bd ? p.band[1] : p.band[0]).cache.cache_lengths + (i - bd * p.batch));
    }
  if constexpr (NORM)
    for (int i = tid; i < 2 * p.n_bands * D; i += kThreads) {
      const int which = i / D, d = i % D;
      const BandDev &bd = (which >> 1) ? p.band[1] : p.band[0];
      const T *g = reinterpret_cast<const T *>((which & 1) ? bd.k_gamma : bd.q_gamma);
      s_gamma[which][d] = static_cast<float>(g[d]) + p.weight_offset;
    }
  if (!__syncthreads_and(good)) {
    if (tid == 0) raise(p.err, ROPE_DEVERR_ROW_OFFSETS);
    return;
  }
  const uint32_t *offs = staged ? s_offs : p.offs;

  int buf = 0;
  for (int tok = blockIdx.x; tok < p.T; tok += gridDim.x, buf ^= 1) {
    uint4 v[U];
    Item items[U];
    // loads of the first pass: they depend on the token only
#pragma unroll
    for (int u = 0; u < U; ++u) {
      items[u] = decode_item(p, grp + u * G);
      const Item &it = items[u];
      if (it.act) {
        const BandDev &bd = it.band ? p.band[1] : p.band[0];
        const int64_t col = (it.kind == 0 ? bd.q_col : it.kind == 1 ? bd.k_col : bd.v_col) +
                            (int64_t)it.head * D + li * N;
        v[u] = ld_stream(reinterpret_cast<const T *>(bd.input) + (int64_t)tok * bd.in_stride +
                         col);
      } else {
        v[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // warp 0: sequence, positions, page translation, freqs rows
    if (tid < 32) {
      const int b = find_seq(offs, p.batch, (uint32_t)tok);
      const uint32_t t = (uint32_t)tok - offs[b];
      for (int k = 0; k < p.n_bands; ++k) {
        const BandDev &bd = k ? p.band[1] : p.band[0];
        const uint32_t cl = staged ? s_cl[k * p.batch + b] : __ldg(bd.cache.cache_lengths + b);
        const uint64_t pos = (uint64_t)cl + t;
        int64_t base = 0;
        uint32_t e = 0;
        if (pos >= p.rope.max_seq_len)
          e = ROPE_DEVERR_POSITION;
        else
          e = translate(bd.cache, p.layer, b, pos, &base);
        if (tid == 0) {
          s_meta[buf].ok[k] = (e == 0);
          s_meta[buf].kv_base[k] = base;
          if (e) raise(p.err, e);
        }
        if (e == 0)
          for (int j = tid; j < p.rope.R; j += 32)
            s_freq[buf][k][j] = load_freq(p.rope.table, p.rope.dtype, (int64_t)pos * p.rope.R + j);
      }
    }
    __syncthreads();

    for (int pass = 0;; ++pass) {
      if (pass > 0) {
        const int base = pass * G * U;
        if (base >= p.rows_total) break;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          items[u] = decode_item(p, base + grp + u * G);
          const Item &it = items[u];
          if (it.act) {
            const BandDev &bd = it.band ? p.band[1] : p.band[0];
            const int64_t col =
                (it.kind == 0 ? bd.q_col : it.kind == 1 ? bd.k_col : bd.v_col) +
                (int64_t)it.head * D + li * N;
            v[u] = ld_stream(reinterpret_cast<const T *>(bd.input) +
                             (int64_t)tok * bd.in_stride + col);
          } else {
            v[u] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const Item &it = items[u];
        const BandDev &bd = it.band ? p.band[1] : p.band[0];
        const bool rotate = it.kind != 2;
        float x[N];
        VT::widen(v[u], x);
        if constexpr (NORM) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < N; ++e) ss += x[e] * x[e];
#pragma unroll
          for (int m = L / 2; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
          if (rotate) {
            const float r = rsqrtf(ss * (1.0f / D) + bd.eps);
            const float *g = s_gamma[it.band * 2 + it.kind] + li * N;
#pragma unroll
            for (int e = 0; e < N; ++e) x[e] = x[e] * r * g[e];
          }
        }
        rope_vec<N, L>(x, s_freq[buf][it.band], p.rope, li, rotate);
        if (it.act && s_meta[buf].ok[it.band]) {
          const int c0 = li * N;
          const bool in_rope = c0 >= p.rope.off && c0 < p.rope.off + p.rope.R;
          const uint4 out = (!rotate || (!NORM && !in_rope)) ? v[u] : VT::narrow(x);
          T *dst;
          if (it.kind == 0) {
            dst = reinterpret_cast<T *>(bd.q_out) + (int64_t)tok * bd.q_out_stride +
                  (int64_t)it.head * D + c0;
          } else {
            dst = reinterpret_cast<T *>(it.kind == 1 ? bd.cache.k : bd.cache.v) +
                  s_meta[buf].kv_base[it.band] + (int64_t)it.head * bd.cache.head_stride + c0;
          }
          st_plain(dst, out);
        }
      }
      if ((pass + 1) * G * U >= p.rows_total) break;
    }
  }
}

// --------------------------------------------------------------- BSHD continuous (K4) --

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
};

struct BshdMeta {
  int64_t k_base;
  int32_t valid, ok;
};

template <typename T, int D, int U>
__global__ void __launch_bounds__(kThreads) bshd_rope_kernel(const __grid_constant__ BshdParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / N;
  constexpr int G = kThreads / L;
  __shared__ float s_freq[2][D];
  __shared__ BshdMeta s_meta[2];
  const int tid = threadIdx.x, li = tid % L, grp = tid / L;
  const int64_t n_tok = (int64_t)p.B * p.S;
  int buf = 0;
  for (int64_t tok = blockIdx.x; tok < n_tok; tok += gridDim.x, buf ^= 1) {
    const T *qrow = reinterpret_cast<const T *>(p.q) + tok * p.n_q * D;
    T *orow = reinterpret_cast<T *>(p.out) + tok * p.n_q * D;
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int h = grp + u * G;
      v[u] = h < p.n_q ? ld_stream(qrow + (int64_t)h * D + li * N) : make_uint4(0, 0, 0, 0);
    }
    if (tid < 32) {
      const int b = (int)(tok / p.S), s = (int)(tok % p.S);
      const bool valid = (uint32_t)s < __ldg(p.valid + b);
      uint32_t e = 0;
      int64_t base = 0;
      uint64_t pos = 0;
      if (valid) {
        const uint32_t slot = __ldg(p.lookup + b);
        pos = (uint64_t)__ldg(p.cache_lengths + b) + (uint32_t)s;
        if (slot >= p.num_slots)
          e = ROPE_DEVERR_BATCH;
        else if (pos >= p.rope.max_seq_len || pos >= p.cache_max_seq)
          e = ROPE_DEVERR_POSITION;
        else
          base = (int64_t)slot * p.slot_stride + (int64_t)p.layer * p.layer_stride +
                 (int64_t)pos * p.pos_stride;
      }
      if (tid == 0) {
        s_meta[buf].valid = valid;
        s_meta[buf].ok = (e == 0);
        s_meta[buf].k_base = base;
        if (e) raise(p.err, e);
      }
      if (valid && e == 0)
        for (int j = tid; j < p.rope.R; j += 32)
          s_freq[buf][j] = load_freq(p.rope.table, p.rope.dtype, (int64_t)pos * p.rope.R + j);
    }
    __syncthreads();
    const bool valid = s_meta[buf].valid, ok = s_meta[buf].ok;
    // Q rows: rotate into output (or copy them beyond the valid length)
    for (int base = 0; base < p.n_q; base += G * U) {
      if (base > 0) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int h = base + grp + u * G;
          v[u] = h < p.n_q ? ld_stream(qrow + (int64_t)h * D + li * N) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int h = base + grp + u * G;
        float x[N];
        VT::widen(v[u], x);
        rope_vec<N, L>(x, s_freq[buf], p.rope, li, valid && ok);
        if (h < p.n_q && (ok || !valid)) {
          const int c0 = li * N;
          const bool in_rope = c0 >= p.rope.off && c0 < p.rope.off + p.rope.R;
          st_plain(orow + (int64_t)h * D + c0, (valid && in_rope) ? VT::narrow(x) : v[u]);
        }
      }
    }
    // K rows: rotate in place in the cache (valid tokens only)
    if (valid && ok) {
      T *krow = reinterpret_cast<T *>(p.k) + s_meta[buf].k_base;
      for (int base = 0; base < p.n_kv; base += G * U) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int h = base + grp + u * G;
          v[u] = h < p.n_kv ? ld_plain(krow + (int64_t)h * p.head_stride + li * N)
                            : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int h = base + grp + u * G;
          float x[N];
          VT::widen(v[u], x);
          rope_vec<N, L>(x, s_freq[buf], p.rope, li, true);
          const int c0 = li * N;
          const bool in_rope = c0 >= p.rope.off && c0 < p.rope.off + p.rope.R;
          if (h < p.n_kv && in_rope) st_plain(krow + (int64_t)h * p.head_stride + c0, VT::narrow(x));
        }
      }
    }
  }
}

// ------------------------------------------------------------------- KV radd (K5) --

struct RaddParams {
  const void *a;
  int64_t a_stride;
  int32_t T, n_kv, batch;
  PagedDev cache;
  const uint32_t *offs;
  uint32_t batch_offset, layer;
  uint32_t *err;
};

template <typename T, int D, int U>
__global__ void __launch_bounds__(kThreads) radd_kernel(const __grid_constant__ RaddParams p) {
  using VT = Vec<T>;
  constexpr int N = VT::N;
  constexpr int L = D / N;
  constexpr int G = kThreads / L;
  extern __shared__ uint32_t s_dyn[];
  __shared__ TokMeta s_meta[2];
  const int tid = threadIdx.x, li = tid % L, grp = tid / L;
  const bool staged = p.batch <= kSmemSeqs;
  uint32_t *s_offs = s_dyn;
  uint32_t *s_cl = s_dyn + (p.batch + 1);
  const bool good = stage_offsets(p.offs, p.batch, p.T, staged, s_offs);
  if (staged)
    for (int i = tid; i < p.batch; i += kThreads) {
      const uint64_t seq = (uint64_t)i + p.batch_offset;
      s_cl[i] = seq < p.cache.n_seqs ? __ldg(p.cache.cache_lengths + seq) : 0u;
    }
  if (!__syncthreads_and(good)) {
    if (tid == 0) raise(p.err, ROPE_DEVERR_ROW_OFFSETS);
    return;
  }
  const uint32_t *offs = staged ? s_offs : p.offs;
  const int rows = 2 * p.n_kv;
  const int64_t hidden = (int64_t)p.n_kv * D;
  int buf = 0;
  for (int tok = blockIdx.x; tok < p.T; tok += gridDim.x, buf ^= 1) {
    const T *arow = reinterpret_cast<const T *>(p.a) + (int64_t)tok * p.a_stride;
    if (tid < 32) {
      const int b = find_seq(offs, p.batch, (uint32_t)tok);
      const uint32_t t = (uint32_t)tok - offs[b];
      const uint64_t seq = (uint64_t)b + p.batch_offset;
      uint32_t e = 0;
      int64_t base = 0;
      if (seq >= p.cache.n_seqs) {
        e = ROPE_DEVERR_BATCH;
      } else {
        const uint32_t cl = staged ? s_cl[b] : __ldg(p.cache.cache_lengths + seq);
        e = translate(p.cache, p.layer, (int)seq, (uint64_t)cl + t, &base);
      }
      if (tid == 0) {
        s_meta[buf].ok[0] = (e == 0);
        s_meta[buf].kv_base[0] = base;
        if (e) raise(p.err, e);
      }
    }
    uint4 va[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = grp + u * G;
      va[u] = j < rows ? ld_stream(arow + (j >= p.n_kv ? hidden : 0) + (int64_t)(j % p.n_kv) * D + li * N)
                       : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    if (!s_meta[buf].ok[0]) continue;
    const int64_t kvb = s_meta[buf].kv_base[0];
    for (int base = 0; base < rows; base += G * U) {
      if (base > 0) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int j = base + grp + u * G;
          va[u] = j < rows ? ld_stream(arow + (j >= p.n_kv ? hidden : 0) +
                                       (int64_t)(j % p.n_kv) * D + li * N)
                           : make_uint4(0, 0, 0, 0);
        }
      }
      uint4 vc[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = base + grp + u * G;
        vc[u] = j < rows ? ld_plain(reinterpret_cast<const T *>(j >= p.n_kv ? p.cache.v : p.cache.k) +
                                    kvb + (int64_t)(j % p.n_kv) * p.cache.head_stride + li * N)
                         : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = base + grp + u * G;
        if (j < rows) {
          float xa[N], xc[N];
          VT::widen(va[u], xa);
          VT::widen(vc[u], xc);
#pragma unroll
          for (int e = 0; e < N; ++e) xc[e] = xc[e] + xa[e];
          st_plain(reinterpret_cast<T *>(j >= p.n_kv ? p.cache.v : p.cache.k) + kvb +
                       (int64_t)(j % p.n_kv) * p.cache.head_stride + li * N,
                   VT::narrow(xc));
        }
      }
    }
  }
}

// ------------------------------------------------------------------------ host side --

static int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

// resident CTAs per SM of `kernel` with the largest dynamic shared memory it is launched with
template <typename K>
static int occupancy(K kernel, int &cache) {
  if (cache == 0) {
    int n = 0;
    const size_t dyn = (size_t)(kSmemSeqs + 1 + 2 * kSmemSeqs) * sizeof(uint32_t);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, dyn) != cudaSuccess ||
        n < 1)
      n = 1;
    cache = n;
  }
  return cache;
}

static int elem_bytes(int dtype) {
  return dtype == ROPE_DTYPE_F32 ? 4 : (dtype == ROPE_DTYPE_BF16 || dtype == ROPE_DTYPE_F16) ? 2 : 0;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool stride16(int64_t elems, int eb) { return ((elems * eb) & 15) == 0; }

static bool head_dim_ok(int dtype, int D) {
  if (dtype == ROPE_DTYPE_F32) return D == 64 || D == 128;
  return D == 64 || D == 128 || D == 256;
}

static rope_status_t check_freqs(const rope_freqs_t *f, int dtype, int D, RopeDev *out) {
  if (f == nullptr) return ROPE_ERR_INVALID_ARG;
  if (f->rope_dim < 0 || (f->rope_dim & 1) || f->rope_dim > D || f->max_seq_len < 0)
    return ROPE_ERR_INVALID_ARG;
  if (f->rope_dim > 0 && f->data == nullptr) return ROPE_ERR_INVALID_ARG;
  if (f->dtype != ROPE_DTYPE_F32 && f->dtype != ROPE_DTYPE_BF16 && f->dtype != ROPE_DTYPE_F16)
    return ROPE_ERR_UNSUPPORTED;
  const int off = f->rope_col_offset < 0 ? D - f->rope_dim : f->rope_col_offset;
  if (off + f->rope_dim > D) return ROPE_ERR_INVALID_ARG;
  const int N = 16 / elem_bytes(dtype);
  if (off % N || f->rope_dim % N) return ROPE_ERR_UNSUPPORTED;
  if (!f->interleaved && (f->rope_dim / 2) % N) return ROPE_ERR_UNSUPPORTED;
  out->table = f->data;
  out->dtype = f->dtype == ROPE_DTYPE_F32 ? 2 : f->dtype == ROPE_DTYPE_F16 ? 1 : 0;
  out->max_seq_len = (uint32_t)f->max_seq_len;
  out->R = f->rope_dim;
  out->off = off;
  out->interleaved = f->interleaved ? 1 : 0;
  return ROPE_OK;
}

static rope_status_t check_paged(const rope_paged_cache_t *c, int dtype, uint32_t layer,
                                 bool need_v, PagedDev *out) {
  if (c == nullptr || c->k == nullptr || c->page_table == nullptr || c->cache_lengths == nullptr)
    return ROPE_ERR_INVALID_ARG;
  if (need_v && c->v == nullptr) return ROPE_ERR_INVALID_ARG;
  if (c->n_kv_heads < 0 || c->page_size <= 0 || c->num_pages < 0 || c->num_layers <= 0 ||
      c->max_pages_per_seq < 0 || c->n_seqs < 0 || c->page_table_stride < 0)
    return ROPE_ERR_INVALID_ARG;
  if (layer >= (uint32_t)c->num_layers) return ROPE_ERR_INVALID_ARG;
  if (c->dtype != dtype) return ROPE_ERR_UNSUPPORTED;
  const int eb = elem_bytes(dtype);
  if (!aligned16(c->k) || (c->v && !aligned16(c->v)) || !stride16(c->page_stride, eb) ||
      !stride16(c->layer_stride, eb) || !stride16(c->slot_stride, eb) ||
      !stride16(c->head_stride, eb))
    return ROPE_ERR_UNSUPPORTED;
  out->k = c->k;
  out->v = c->v;
  out->page_stride = c->page_stride;
  out->layer_stride = c->layer_stride;
  out->slot_stride = c->slot_stride;
  out->head_stride = c->head_stride;
  out->page_table = c->page_table;
  out->pt_stride = c->page_table_stride;
  out->cache_lengths = c->cache_lengths;
  out->max_pages = (uint32_t)c->max_pages_per_seq;
  out->page_size = (uint32_t)c->page_size;
  out->num_pages = (uint32_t)c->num_pages;
  out->n_seqs = (uint32_t)c->n_seqs;
  return ROPE_OK;
}

static float round_to_elem(float x, int dtype) {
  if (dtype == ROPE_DTYPE_BF16) return __bfloat162float(__float2bfloat16_rn(x));
  if (dtype == ROPE_DTYPE_F16) return __half2float(__float2half_rn(x));
  return x;
}

static size_t offsets_smem(int batch, int n_bands) {
  return batch <= kSmemSeqs ? (size_t)(batch + 1 + n_bands * batch) * sizeof(uint32_t) : 0;
}

template <typename T, int D, bool NORM, int U>
static rope_status_t launch_banded_t(const BandedParams &p, cudaStream_t st) {
  static int occ = 0;
  auto kern = banded_store_kernel<T, D, NORM, U>;
  const int64_t slots = (int64_t)sm_count() * occupancy(kern, occ);
  const int grid = (int)(slots < p.T ? slots : p.T);
  kern<<<grid, kThreads, offsets_smem(p.batch, p.n_bands), st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ROPE_OK : ROPE_ERR_CUDA;
}

template <typename T, bool NORM>
static rope_status_t launch_banded_d(int D, const BandedParams &p, cudaStream_t st) {
  constexpr int N = Vec<T>::N;
  auto pick = [&](auto dconst) -> rope_status_t {
    constexpr int DD = decltype(dconst)::value;
    constexpr int G = kThreads / (DD / N);
    if ((p.rows_total + G - 1) / G <= 4) return launch_banded_t<T, DD, NORM, 4>(p, st);
    return launch_banded_t<T, DD, NORM, 8>(p, st);
  };
  if (D == 64) return pick(std::integral_constant<int, 64>{});
  if (D == 128) return pick(std::integral_constant<int, 128>{});
  if constexpr (sizeof(T) == 2)
    if (D == 256) return pick(std::integral_constant<int, 256>{});
  return ROPE_ERR_UNSUPPORTED;
}

static rope_status_t launch_banded(int dtype, int D, bool norm, const BandedParams &p,
                                   cudaStream_t st) {
  if (dtype == ROPE_DTYPE_BF16)
    return norm ? launch_banded_d<__nv_bfloat16, true>(D, p, st)
                : launch_banded_d<__nv_bfloat16, false>(D, p, st);
  if (dtype == ROPE_DTYPE_F16)
    return norm ? launch_banded_d<__half, true>(D, p, st) : launch_banded_d<__half, false>(D, p, st);
  if (dtype == ROPE_DTYPE_F32)
    return norm ? launch_banded_d<float, true>(D, p, st) : launch_banded_d<float, false>(D, p, st);
  return ROPE_ERR_UNSUPPORTED;
}

// Validate one band and fill its device descriptor.
static rope_status_t fill_band(BandDev *bd, const void *input, int64_t in_stride, int64_t q_col,
                               int64_t k_col, int64_t v_col, int32_t n_q,
                               const rope_paged_cache_t *kv, const void *qg, const void *kg,
                               float eps, void *q_out, int64_t q_out_stride, int dtype,
                               uint32_t layer, int32_t T, bool norm) {
  if (input == nullptr || q_out == nullptr || n_q < 0 || in_stride < 0 || q_out_stride < 0 ||
      q_col < 0 || k_col < 0)
    return ROPE_ERR_INVALID_ARG;
  if (norm && (qg == nullptr || kg == nullptr)) return ROPE_ERR_INVALID_ARG;
  rope_status_t s = check_paged(kv, dtype, layer, v_col >= 0, &bd->cache);
  if (s != ROPE_OK) return s;
  const int D = kv->head_dim;
  const int eb = elem_bytes(dtype);
  const int64_t rowlen = (int64_t)n_q * D;
  if (T > 1 && (in_stride < q_col + rowlen || q_out_stride < rowlen)) return ROPE_ERR_INVALID_ARG;
  if (!aligned16(input) || !aligned16(q_out) || !stride16(in_stride, eb) ||
      !stride16(q_out_stride, eb) || !stride16(q_col, eb) || !stride16(k_col, eb) ||
      (v_col >= 0 && !stride16(v_col, eb)))
    return ROPE_ERR_UNSUPPORTED;
  bd->input = input;
  bd->in_stride = in_stride;
  bd->q_col = q_col;
  bd->k_col = k_col;
  bd->v_col = v_col;
  bd->n_q = n_q;
  bd->n_kv = kv->n_kv_heads;
  bd->n_v = v_col >= 0 ? kv->n_kv_heads : 0;
  bd->q_out = q_out;
  bd->q_out_stride = q_out_stride;
  bd->q_gamma = qg;
  bd->k_gamma = kg;
  bd->eps = eps;
  return ROPE_OK;
}

static rope_status_t common_checks(int dtype, int D, const uint32_t *offs, int32_t batch,
                                   int32_t T) {
  if (offs == nullptr || batch < 0 || T < 0) return ROPE_ERR_INVALID_ARG;
  if (T > 0 && batch == 0) return ROPE_ERR_INVALID_ARG;
  if (elem_bytes(dtype) == 0 || !head_dim_ok(dtype, D)) return ROPE_ERR_UNSUPPORTED;
  return ROPE_OK;
}

}  // namespace rs

using namespace rs;

extern "C" {

const char *rope_status_string(rope_status_t s) {
  switch (s) {
    case ROPE_OK: return "ok";
    case ROPE_ERR_INVALID_ARG: return "invalid argument";
    case ROPE_ERR_UNSUPPORTED: return "unsupported dtype, head_dim, rope geometry or alignment";
    case ROPE_ERR_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

rope_status_t rope_split_store_paged_ragged(const void *qkv, int64_t qkv_row_stride,
                                            int32_t total_tokens, int32_t n_q_heads,
                                            const uint32_t *input_row_offsets, int32_t batch,
                                            const rope_freqs_t *freqs,
                                            const rope_paged_cache_t *kv, uint32_t layer_idx,
                                            void *q_out, int64_t q_out_row_stride,
                                            uint32_t *err_word, rope_stream_t stream) {
  if (kv == nullptr) return ROPE_ERR_INVALID_ARG;
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  const int dtype = kv->dtype, D = kv->head_dim;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  if (batch > kv->n_seqs || n_q_heads < 0) return ROPE_ERR_INVALID_ARG;
  BandedParams p{};
  s = check_freqs(freqs, dtype, D, &p.rope);
  if (s != ROPE_OK) return s;
  const int64_t Hq = n_q_heads, Hk = kv->n_kv_heads;
  s = fill_band(&p.band[0], qkv, qkv_row_stride, 0, Hq * D, (Hq + Hk) * D, n_q_heads, kv,
                nullptr, nullptr, 0.f, q_out, q_out_row_stride, dtype, layer_idx, total_tokens,
                false);
  if (s != ROPE_OK) return s;
  if (total_tokens > 1 && qkv_row_stride < (Hq + 2 * Hk) * D) return ROPE_ERR_INVALID_ARG;
  if (total_tokens == 0) return ROPE_OK;
  p.n_bands = 1;
  p.rows0 = p.rows_total = (int32_t)(Hq + 2 * Hk);
  p.offs = input_row_offsets;
  p.batch = batch;
  p.T = total_tokens;
  p.layer = layer_idx;
  p.err = err_word;
  if (p.rows_total == 0) return ROPE_OK;
  return launch_banded(dtype, D, false, p, (cudaStream_t)stream);
}

rope_status_t fused_qk_rmsnorm_rope_paged(const void *qkv, int64_t qkv_row_stride,
                                          int32_t total_tokens, int32_t n_q_heads,
                                          const uint32_t *input_row_offsets, int32_t batch,
                                          const rope_freqs_t *freqs,
                                          const rope_paged_cache_t *kv, const void *q_gamma,
                                          const void *k_gamma, float epsilon,
                                          float weight_offset, int32_t multiply_before_cast,
                                          uint32_t layer_idx, void *q_out,
                                          int64_t q_out_row_stride, uint32_t *err_word,
                                          rope_stream_t stream) {
  if (kv == nullptr) return ROPE_ERR_INVALID_ARG;
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  const int dtype = kv->dtype, D = kv->head_dim;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  if (batch > kv->n_seqs || n_q_heads < 0) return ROPE_ERR_INVALID_ARG;
  if (multiply_before_cast != 1) return ROPE_ERR_UNSUPPORTED;
  BandedParams p{};
  s = check_freqs(freqs, dtype, D, &p.rope);
  if (s != ROPE_OK) return s;
  const int64_t Hq = n_q_heads, Hk = kv->n_kv_heads;
  s = fill_band(&p.band[0], qkv, qkv_row_stride, 0, Hq * D, (Hq + Hk) * D, n_q_heads, kv,
                q_gamma, k_gamma, epsilon, q_out, q_out_row_stride, dtype, layer_idx,
                total_tokens, true);
  if (s != ROPE_OK) return s;
  if (total_tokens > 1 && qkv_row_stride < (Hq + 2 * Hk) * D) return ROPE_ERR_INVALID_ARG;
  if (total_tokens == 0) return ROPE_OK;
  p.n_bands = 1;
  p.rows0 = p.rows_total = (int32_t)(Hq + 2 * Hk);
  p.offs = input_row_offsets;
  p.batch = batch;
  p.T = total_tokens;
  p.layer = layer_idx;
  p.err = err_word;
  p.weight_offset = round_to_elem(weight_offset, dtype);
  if (p.rows_total == 0) return ROPE_OK;
  return launch_banded(dtype, D, true, p, (cudaStream_t)stream);
}

rope_status_t fused_dual_qk_rmsnorm_rope_paged(const rope_norm_band_t *main_band,
                                               const rope_norm_band_t *index_band,
                                               const uint32_t *input_row_offsets,
                                               int32_t batch, int32_t total_tokens,
                                               const rope_freqs_t *freqs, float weight_offset,
                                               int32_t multiply_before_cast, uint32_t layer_idx,
                                               uint32_t *err_word, rope_stream_t stream) {
  if (main_band == nullptr || index_band == nullptr || main_band->cache == nullptr ||
      index_band->cache == nullptr)
    return ROPE_ERR_INVALID_ARG;
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  const rope_paged_cache_t *mc = main_band->cache, *ic = index_band->cache;
  // the rope geometry must agree across the bands
  if (mc->dtype != ic->dtype || mc->head_dim != ic->head_dim) return ROPE_ERR_INVALID_ARG;
  const int dtype = mc->dtype, D = mc->head_dim;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  if (batch > mc->n_seqs || batch > ic->n_seqs) return ROPE_ERR_INVALID_ARG;
  if (multiply_before_cast != 1) return ROPE_ERR_UNSUPPORTED;
  BandedParams p{};
  s = check_freqs(freqs, dtype, D, &p.rope);
  if (s != ROPE_OK) return s;
  const rope_norm_band_t *bands[2] = {main_band, index_band};
  int32_t rows[2];
  for (int k = 0; k < 2; ++k) {
    const rope_norm_band_t *b = bands[k];
    s = fill_band(&p.band[k], b->input, b->input_row_stride, b->q_col, b->k_col, b->v_col,
                  b->n_q_heads, b->cache, b->q_gamma, b->k_gamma, b->epsilon, b->q_out,
                  b->q_out_row_stride, dtype, layer_idx, total_tokens, true);
    if (s != ROPE_OK) return s;
    const int64_t Hk = b->cache->n_kv_heads;
    const int64_t need = b->k_col + Hk * D;
    if (total_tokens > 1 && (b->input_row_stride < need ||
                             (b->v_col >= 0 && b->input_row_stride < b->v_col + Hk * D)))
      return ROPE_ERR_INVALID_ARG;
    rows[k] = p.band[k].n_q + p.band[k].n_kv + p.band[k].n_v;
  }
  if (total_tokens == 0) return ROPE_OK;
  p.n_bands = 2;
  p.rows0 = rows[0];
  p.rows_total = rows[0] + rows[1];
  p.offs = input_row_offsets;
  p.batch = batch;
  p.T = total_tokens;
  p.layer = layer_idx;
  p.err = err_word;
  p.weight_offset = round_to_elem(weight_offset, dtype);
  if (p.rows_total == 0) return ROPE_OK;
  return launch_banded(dtype, D, true, p, (cudaStream_t)stream);
}

}  // extern "C"

namespace rs {

template <typename T, int D, int U>
static rope_status_t launch_bshd_t(const BshdParams &p, cudaStream_t st) {
  static int occ = 0;
  auto kern = bshd_rope_kernel<T, D, U>;
  const int64_t n_tok = (int64_t)p.B * p.S;
  const int64_t slots = (int64_t)sm_count() * occupancy(kern, occ);
  const int grid = (int)(slots < n_tok ? slots : n_tok);
  kern<<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ROPE_OK : ROPE_ERR_CUDA;
}

template <typename T>
static rope_status_t launch_bshd_d(int D, const BshdParams &p, cudaStream_t st) {
  if (D == 64) return launch_bshd_t<T, 64, 2>(p, st);
  if (D == 128) return launch_bshd_t<T, 128, 2>(p, st);
  if constexpr (sizeof(T) == 2)
    if (D == 256) return launch_bshd_t<T, 256, 2>(p, st);
  return ROPE_ERR_UNSUPPORTED;
}

template <typename T, int D, int U>
static rope_status_t launch_radd_t(const RaddParams &p, cudaStream_t st) {
  static int occ = 0;
  auto kern = radd_kernel<T, D, U>;
  const int64_t slots = (int64_t)sm_count() * occupancy(kern, occ);
  const int grid = (int)(slots < p.T ? slots : p.T);
  kern<<<grid, kThreads, offsets_smem(p.batch, 1), st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ROPE_OK : ROPE_ERR_CUDA;
}

template <typename T>
static rope_status_t launch_radd_d(int D, const RaddParams &p, cudaStream_t st) {
  if (D == 64) return launch_radd_t<T, 64, 2>(p, st);
  if (D == 128) return launch_radd_t<T, 128, 2>(p, st);
  if constexpr (sizeof(T) == 2)
    if (D == 256) return launch_radd_t<T, 256, 2>(p, st);
  return ROPE_ERR_UNSUPPORTED;
}

}  // namespace rs

extern "C" {

rope_status_t qk_rope_bshd_continuous(const void *q_proj, int32_t batch, int32_t seq_len,
                                      int32_t n_q_heads, int32_t head_dim,
                                      const rope_cont_cache_t *kv, const rope_freqs_t *freqs,
                                      uint32_t layer_idx, const uint32_t *valid_lengths,
                                      void *output, uint32_t *err_word, rope_stream_t stream) {
  if (batch >= 0 && seq_len >= 0 && (int64_t)batch * seq_len == 0) return ROPE_OK;
  if (q_proj == nullptr || kv == nullptr || valid_lengths == nullptr || output == nullptr ||
      kv->k == nullptr || kv->lookup_table == nullptr || kv->cache_lengths == nullptr)
    return ROPE_ERR_INVALID_ARG;
  if (batch < 0 || seq_len < 0 || n_q_heads < 0 || kv->n_kv_heads < 0 || kv->num_slots < 0 ||
      kv->num_layers <= 0 || kv->max_seq_len < 0 || batch > kv->n_seqs)
    return ROPE_ERR_INVALID_ARG;
  if (kv->head_dim != head_dim || layer_idx >= (uint32_t)kv->num_layers) return ROPE_ERR_INVALID_ARG;
  const int dtype = kv->dtype, D = head_dim;
  if (elem_bytes(dtype) == 0 || !head_dim_ok(dtype, D)) return ROPE_ERR_UNSUPPORTED;
  BshdParams p{};
  rope_status_t s = check_freqs(freqs, dtype, D, &p.rope);
  if (s != ROPE_OK) return s;
  const int eb = elem_bytes(dtype);
  if (!aligned16(q_proj) || !aligned16(output) || !aligned16(kv->k) ||
      !stride16(kv->slot_stride, eb) || !stride16(kv->layer_stride, eb) ||
      !stride16(kv->pos_stride, eb) || !stride16(kv->head_stride, eb))
    return ROPE_ERR_UNSUPPORTED;
  if ((int64_t)batch * seq_len == 0) return ROPE_OK;
  p.q = q_proj;
  p.out = output;
  p.B = batch;
  p.S = seq_len;
  p.n_q = n_q_heads;
  p.n_kv = kv->n_kv_heads;
  p.k = kv->k;
  p.slot_stride = kv->slot_stride;
  p.layer_stride = kv->layer_stride;
  p.pos_stride = kv->pos_stride;
  p.head_stride = kv->head_stride;
  p.lookup = kv->lookup_table;
  p.cache_lengths = kv->cache_lengths;
  p.valid = valid_lengths;
  p.num_slots = (uint32_t)kv->num_slots;
  p.cache_max_seq = (uint32_t)kv->max_seq_len;
  p.layer = layer_idx;
  p.err = err_word;
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == ROPE_DTYPE_BF16) return launch_bshd_d<__nv_bfloat16>(D, p, st);
  if (dtype == ROPE_DTYPE_F16) return launch_bshd_d<__half>(D, p, st);
  return launch_bshd_d<float>(D, p, st);
}

rope_status_t kv_cache_radd(const void *a, int64_t a_row_stride, int32_t total_tokens,
                            const rope_paged_cache_t *kv, const uint32_t *input_row_offsets,
                            int32_t batch, uint32_t batch_offset, uint32_t layer_idx,
                            uint32_t *err_word, rope_stream_t stream) {
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  if (kv == nullptr || a == nullptr) return ROPE_ERR_INVALID_ARG;
  const int dtype = kv->dtype, D = kv->head_dim;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  RaddParams p{};
  s = check_paged(kv, dtype, layer_idx, true, &p.cache);
  if (s != ROPE_OK) return s;
  const int eb = elem_bytes(dtype);
  const int64_t hidden = (int64_t)kv->n_kv_heads * D;
  if (a_row_stride < 0 || (total_tokens > 1 && a_row_stride < 2 * hidden)) return ROPE_ERR_INVALID_ARG;
  if (!aligned16(a) || !stride16(a_row_stride, eb)) return ROPE_ERR_UNSUPPORTED;
  if (total_tokens == 0 || hidden == 0) return ROPE_OK;
  p.a = a;
  p.a_stride = a_row_stride;
  p.T = total_tokens;
  p.n_kv = kv->n_kv_heads;
  p.batch = batch;
  p.offs = input_row_offsets;
  p.batch_offset = batch_offset;
  p.layer = layer_idx;
  p.err = err_word;
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == ROPE_DTYPE_BF16) return launch_radd_d<__nv_bfloat16>(D, p, st);
  if (dtype == ROPE_DTYPE_F16) return launch_radd_d<__half>(D, p, st);
  return launch_radd_d<float>(D, p, st);
}

}  // extern "C"
