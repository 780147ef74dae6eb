// rope_store.cu -- host side of rope_store.h: argument checks, launch shaping, dispatch.
//
// Kernels (see the headers):
//   banded.cuh  ragged paged store, optional per-head RMSNorm, one or two bands: persistent
//               CTAs, a producer warp bulk-copying token rows into a shared-memory ring,
//               four, six or eight consumer warps rotating / normalising in place (an FP8
//               cache's codes to stage regions of their own), a storer warp bulk-copying
//               the results out;
//   radd.cuh    in-place cache add on the same staging scheme;
//   bshd.cuh    decode-shaped BSHD RoPE with in-place K, one CTA per token;
//   gemv_norm.cuh  one-row GEMV + partial RMSNorm, one or a few rows of W per CTA, the last
//               CTA normalising.
#include "../../include/rope_store.h"
#include "banded.cuh"
#include "bshd.cuh"
#include "gemv_norm.cuh"
#include "radd.cuh"

#include <cuda_runtime.h>

#include <atomic>
#include <initializer_list>
#include <mutex>
#include <type_traits>

namespace rs {

constexpr int kSmemSeqs = 1024;         // batches up to this size stage offsets in smem
constexpr int kMaxStages = 8;

// Launch shapes of the banded kernel (measured on B200 over the named workloads): consumer
// warps, store lag and the shared memory given to a CTA's stage ring.
struct BandedShape {
  int cw, lag, ring_kb;
};
#ifndef ROPE_LIGHT_CW
#define ROPE_LIGHT_CW 4
#define ROPE_LIGHT_LAG 2
#define ROPE_LIGHT_RING 64
#endif
// <= 64 Q+K head rows a token, no norm
constexpr BandedShape kLightShape = {ROPE_LIGHT_CW, ROPE_LIGHT_LAG, ROPE_LIGHT_RING};
// RMSNorm or many heads: six or eight consumer warps, whichever takes fewer passes over a
// token's head rows (six on a tie: the per-head-norm workload's 72 rows take three passes
// either way; eight on the dual-band one, 81 rows in three passes instead of four).  One
// CTA an SM with ten or twelve consumer warps and an eight-stage ring ran 140-150 us on the
// per-head norm and 372-389 us on the dual band, against 119 and 248 us: two producers and
// two storers an SM keep more copies in flight.
#ifndef ROPE_MID_CW
#define ROPE_MID_CW 6
#define ROPE_MID_LAG 0
#define ROPE_MID_RING 96
#endif
#ifndef ROPE_HEAVY_CW
#define ROPE_HEAVY_CW 8
#define ROPE_HEAVY_LAG 0
#define ROPE_HEAVY_RING 96
#endif
constexpr BandedShape kMidShape = {ROPE_MID_CW, ROPE_MID_LAG, ROPE_MID_RING};
constexpr BandedShape kHeavyShape = {ROPE_HEAVY_CW, ROPE_HEAVY_LAG, ROPE_HEAVY_RING};

enum ShapeId { kLight = 0, kMid = 1, kHeavy = 2 };

static int passes(const BandedParams &p, int D, int cw) {
  const int rows_per_pass = 32 * cw / (D / (2 * (16 / p.elem_bytes)));
  return (p.work_total + rows_per_pass - 1) / rows_per_pass;
}

static ShapeId pick_shape(const BandedParams &p, int D, bool norm) {
  // few head rows without norm (Q, K and, for an FP8 cache, V), or Q converted to another
  // type: the light shape
  if (!norm && (p.work_total <= 64 || p.band[0].q_conv)) return kLight;
  return passes(p, D, kMidShape.cw) <= passes(p, D, kHeavyShape.cw) ? kMid : kHeavy;
}

static const BandedShape &shape_of(ShapeId id) {
  return id == kLight ? kLightShape : id == kMid ? kMidShape : kHeavyShape;
}

// ------------------------------------------------------------------------ host side --

// launch-overlap mode of every launch that follows (rope_set_launch_overlap)
static std::atomic<int> g_overlap{kOverlapPdl};
// the stall test of the launches that follow (rope_set_stall_test): 0 off, else the limit of
// the wait nothing completes, in nanoseconds
static std::atomic<uint32_t> g_stall_test_ns{0};

// Launch `kern` with one parameter block; modes 1 and 2 launch it as a programmatic
// dependent of the previous kernel in the stream.
template <typename K, typename P>
static rope_status_t launch(K kern, int grid, int threads, size_t smem, cudaStream_t st,
                            const P &p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  if (p.overlap != kOverlapOff) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return ROPE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ROPE_OK : ROPE_ERR_CUDA;
}

static bool sched_ok(const uint32_t *sched) {
  return (reinterpret_cast<uintptr_t>(sched) & 3u) == 0;
}

static int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

// Launch-shape cache of one kernel: the dynamic shared memory it was last sized for and
// the resident CTAs per SM that gives.
struct ShapeCache {
  size_t smem = 0;
  int occ = 0;
  size_t attr_smem = 0;
};

template <typename K>
static int resident_ctas(K kernel, int threads, size_t smem, ShapeCache &c) {
  if (smem > 48 * 1024 && smem > c.attr_smem) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return 0;
    c.attr_smem = smem;
  }
  if (c.occ == 0 || c.smem != smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
      return 0;
    c.smem = smem;
    c.occ = n;
  }
  return c.occ;
}

static int elem_bytes(int dtype) {
  return dtype == ROPE_DTYPE_F32 ? 4 : (dtype == ROPE_DTYPE_BF16 || dtype == ROPE_DTYPE_F16) ? 2 : 0;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool stride16(int64_t elems, int eb) { return ((elems * eb) & 15) == 0; }
static int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

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
  // freqs rows are moved in 16-byte units
  if (f->rope_dim > 0 && (!aligned16(f->data) || (f->rope_dim * elem_bytes(f->dtype)) % 16))
    return ROPE_ERR_UNSUPPORTED;
  out->table = f->data;
  out->dtype = f->dtype == ROPE_DTYPE_F32 ? 2 : f->dtype == ROPE_DTYPE_F16 ? 1 : 0;
  out->max_seq_len = (uint32_t)f->max_seq_len;
  out->R = f->rope_dim;
  out->off = off;
  out->interleaved = f->interleaved ? 1 : 0;
  return ROPE_OK;
}

// allow_fp8: the cache may hold E4M3 codes (with its scales) instead of the input's type
static rope_status_t check_paged(const rope_paged_cache_t *c, int dtype, uint32_t layer,
                                 bool need_v, PagedDev *out, bool allow_fp8 = false) {
  if (c == nullptr || c->k == nullptr || c->page_table == nullptr || c->cache_lengths == nullptr)
    return ROPE_ERR_INVALID_ARG;
  if (need_v && c->v == nullptr) return ROPE_ERR_INVALID_ARG;
  if (c->n_kv_heads < 0 || c->page_size <= 0 || c->num_pages < 0 || c->num_layers <= 0 ||
      c->max_pages_per_seq < 0 || c->n_seqs < 0 || c->page_table_stride < 0)
    return ROPE_ERR_INVALID_ARG;
  if (layer >= (uint32_t)c->num_layers) return ROPE_ERR_INVALID_ARG;
  const bool fp8 = c->dtype == ROPE_DTYPE_FP8_E4M3;
  if (c->dtype != dtype && !(allow_fp8 && fp8)) return ROPE_ERR_UNSUPPORTED;
  if (fp8 && (c->k_scale == nullptr || (c->v != nullptr && c->v_scale == nullptr)))
    return ROPE_ERR_INVALID_ARG;
  const int eb = fp8 ? 1 : elem_bytes(dtype);
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

// Validate one band and fill its device descriptor (staging segments included; the
// band's stage offset is set by the caller).  k_col < 0: K is read from the cache slot.
static rope_status_t fill_band(BandDev *bd, const void *input, int64_t in_stride, int64_t q_col,
                               int64_t k_col, int64_t v_col, int32_t n_q,
                               const rope_paged_cache_t *kv, const void *qg, const void *kg,
                               float eps, void *q_out, int64_t q_out_stride, int dtype,
                               uint32_t layer, bool norm, int q_dtype = -1) {
  if (input == nullptr || q_out == nullptr || n_q < 0 || in_stride < 0 || q_out_stride < 0 ||
      q_col < 0)
    return ROPE_ERR_INVALID_ARG;
  const bool k_inplace = k_col < 0;
  if (norm && (qg == nullptr || kg == nullptr)) return ROPE_ERR_INVALID_ARG;
  rope_status_t s = check_paged(kv, dtype, layer, v_col >= 0, &bd->cache, true);
  if (s != ROPE_OK) return s;
  const int64_t D = kv->head_dim, Hk = kv->n_kv_heads;
  const int eb = elem_bytes(dtype);
  if (q_dtype < 0) q_dtype = dtype;
  const int qeb = elem_bytes(q_dtype);
  if (qeb == 0 || (norm && q_dtype != dtype)) return ROPE_ERR_UNSUPPORTED;
  const int64_t nv = v_col >= 0 ? Hk : 0;
  if (in_stride < q_col + n_q * D || (!k_inplace && in_stride < k_col + Hk * D) ||
      (v_col >= 0 && in_stride < v_col + Hk * D) || q_out_stride < n_q * D)
    return ROPE_ERR_INVALID_ARG;
  if (!aligned16(input) || !aligned16(q_out) || !stride16(in_stride, eb) ||
      !stride16(q_out_stride, qeb) || !stride16(q_col, eb) ||
      (!k_inplace && !stride16(k_col, eb)) || (v_col >= 0 && !stride16(v_col, eb)))
    return ROPE_ERR_UNSUPPORTED;
  bd->input = input;
  bd->in_stride = in_stride;
  bd->q_col = q_col;
  bd->k_col = k_col;
  bd->v_col = v_col;
  bd->n_q = n_q;
  bd->n_kv = (int32_t)Hk;
  bd->n_v = (int32_t)nv;
  bd->q_out = q_out;
  bd->q_out_stride = q_out_stride;
  bd->q_gamma = qg;
  bd->k_gamma = kg;
  bd->eps = eps;
  bd->kv_contig = kv->head_stride == D ? 1 : 0;
  bd->k_inplace = k_inplace ? 1 : 0;
  bd->kv8 = kv->dtype == ROPE_DTYPE_FP8_E4M3 ? 1 : 0;
  if (bd->kv8 && k_inplace) return ROPE_ERR_UNSUPPORTED;  // K would have to be decoded
  bd->k_scale = kv->k_scale;
  bd->v_scale = kv->v_scale;
  bd->q_conv = q_dtype != dtype ? 1 : 0;
  bd->q_dtype = q_dtype == ROPE_DTYPE_F32 ? 2 : q_dtype == ROPE_DTYPE_F16 ? 1 : 0;
  bd->q_eb = qeb;
  // staging segments: Q, K, V blocks (merged when adjacent in the input row); an in-place
  // K block keeps its place in the stage but is loaded from the cache
  const int64_t cols[3] = {q_col, k_col, v_col};
  const int64_t cnt[3] = {n_q * D, Hk * D, nv * D};
  int nseg = 0;
  int64_t dst = 0, next_col = -1;
  for (int q = 0; q < 3; ++q) {
    if (cnt[q] == 0) continue;
    if (q == 1 && k_inplace) {
      dst += cnt[q] * eb;
      next_col = -1;
      continue;
    }
    if (nseg > 0 && cols[q] == next_col) {
      bd->seg_bytes[nseg - 1] += (int32_t)(cnt[q] * eb);
    } else {
      bd->seg_col[nseg] = cols[q];
      bd->seg_bytes[nseg] = (int32_t)(cnt[q] * eb);
      bd->seg_dst[nseg] = (int32_t)dst;  // relative to the band's block, fixed up later
      ++nseg;
    }
    next_col = cols[q] + cnt[q];
    dst += cnt[q] * eb;
  }
  bd->nseg = nseg;
  bd->tx_bytes = (int32_t)dst;
  return ROPE_OK;
}

static rope_status_t common_checks(int dtype, int D, const uint32_t *offs, int32_t batch,
                                   int32_t T) {
  if (offs == nullptr || batch < 0 || T < 0) return ROPE_ERR_INVALID_ARG;
  if (T > 0 && batch == 0) return ROPE_ERR_INVALID_ARG;
  if (elem_bytes(dtype) == 0 || !head_dim_ok(dtype, D)) return ROPE_ERR_UNSUPPORTED;
  return ROPE_OK;
}

static int elem_bytes_of(const BandedParams &p) { return p.elem_bytes; }

// Shared-memory layout of the banded kernel: [stages | full, empty barriers | metadata |
// gammas | offsets, cache lengths].  Returns the dynamic shared memory size.
static size_t layout_banded(BandedParams &p, int D, bool norm, const BandedShape &sh) {
  const int kConsumers = 32 * sh.cw, kStoreLag = sh.lag, kStageTarget = sh.ring_kb << 10;
  int64_t off = 0;
  for (int k = 0; k < p.n_bands; ++k) {
    BandDev &bd = p.band[k];
    bd.smem_off = (int32_t)off;
    for (int q = 0; q < bd.nseg; ++q) bd.seg_dst[q] += (int32_t)off;
    off = round_up(off + bd.tx_bytes, 16);
  }
  p.f_row_bytes = p.rope.R * (p.rope.dtype == 2 ? 4 : 2);
  for (int k = 0; k < p.n_bands; ++k) {
    p.band[k].f_off = (int32_t)off;
    off = round_up(off + p.f_row_bytes, 16);
  }
  for (int k = 0; k < p.n_bands; ++k) {  // converted Q rows, FP8 K and V rows
    BandDev &bd = p.band[k];
    bd.qo_off = (int32_t)off;
    if (bd.q_conv) off = round_up(off + (int64_t)bd.n_q * D * bd.q_eb, 16);
    bd.k8_off = (int32_t)off;
    if (bd.kv8) off = round_up(off + (int64_t)bd.n_kv * D, 16);
    bd.v8_off = (int32_t)off;
    if (bd.kv8) off = round_up(off + (int64_t)bd.n_v * D, 16);
  }
  p.stage_bytes = (int32_t)round_up(off, 128);
  int S = (int)(kStageTarget / p.stage_bytes);
  // the storer holds up to kStoreLag + 1 stages; keep at least two for loading / compute
  S = S < kStoreLag + 3 ? kStoreLag + 3 : (S > kMaxStages ? kMaxStages : S);
  if (S < 3) S = 3;
  p.S = S;
  int64_t total = (int64_t)S * p.stage_bytes;
  p.bar_off = (int32_t)total;
  total += 3 * S * 8;  // full, done, empty
  p.meta_off = (int32_t)round_up(total, 16);
  total = p.meta_off + S * (int64_t)sizeof(StageMeta);
  p.gamma_off = (int32_t)round_up(total, 16);
  total = p.gamma_off + (norm ? 4 * D * 4 : 0);
  p.items_off = (int32_t)round_up(total, 16);
  const int G = kConsumers / (D / (2 * (16 / elem_bytes_of(p))));  // lanes per row: D / 2N
  total = p.items_off + (int64_t)((p.work_total + G - 1) / G) * kConsumers * 4;
  p.offs_off = (int32_t)round_up(total, 16);
  p.staged = p.batch <= kSmemSeqs;
  total = p.offs_off + (p.staged ? (int64_t)(p.batch + 1 + p.n_bands * p.batch) * 4 : 0);
  return (size_t)round_up(total, 128);
}

template <typename T, int D, bool NORM, int CW, int LAG, bool EXT = false>
static rope_status_t launch_banded_t(const BandedParams &p, size_t smem, cudaStream_t st) {
  static ShapeCache cache;
  auto kern = banded_store_kernel<T, D, NORM, CW, LAG, EXT>;
  const int occ = resident_ctas(kern, pipe_threads<CW>(), smem, cache);
  if (occ <= 0) return ROPE_ERR_UNSUPPORTED;  // the stage ring does not fit
  const int64_t slots = (int64_t)sm_count() * occ;
  const int grid = (int)(slots < p.T ? slots : p.T);
  return launch(kern, grid, pipe_threads<CW>(), smem, st, p);
}

template <typename T, int D, bool NORM>
static rope_status_t launch_banded_s(ShapeId id, const BandedParams &p, size_t smem,
                                     cudaStream_t st) {
  // Q in another element type or an FP8 cache: the instantiation with those outputs
  const bool ext = p.band[0].q_conv || p.band[0].kv8 || (p.n_bands > 1 && p.band[1].kv8);
  if constexpr (!NORM) {  // (the light shape is never picked for a launch with the norm)
    if (id == kLight)
      return ext ? launch_banded_t<T, D, NORM, kLightShape.cw, kLightShape.lag, true>(p, smem,
                                                                                      st)
                 : launch_banded_t<T, D, NORM, kLightShape.cw, kLightShape.lag>(p, smem, st);
  }
  if (id == kMid)
    return ext ? launch_banded_t<T, D, NORM, kMidShape.cw, kMidShape.lag, true>(p, smem, st)
               : launch_banded_t<T, D, NORM, kMidShape.cw, kMidShape.lag>(p, smem, st);
  return ext ? launch_banded_t<T, D, NORM, kHeavyShape.cw, kHeavyShape.lag, true>(p, smem, st)
             : launch_banded_t<T, D, NORM, kHeavyShape.cw, kHeavyShape.lag>(p, smem, st);
}

template <typename T, bool NORM>
static rope_status_t launch_banded_d(int D, ShapeId id, const BandedParams &p, size_t smem,
                                     cudaStream_t st) {
  if (D == 64) return launch_banded_s<T, 64, NORM>(id, p, smem, st);
  if (D == 128) return launch_banded_s<T, 128, NORM>(id, p, smem, st);
  if constexpr (sizeof(T) == 2)
    if (D == 256) return launch_banded_s<T, 256, NORM>(id, p, smem, st);
  return ROPE_ERR_UNSUPPORTED;
}

static rope_status_t launch_banded(int dtype, int D, bool norm, BandedParams &p,
                                   cudaStream_t st) {
  p.elem_bytes = elem_bytes(dtype);
  ShapeId id = pick_shape(p, D, norm);
  const BandedParams unplaced = p;  // layout_banded places the stage offsets in p
  size_t smem = layout_banded(p, D, norm, shape_of(id));
  if (smem > 227 * 1024 && id == kLight) {  // stages too large for its ring of >= 5
    p = unplaced;
    id = kHeavy;
    smem = layout_banded(p, D, norm, kHeavyShape);
  }
  if (smem > 227 * 1024) return ROPE_ERR_UNSUPPORTED;
  if (dtype == ROPE_DTYPE_BF16)
    return norm ? launch_banded_d<__nv_bfloat16, true>(D, id, p, smem, st)
                : launch_banded_d<__nv_bfloat16, false>(D, id, p, smem, st);
  if (dtype == ROPE_DTYPE_F16)
    return norm ? launch_banded_d<__half, true>(D, id, p, smem, st)
                : launch_banded_d<__half, false>(D, id, p, smem, st);
  if (dtype == ROPE_DTYPE_F32)
    return norm ? launch_banded_d<float, true>(D, id, p, smem, st)
                : launch_banded_d<float, false>(D, id, p, smem, st);
  return ROPE_ERR_UNSUPPORTED;
}

template <typename T, int D>
static rope_status_t launch_bshd_t(const BshdParams &p, cudaStream_t st) {
  constexpr int G = kBshdThreads / (D / Vec<T>::N);
  const int64_t n_tok = (int64_t)p.B * p.S;
  const int64_t cap = (int64_t)1 << 30;
  const int grid = (int)(n_tok < cap ? n_tok : cap);
  if (p.n_q <= 2 * G && p.n_kv <= G)
    return launch(bshd_rope_kernel<T, D, 2, 1>, grid, kBshdThreads, 0, st, p);
  return launch(bshd_rope_kernel<T, D, 4, 2>, grid, kBshdThreads, 0, st, p);
}

template <typename T>
static rope_status_t launch_bshd_d(int D, const BshdParams &p, cudaStream_t st) {
  if (D == 64) return launch_bshd_t<T, 64>(p, st);
  if (D == 128) return launch_bshd_t<T, 128>(p, st);
  if constexpr (sizeof(T) == 2)
    if (D == 256) return launch_bshd_t<T, 256>(p, st);
  return ROPE_ERR_UNSUPPORTED;
}

// Launch shape of the radd kernel (consumer warps, store lag, stage-ring shared memory),
// measured on B200 over the radd workload: three stages a CTA and four CTAs an SM (65.7 us)
// beat four stages and three CTAs (76.0 us); the producer and storer threads of more CTAs
// keep more bulk copies in flight.
#ifndef ROPE_RADD_CW
#define ROPE_RADD_CW 4
#define ROPE_RADD_LAG 0
#define ROPE_RADD_RING 48
#endif
constexpr BandedShape kRaddShape = {ROPE_RADD_CW, ROPE_RADD_LAG, ROPE_RADD_RING};

static size_t layout_radd(RaddParams &p, int D, int eb) {
  const int kStageTarget = kRaddShape.ring_kb << 10;
  p.stage_bytes = (int32_t)round_up(4LL * p.n_kv * D * eb, 128);
  int S = (int)(kStageTarget / p.stage_bytes);
  // the storer holds up to lag + 1 stages; keep at least two for loading / compute
  S = S < kRaddShape.lag + 3 ? kRaddShape.lag + 3 : (S > kMaxStages ? kMaxStages : S);
  p.S = S;
  int64_t total = (int64_t)S * p.stage_bytes;
  p.bar_off = (int32_t)total;
  total += 3 * S * 8;  // full, done, empty
  p.meta_off = (int32_t)round_up(total, 16);
  total = p.meta_off + S * (int64_t)sizeof(RaddMeta);
  p.offs_off = (int32_t)round_up(total, 16);
  p.staged = p.batch <= kSmemSeqs;
  total = p.offs_off + (p.staged ? (int64_t)(2 * p.batch + 1) * 4 : 0);
  return (size_t)round_up(total, 128);
}

template <typename T, int D>
static rope_status_t launch_radd_t(const RaddParams &p, size_t smem, cudaStream_t st) {
  static ShapeCache cache;
  constexpr int kThreads = radd_threads<kRaddShape.cw>();
  auto kern = radd_kernel<T, D, kRaddShape.cw, kRaddShape.lag>;
  const int occ = resident_ctas(kern, kThreads, smem, cache);
  if (occ <= 0) return ROPE_ERR_UNSUPPORTED;
  const int64_t slots = (int64_t)sm_count() * occ;
  const int grid = (int)(slots < p.T ? slots : p.T);
  return launch(kern, grid, kThreads, smem, st, p);
}

template <typename T>
static rope_status_t launch_radd_d(int D, const RaddParams &p, size_t smem, cudaStream_t st) {
  if (D == 64) return launch_radd_t<T, 64>(p, smem, st);
  if (D == 128) return launch_radd_t<T, 128>(p, smem, st);
  if constexpr (sizeof(T) == 2)
    if (D == 256) return launch_radd_t<T, 256>(p, smem, st);
  return ROPE_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------- GEMV + partial RMSNorm --

constexpr int kGemvSmemMax = 200 << 10;  // shared memory a staged GEMV CTA may take

template <typename T, int R>
static rope_status_t launch_gemv_r(const GemvParams &p, cudaStream_t st) {
  const int grid = (p.n + R - 1) / R;
  const size_t smem = (size_t)p.row_bytes * (R + 1);
  if (smem <= (size_t)kGemvSmemMax) {  // x and the CTA's rows fit: bulk-copy them
    static ShapeCache cache;
    auto kern = gemv_norm_kernel<T, R, true>;
    if (resident_ctas(kern, kGemvThreads, smem, cache) <= 0) return ROPE_ERR_UNSUPPORTED;
    return launch(kern, grid, kGemvThreads, smem, st, p);
  }
  return launch(gemv_norm_kernel<T, R, false>, grid, kGemvThreads, 0, st, p);
}

// rows per CTA: the fewest that keep the grid within four CTAs an SM (at most 8).  On the
// latent-attention KV projection (W [576, 7168]) one row a CTA, 576 CTAs, ran 6.5 us a call
// in a CUDA graph, against 6.7 with four rows (144 CTAs) and 7.0 with eight.
template <typename T>
static rope_status_t launch_gemv_t(const GemvParams &p, cudaStream_t st) {
  const int sms = sm_count() > 0 ? sm_count() : 1;
  if (p.n <= 4 * sms) return launch_gemv_r<T, 1>(p, st);
  if (p.n <= 8 * sms) return launch_gemv_r<T, 2>(p, st);
  if (p.n <= 16 * sms) return launch_gemv_r<T, 4>(p, st);
  return launch_gemv_r<T, 8>(p, st);
}

// Argument checks and parameter block of rope_split_store_paged_ragged (total_tokens > 0);
// *work is false when the call has nothing to launch.  Nothing is queued on any stream.
static rope_status_t prepare_ragged_store(const void *qkv, int64_t qkv_row_stride,
                                          int32_t qkv_dtype, int32_t total_tokens,
                                          int32_t n_q_heads, const uint32_t *input_row_offsets,
                                          int32_t batch, const rope_freqs_t *freqs,
                                          const rope_paged_cache_t *kv, uint32_t layer_idx,
                                          void *q_out, int64_t q_out_row_stride,
                                          int32_t q_out_dtype, uint32_t *err_word,
                                          uint32_t *sched, BandedParams &p, int &dtype, int &D,
                                          bool &work) {
  work = false;
  if (kv == nullptr || !sched_ok(sched)) return ROPE_ERR_INVALID_ARG;
  // the input's element type: given, or the cache's
  dtype = qkv_dtype >= 0 ? qkv_dtype : kv->dtype;
  D = kv->head_dim;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  if (batch > kv->n_seqs || n_q_heads < 0) return ROPE_ERR_INVALID_ARG;
  s = check_freqs(freqs, dtype, D, &p.rope);
  if (s != ROPE_OK) return s;
  const int64_t Hq = n_q_heads, Hk = kv->n_kv_heads;
  s = fill_band(&p.band[0], qkv, qkv_row_stride, 0, Hq * D, (Hq + Hk) * D, n_q_heads, kv,
                nullptr, nullptr, 0.f, q_out, q_out_row_stride, dtype, layer_idx, false,
                q_out_dtype);
  if (s != ROPE_OK) return s;
  p.n_bands = 1;
  // the head rows the consumers take: Q and K, and V when it is encoded for an FP8 cache
  p.work0 = p.work_total = (int32_t)(Hq + Hk + (p.band[0].kv8 ? Hk : 0));
  p.offs = input_row_offsets;
  p.batch = batch;
  p.T = total_tokens;
  p.layer = layer_idx;
  p.err = err_word;
  p.sched = sched;
  p.overlap = g_overlap.load(std::memory_order_relaxed);
  p.stall_test_ns = g_stall_test_ns.load(std::memory_order_relaxed);
  work = p.work_total + Hk > 0;  // V alone (no Q or K heads) is still copied
  return ROPE_OK;
}

// ------------------------------------------------------- allocation-free entry point --
// Scheduling workspace of rope_split_store_paged_ragged_noalloc.  Every device that loads
// the library holds one copy of this array until the process exits, and every call of that
// entry point on the device uses it.  The schedule needs ROPE_SCHED_WORDS words of it
// whatever the call's sizes.
constexpr int kNoAllocScratchWords = 64;  // 256 bytes
static_assert(ROPE_SCHED_WORDS <= kNoAllocScratchWords, "the schedule must fit the array");
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocScratchWords];

// Identity of the calling thread's current CUDA context: its process-unique id (the driver's
// cuCtxGetId, reached through the runtime without linking the driver library), or 0 when no
// context is current or the driver cannot tell.
typedef int (*CtxGetCurrentFn)(void **);
typedef int (*CtxGetIdFn)(void *, unsigned long long *);
static unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *a = nullptr, *b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 12000, cudaEnableDefault,
                                         &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &qb) ==
            cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
  });
  void *ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_current(&ctx) != 0 || ctx == nullptr || get_id(ctx, &id) != 0)
    return 0;
  return id;
}

// The array's device address in the current device's context.  In host code the symbol only
// names a host-side stand-in, so the address is looked up with cudaGetSymbolAddress (with the
// device current) and kept, together with the id of the context it belongs to: a context
// made after a device reset gets its own copy of the module, and with it a new lookup.
// nullptr if the lookup fails.
static uint32_t *noalloc_scratch() {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static uint32_t *addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (ctx != 0 && ctx == ctx_of[dev] && addr[dev] != nullptr) return addr[dev];
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  addr[dev] = static_cast<uint32_t *>(p);
  ctx_of[dev] = current_context_id();  // the lookup made the device's context current
  return addr[dev];
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
                                            int32_t qkv_dtype, int32_t total_tokens,
                                            int32_t n_q_heads,
                                            const uint32_t *input_row_offsets, int32_t batch,
                                            const rope_freqs_t *freqs,
                                            const rope_paged_cache_t *kv, uint32_t layer_idx,
                                            void *q_out, int64_t q_out_row_stride,
                                            int32_t q_out_dtype, uint32_t *err_word,
                                            uint32_t *sched, rope_stream_t stream) {
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  BandedParams p{};
  int dtype = 0, D = 0;
  bool work = false;
  const rope_status_t s = prepare_ragged_store(
      qkv, qkv_row_stride, qkv_dtype, total_tokens, n_q_heads, input_row_offsets, batch, freqs,
      kv, layer_idx, q_out, q_out_row_stride, q_out_dtype, err_word, sched, p, dtype, D, work);
  if (s != ROPE_OK || !work) return s;
  return launch_banded(dtype, D, false, p, (cudaStream_t)stream);
}

rope_status_t fused_qk_rmsnorm_rope_paged(const void *qkv, int64_t qkv_row_stride,
                                          int32_t qkv_dtype, int32_t total_tokens,
                                          int32_t n_q_heads,
                                          const uint32_t *input_row_offsets, int32_t batch,
                                          const rope_freqs_t *freqs,
                                          const rope_paged_cache_t *kv, const void *q_gamma,
                                          const void *k_gamma, float epsilon,
                                          float weight_offset, int32_t multiply_before_cast,
                                          uint32_t layer_idx, void *q_out,
                                          int64_t q_out_row_stride, uint32_t *err_word,
                                          uint32_t *sched, rope_stream_t stream) {
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  if (kv == nullptr || !sched_ok(sched)) return ROPE_ERR_INVALID_ARG;
  // the input's element type: given, or the cache's
  const int dtype = qkv_dtype >= 0 ? qkv_dtype : kv->dtype, D = kv->head_dim;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  if (batch > kv->n_seqs || n_q_heads < 0) return ROPE_ERR_INVALID_ARG;
  BandedParams p{};
  p.mbc = multiply_before_cast != 0;
  s = check_freqs(freqs, dtype, D, &p.rope);
  if (s != ROPE_OK) return s;
  const int64_t Hq = n_q_heads, Hk = kv->n_kv_heads;
  s = fill_band(&p.band[0], qkv, qkv_row_stride, 0, Hq * D, (Hq + Hk) * D, n_q_heads, kv,
                q_gamma, k_gamma, epsilon, q_out, q_out_row_stride, dtype, layer_idx, true);
  if (s != ROPE_OK) return s;
  p.n_bands = 1;
  // the head rows the consumers take: Q and K, and V when it is encoded for an FP8 cache
  p.work0 = p.work_total = (int32_t)(Hq + Hk + (p.band[0].kv8 ? Hk : 0));
  p.offs = input_row_offsets;
  p.batch = batch;
  p.T = total_tokens;
  p.layer = layer_idx;
  p.err = err_word;
  p.sched = sched;
  p.overlap = g_overlap.load(std::memory_order_relaxed);
  p.stall_test_ns = g_stall_test_ns.load(std::memory_order_relaxed);
  p.weight_offset = round_to_elem(weight_offset, dtype);
  if (p.work_total + Hk == 0) return ROPE_OK;
  return launch_banded(dtype, D, true, p, (cudaStream_t)stream);
}

rope_status_t fused_dual_qk_rmsnorm_rope_paged(const rope_norm_band_t *main_band,
                                               const rope_norm_band_t *index_band,
                                               int32_t input_dtype,
                                               const uint32_t *input_row_offsets,
                                               int32_t batch, int32_t total_tokens,
                                               const rope_freqs_t *freqs, float weight_offset,
                                               int32_t multiply_before_cast, uint32_t layer_idx,
                                               uint32_t *err_word, uint32_t *sched,
                                               rope_stream_t stream) {
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  // index_band == NULL: a launch of the main band alone
  const int n_bands = index_band == nullptr ? 1 : 2;
  if (main_band == nullptr || main_band->cache == nullptr ||
      (index_band != nullptr && index_band->cache == nullptr) || !sched_ok(sched))
    return ROPE_ERR_INVALID_ARG;
  const rope_paged_cache_t *mc = main_band->cache;
  const rope_paged_cache_t *ic = n_bands == 2 ? index_band->cache : mc;
  // the rope geometry must agree across the bands: one input type, one head_dim (each cache
  // holds that type or FP8 codes)
  const int dtype = input_dtype >= 0 ? input_dtype : mc->dtype, D = mc->head_dim;
  if (mc->head_dim != ic->head_dim) return ROPE_ERR_INVALID_ARG;
  for (const rope_paged_cache_t *c : {mc, ic})
    if (c->dtype != dtype && c->dtype != ROPE_DTYPE_FP8_E4M3) return ROPE_ERR_INVALID_ARG;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  if (batch > mc->n_seqs || batch > ic->n_seqs) return ROPE_ERR_INVALID_ARG;
  BandedParams p{};
  p.mbc = multiply_before_cast != 0;
  s = check_freqs(freqs, dtype, D, &p.rope);
  if (s != ROPE_OK) return s;
  const rope_norm_band_t *bands[2] = {main_band, index_band};
  int32_t rows[2] = {0, 0};
  for (int k = 0; k < n_bands; ++k) {
    const rope_norm_band_t *b = bands[k];
    s = fill_band(&p.band[k], b->input, b->input_row_stride, b->q_col, b->k_col, b->v_col,
                  b->n_q_heads, b->cache, b->q_gamma, b->k_gamma, b->epsilon, b->q_out,
                  b->q_out_row_stride, dtype, layer_idx, true);
    if (s != ROPE_OK) return s;
    // the head rows the consumers take: Q and K, and V when it is encoded for an FP8 cache
    rows[k] = p.band[k].n_q + p.band[k].n_kv + (p.band[k].kv8 ? p.band[k].n_v : 0);
  }
  p.n_bands = n_bands;
  p.work0 = rows[0];
  p.work_total = rows[0] + rows[1];
  p.offs = input_row_offsets;
  p.batch = batch;
  p.T = total_tokens;
  p.layer = layer_idx;
  p.err = err_word;
  p.sched = sched;
  p.overlap = g_overlap.load(std::memory_order_relaxed);
  p.stall_test_ns = g_stall_test_ns.load(std::memory_order_relaxed);
  p.weight_offset = round_to_elem(weight_offset, dtype);
  if (p.work_total == 0) return ROPE_OK;
  return launch_banded(dtype, D, true, p, (cudaStream_t)stream);
}

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
  p.f_row_bytes = p.rope.R * (p.rope.dtype == 2 ? 4 : 2);
  p.overlap = g_overlap.load(std::memory_order_relaxed);
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == ROPE_DTYPE_BF16) return launch_bshd_d<__nv_bfloat16>(D, p, st);
  if (dtype == ROPE_DTYPE_F16) return launch_bshd_d<__half>(D, p, st);
  return launch_bshd_d<float>(D, p, st);
}

rope_status_t kv_cache_radd(const void *a, int64_t a_row_stride, int32_t total_tokens,
                            const rope_paged_cache_t *kv, const uint32_t *input_row_offsets,
                            int32_t batch, uint32_t batch_offset, uint32_t layer_idx,
                            uint32_t *err_word, uint32_t *sched, rope_stream_t stream) {
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  if (kv == nullptr || a == nullptr || !sched_ok(sched)) return ROPE_ERR_INVALID_ARG;
  const int dtype = kv->dtype, D = kv->head_dim;
  rope_status_t s = common_checks(dtype, D, input_row_offsets, batch, total_tokens);
  if (s != ROPE_OK) return s;
  RaddParams p{};
  s = check_paged(kv, dtype, layer_idx, true, &p.cache);
  if (s != ROPE_OK) return s;
  const int eb = elem_bytes(dtype);
  const int64_t hidden = (int64_t)kv->n_kv_heads * D;
  if (a_row_stride < 2 * hidden) return ROPE_ERR_INVALID_ARG;
  if (!aligned16(a) || !stride16(a_row_stride, eb)) return ROPE_ERR_UNSUPPORTED;
  if (hidden == 0) return ROPE_OK;
  p.a = a;
  p.a_stride = a_row_stride;
  p.T = total_tokens;
  p.n_kv = kv->n_kv_heads;
  p.batch = batch;
  p.offs = input_row_offsets;
  p.batch_offset = batch_offset;
  p.layer = layer_idx;
  p.err = err_word;
  p.sched = sched;
  p.overlap = g_overlap.load(std::memory_order_relaxed);
  p.stall_test_ns = g_stall_test_ns.load(std::memory_order_relaxed);
  p.kv_contig = kv->head_stride == D ? 1 : 0;
  const size_t smem = layout_radd(p, D, eb);
  if (smem > 227 * 1024) return ROPE_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == ROPE_DTYPE_BF16) return launch_radd_d<__nv_bfloat16>(D, p, smem, st);
  if (dtype == ROPE_DTYPE_F16) return launch_radd_d<__half>(D, p, smem, st);
  return launch_radd_d<float>(D, p, smem, st);
}

rope_status_t rope_split_store_paged_ragged_noalloc(
    const void *qkv, int64_t qkv_row_stride, int32_t qkv_dtype, int32_t total_tokens,
    int32_t n_q_heads,
    const uint32_t *input_row_offsets, int32_t batch, const rope_freqs_t *freqs,
    const rope_paged_cache_t *kv, uint32_t layer_idx, void *q_out, int64_t q_out_row_stride,
    int32_t q_out_dtype, uint32_t *err_word, rope_stream_t stream) {
  if (total_tokens == 0) return ROPE_OK;  // no work: nothing is read or written
  // every argument check first: a call that is rejected queues nothing on the stream
  BandedParams p{};
  int dtype = 0, D = 0;
  bool work = false;
  rope_status_t s = prepare_ragged_store(qkv, qkv_row_stride, qkv_dtype, total_tokens,
                                         n_q_heads, input_row_offsets, batch, freqs, kv,
                                         layer_idx, q_out, q_out_row_stride, q_out_dtype,
                                         err_word, nullptr, p, dtype, D, work);
  if (s != ROPE_OK || !work) return s;
  uint32_t *scratch = noalloc_scratch();
  if (scratch == nullptr) return ROPE_ERR_CUDA;
  // the workspace starts each call at zero (a call that gave up early may have left counts)
  if (cudaMemsetAsync(scratch, 0, ROPE_SCHED_WORDS * sizeof(uint32_t), (cudaStream_t)stream) !=
      cudaSuccess)
    return ROPE_ERR_CUDA;
  p.sched = scratch;
  return launch_banded(dtype, D, false, p, (cudaStream_t)stream);
}

rope_status_t matmul_fused_partial_rmsnorm(const void *input, const void *weight,
                                           int64_t weight_row_stride, int32_t n, int32_t k,
                                           int32_t transpose_b, const void *gamma,
                                           float epsilon, float weight_offset,
                                           void *normed_output, int32_t n_normed,
                                           void *unnormed_output, int32_t dtype,
                                           uint32_t *err_word, void *workspace,
                                           int64_t workspace_bytes, rope_stream_t stream) {
  (void)weight_offset;  // accepted for a uniform signature; not used by this operation
  if (n < 0 || k < 0 || n_normed < 0 || n_normed > n) return ROPE_ERR_INVALID_ARG;
  if (n == 0) return ROPE_OK;  // no output: nothing is read or written
  if (transpose_b == 0) return ROPE_ERR_UNSUPPORTED;
  const int eb = elem_bytes(dtype);
  if (eb == 0) return ROPE_ERR_UNSUPPORTED;
  if (weight == nullptr || weight_row_stride < k || (k > 0 && input == nullptr) ||
      (n_normed > 0 && (gamma == nullptr || normed_output == nullptr || workspace == nullptr)) ||
      (n > n_normed && unnormed_output == nullptr))
    return ROPE_ERR_INVALID_ARG;
  if (n_normed > 0 && workspace_bytes < ROPE_GEMV_WORKSPACE_BYTES(n_normed))
    return ROPE_ERR_INVALID_ARG;
  if ((k * eb) % 16 || !aligned16(weight) || !stride16(weight_row_stride, eb) ||
      (k > 0 && !aligned16(input)) || (n_normed > 0 && !aligned16(workspace)))
    return ROPE_ERR_UNSUPPORTED;
  GemvParams p{};
  p.x = input;
  p.w = weight;
  p.w_stride = weight_row_stride;
  p.n = n;
  p.k = k;
  p.n_normed = n_normed;
  p.gamma = gamma;
  p.eps = epsilon;
  p.normed = normed_output;
  p.unnormed = unnormed_output;
  p.count = static_cast<uint32_t *>(workspace);
  p.ws = workspace ? reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + 16)
                   : nullptr;
  p.err = err_word;
  p.row_bytes = (int32_t)round_up((int64_t)k * eb, 16);
  p.overlap = g_overlap.load(std::memory_order_relaxed);
  p.stall_test_ns = g_stall_test_ns.load(std::memory_order_relaxed);
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == ROPE_DTYPE_BF16) return launch_gemv_t<__nv_bfloat16>(p, st);
  if (dtype == ROPE_DTYPE_F16) return launch_gemv_t<__half>(p, st);
  return launch_gemv_t<float>(p, st);
}

rope_status_t rope_set_launch_overlap(int32_t mode) {
  if (mode != ROPE_OVERLAP_OFF && mode != ROPE_OVERLAP_PDL && mode != ROPE_OVERLAP_PDL_EARLY_METADATA)
    return ROPE_ERR_INVALID_ARG;
  g_overlap.store(mode, std::memory_order_relaxed);
  return ROPE_OK;
}

int32_t rope_get_launch_overlap(void) { return g_overlap.load(std::memory_order_relaxed); }

rope_status_t rope_set_stall_test(uint32_t timeout_us) {
  if (timeout_us > 1000000u) return ROPE_ERR_INVALID_ARG;
  g_stall_test_ns.store(timeout_us * 1000u, std::memory_order_relaxed);
  return ROPE_OK;
}

uint32_t rope_get_stall_test(void) {
  return g_stall_test_ns.load(std::memory_order_relaxed) / 1000u;
}

}  // extern "C"
