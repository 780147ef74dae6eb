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
//                      L = head_dim / (2 * vector) lanes; each lane owns two 16-byte vectors
//                      of a row (for half-split RoPE the two halves of its rotation pairs),
//                      normalises them (shuffle reduction over its group), rotates them and
//                      writes them back in place; with the norm, a first pass over up to
//                      three of its rows reduces their sums of squares together, and a second
//                      reads each row again to scale, rotate and write it (rows_step);
//   warp 1, storer:    once the consumers are done with a token, bulk-copies the stage's Q
//                      block to q_out and its K and V blocks to the cache page, waits until
//                      the copies have read the stage, and hands the stage back.
// V rows never enter registers, except for an FP8 cache, where they are consumer rows too
// (encoded exactly: e4m3_exact4).  The extended-output instantiation (EXT) writes some
// results to stage regions of their own instead of in place: Q rounded into another element
// type, and the E4M3 codes of K and V for an FP8 cache; the storer copies those regions out.  The row range of a token is the band concatenation
// [Q main | K main | V main | Q index | K index | (V index)].
#pragma once

#include "common.cuh"

#include <cuda_fp8.h>

#include <type_traits>

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

// N float values as N E4M3 codes, code i in byte i % 4 of word i / 4 (nearest, ties to
// even, saturating at +-448)
template <int N>
__device__ __forceinline__ void e4m3_words(const float (&x)[N], uint32_t (&w)[N / 4]) {
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i], x[4 * i + 1]),
                                                 __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i + 2], x[4 * i + 3]),
                                                 __NV_SATFINITE, __NV_E4M3);
    w[i] = lo | (hi << 16);
  }
}

// The N / 4 code words of N values at shared address a
template <int N>
__device__ __forceinline__ void sts_words(uint32_t a, const uint32_t (&w)[N / 4]) {
  if constexpr (N == 8) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(w[0]), "r"(w[1]) : "memory");
  } else {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(w[0]) : "memory");
  }
}

// N float values written at shared address a as N elements of type qd (0 bf16, 1 f16,
// 2 f32), rounded to nearest even
template <int N>
__device__ __forceinline__ void sts_elems(uint32_t a, const float (&x)[N], int qd) {
  if (qd == 2) {
#pragma unroll
    for (int k = 0; k < N; k += 4)
      sts_v4(a + k * 4, make_uint4(__float_as_uint(x[k]), __float_as_uint(x[k + 1]),
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
    sts_v4(a, make_uint4(w[0], w[1], w[2], w[3]));
  } else {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(w[0]), "r"(w[1]) : "memory");
  }
}

__device__ __forceinline__ uint32_t e4m3_code(float x) {
  return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3)));
}

// The E4M3 code of v / s rounded exactly as one rounding of the true quotient would
// (nearest, ties to even, saturating at +-448), for finite v and a finite scale s whose
// rounded reciprocal inv is a normal float.  q = v * inv lies within two float32 ulps of
// v / s, so the codes of q moved two ulps down and up in magnitude agree (and are the
// answer) unless a rounding boundary m of the E4M3 grid lies between them; then the sign
// of v - m * s, which one fused multiply-add gives exactly, says on which side of m the
// quotient lies (zero: it is m, and the tie goes to the even code).
__device__ __forceinline__ uint32_t e4m3_exact(float v, float inv, float s) {
  const float q = v * inv;
  const uint32_t b = __float_as_uint(q), mag = b & 0x7fffffffu, sgn = b & 0x80000000u;
  if (mag >= 0x7f7ffffeu) return e4m3_code(q);  // saturates (or is not finite) either way
  const float lo = __uint_as_float((mag < 2u ? 0u : mag - 2u) | sgn);
  const float hi = __uint_as_float((mag + 2u) | sgn);
  const uint32_t pr = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
  const uint32_t cl = pr & 0xffu, ch = pr >> 8;
  if (cl == ch) return cl;
  const float m = 0.5f * (e4m3_value(cl) + e4m3_value(ch));  // exact: a 5-bit number
  const float r = fmaf(-m, s, v);
  if (r == 0.f) return e4m3_code(m);
  const bool above = (r > 0.f) == (s > 0.f);  // v / s > m
  // ch has the larger magnitude: the larger value when q >= 0
  return above == (sgn == 0u) ? ch : cl;
}

// E4M3 codes of v0..v3 * inv as one word (code i in byte i), each converted once (nearest,
// ties to even, saturating)
__device__ __forceinline__ uint32_t e4m3_scaled4(float v0, float v1, float v2, float v3,
                                                 float inv) {
  return __nv_cvt_float2_to_fp8x2(make_float2(v0 * inv, v1 * inv), __NV_SATFINITE, __NV_E4M3) |
         (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(v2 * inv, v3 * inv), __NV_SATFINITE,
                                            __NV_E4M3)
             << 16;
}

// Whether s is 2^k with both s and 1/s normal floats: then v * (1/s) is v / s exactly, up to
// an overflow or underflow that E4M3 saturates or rounds to zero either way.
__device__ __forceinline__ int pow2_scale(float s) {
  const uint32_t b = __float_as_uint(s), e = (b >> 23) & 0xffu;
  return (b & 0x807fffffu) == 0u && e >= 1u && e <= 253u;
}

// E4M3 codes of v0..v3 / s as one word (code i in byte i), each rounded exactly once as
// e4m3_exact does.  The conversion of q = v * inv is the answer unless q is not the exact
// quotient (v - q * s, exact in one fused multiply-add, is not zero) and lies within two
// ulps of a rounding boundary of the normal E4M3 grid (bit 19 of the mantissa set, bits
// 18..0 clear: a midpoint between codes), or below it (|q| < 2^-6, the subnormal codes);
// such a value, which is rare, goes through e4m3_exact.  With a power-of-two scale q is
// always exact.
__device__ __forceinline__ uint32_t e4m3_exact4(float v0, float v1, float v2, float v3,
                                                float inv, float s) {
  const float v[4] = {v0, v1, v2, v3};
  float q[4];
  bool slow = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    q[i] = v[i] * inv;
    const uint32_t b = __float_as_uint(q[i]), e = (b >> 23) & 0xffu;
    const bool near = ((b & 0xfffffu) - 0x7fffeu) <= 4u;
    slow |= (near || e < 121u) && fmaf(-q[i], s, v[i]) != 0.f;
  }
  if (!slow)
    return __nv_cvt_float2_to_fp8x2(make_float2(q[0], q[1]), __NV_SATFINITE, __NV_E4M3) |
           (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(q[2], q[3]), __NV_SATFINITE,
                                              __NV_E4M3)
               << 16;
  return e4m3_exact(v[0], inv, s) | e4m3_exact(v[1], inv, s) << 8 |
         e4m3_exact(v[2], inv, s) << 16 | e4m3_exact(v[3], inv, s) << 24;
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
  uint32_t stall_test_ns;  // > 0: the launch starts with a wait nothing completes (a test)
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

// Whether the per-lane table and gamma loads rotate their chunk order so that the lanes of
// a quarter-warp hit distinct banks (undone with selects), or read in plain order.
#ifndef ROPE_LDS_ROTATE
#define ROPE_LDS_ROTATE 1
#endif
constexpr bool kLdsRotate = ROPE_LDS_ROTATE != 0;

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
    lds_chunks<C>(F + col * 4, kLdsRotate ? (gl / LP) % C : 0, c);
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
      lds_chunks<C>(F + col * 2, kLdsRotate ? (gl / LP) % C : 0, c);
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

// Head rows whose norm reductions a consumer thread overlaps (rows_step's first pass), within
// the register budget of the shape: light CTAs run three to an SM, the others two.  Three
// for the six-warp norm shape, one elsewhere (the eight-warp shape has 96 registers, and two
// rows spilled there; a store without the norm has no reduction).
#ifndef ROPE_CHUNK_ROWS_NORM
#define ROPE_CHUNK_ROWS_NORM 3
#endif
template <int CW, bool NORM>
__host__ __device__ constexpr int chunk_rows() {
  return NORM && CW > 4 && CW < 8 ? ROPE_CHUNK_ROWS_NORM : 1;
}

// M consecutive float32 values from shared address a (16-byte aligned), read bank-conflict
// free across the lanes of a group (gl = lane index inside the group), as lds_freqs does.
template <int M>
__device__ __forceinline__ void lds_f32(uint32_t a, int gl, float (&f)[M]) {
  constexpr int C = M / 4;
  constexpr int LP = 32 / M > 0 ? 32 / M : 1;
  const int rot = kLdsRotate ? (gl / LP) % C : 0;
  uint4 t[C], c[C];
#pragma unroll
  for (int k = 0; k < C; ++k) t[k] = lds_v4(a + ((k + rot) % C) * 16);
#pragma unroll
  for (int k = 0; k < C; ++k) c[k] = t[k];
  if constexpr (C >= 2) {
    if (rot & 1) {
#pragma unroll
      for (int k = 0; k < C; ++k) c[(k + 1) % C] = t[k];
#pragma unroll
      for (int k = 0; k < C; ++k) t[k] = c[k];
    }
  }
  if constexpr (C >= 4) {
    if (rot & 2) {
#pragma unroll
      for (int k = 0; k < C; ++k) c[(k + 2) % C] = t[k];
    }
  }
#pragma unroll
  for (int k = 0; k < C; ++k) {
    f[4 * k] = __uint_as_float(c[k].x);
    f[4 * k + 1] = __uint_as_float(c[k].y);
    f[4 * k + 2] = __uint_as_float(c[k].z);
    f[4 * k + 3] = __uint_as_float(c[k].w);
  }
}

// What a consumer lane owns of every head row: its two vectors (first columns ca, cb; table
// columns fa, fb), whether each is rotated, the layout and the lane's group.
struct ConsumerLane {
  int li, ca, cb, fa, fb, fdt;
  bool inter, rot_a, rot_b;
  unsigned gmask;
};

// Two float values rounded to the element type T (nearest even) and widened back.
template <typename T>
__device__ __forceinline__ float2 round2(float2 v) {
  if constexpr (sizeof(T) == 4) {
    return v;
  } else if constexpr (std::is_same<T, __half>::value) {
    return __half22float2(__floats2half2_rn(v.x, v.y));
  } else {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    const uint32_t w = *reinterpret_cast<const uint32_t *>(&h);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
}

// The token's (cos, sin) for a consumer lane.  Interleaved, pair k of vector a: (c[k],
// s[k]); of vector b: (c2[k], s2[k]).  Half-split, as float2 over the lane's N pairs: P[k] =
// (c_2k, c_2k+1), Q = (s_2k, s_2k+1), R = -Q.
template <int N, bool INTER>
struct LaneFreqs;
template <int N>
struct LaneFreqs<N, true> {
  float c[N / 2], s[N / 2], c2[N / 2], s2[N / 2];
};
template <int N>
struct LaneFreqs<N, false> {
  float2 P[N / 2], Q[N / 2], R[N / 2];
};

template <int N, bool INTER>
__device__ __forceinline__ void load_lane_freqs(LaneFreqs<N, INTER> &fr, const ConsumerLane &cl,
                                                const unsigned char *F) {
  if constexpr (INTER) {
    float f[N];
    if (cl.rot_a) {
      lds_freqs<N>(F, cl.fdt, cl.fa, cl.li, f);
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        fr.c[k] = f[2 * k];
        fr.s[k] = f[2 * k + 1];
      }
    }
    if (cl.rot_b) {
      lds_freqs<N>(F, cl.fdt, cl.fb, cl.li, f);
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        fr.c2[k] = f[2 * k];
        fr.s2[k] = f[2 * k + 1];
      }
    }
  } else if (cl.rot_a) {
    float f[2 * N];
    lds_freqs<2 * N>(F, cl.fdt, cl.fa, cl.li, f);
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
      fr.P[k] = make_float2(f[4 * k], f[4 * k + 2]);
      fr.Q[k] = make_float2(f[4 * k + 1], f[4 * k + 3]);
      fr.R[k] = make_float2(-f[4 * k + 1], -f[4 * k + 3]);
    }
  }
}

// RoPE of a lane's two vectors of one head row.
template <int H2, bool INTER>
__device__ __forceinline__ void rotate_lane(const LaneFreqs<2 * H2, INTER> &fr,
                                            const ConsumerLane &cl, float2 (&xa)[H2],
                                            float2 (&xb)[H2]) {
  if constexpr (INTER) {
    if (cl.rot_a)
#pragma unroll
      for (int k = 0; k < H2; ++k) {  // (a, b) -> (a c - b s, a s + b c)
        const float a = xa[k].x, b = xa[k].y;
        xa[k] = make_float2(fmaf(a, fr.c[k], -b * fr.s[k]), fmaf(a, fr.s[k], b * fr.c[k]));
      }
    if (cl.rot_b)
#pragma unroll
      for (int k = 0; k < H2; ++k) {
        const float a = xb[k].x, b = xb[k].y;
        xb[k] = make_float2(fmaf(a, fr.c2[k], -b * fr.s2[k]), fmaf(a, fr.s2[k], b * fr.c2[k]));
      }
  } else if (cl.rot_a) {
    // pair element e of vector a with element e of vector b
#pragma unroll
    for (int k = 0; k < H2; ++k) {
      const float2 a = xa[k], b = xb[k];
      xa[k] = __ffma2_rn(b, fr.R[k], __fmul2_rn(a, fr.P[k]));
      xb[k] = __ffma2_rn(a, fr.Q[k], __fmul2_rn(b, fr.P[k]));
    }
  }
}

// Where a band's rows go in the extended-output instantiation: Q rows rounded into q_dtype
// at shared address qo (when q_conv), K rows as E4M3 codes of value * kinv at k8 and V rows
// as the exactly rounded codes of value / vs at v8 (when kv8), others back in place; row r
// of the band's block sits at blk + r * D * element size.
struct BandOut {
  uint32_t blk, qo, k8, v8;
  int q_conv, q_dtype, q_eb, kv8, n_q, n_kv, v_pow2;
  float kinv, vinv, vs;
};

// J head rows of a staged token, listed at it[0], it[stride], ...: optionally normalised
// (per-head RMSNorm with the gamma rows at shared addresses gq / gk for Q / K rows), then
// rotated with the token's table row, held in `fr` (INTER: the interleaved layout), and
// written back in place (EXT: outputs as `bo` says).  With the norm, a first pass reads the
// J rows and reduces their sums of squares together, so that their shuffle and reciprocal
// square-root latencies overlap while only one float a row stays live; the second pass reads
// each row again (shared memory has the bandwidth to spare) and scales, rotates and writes
// it.  Three rows held whole through the reduction spilled at 128 registers (per-head norm
// 118.8 us, against 105 us for the two passes).
template <int J, typename T, int D, bool NORM, int L, bool INTER, bool EXT>
__device__ __forceinline__ void rows_step(const ConsumerLane &cl, const uint32_t *it, int stride,
                                          uint32_t st, uint32_t gq, uint32_t gk, float eps,
                                          int mbc, const LaneFreqs<Vec<T>::N, INTER> &fr,
                                          const BandOut &bo) {
  using VT = Vec<T>;
  constexpr int N = VT::N, H2 = N / 2, EB = (int)sizeof(T);
  uint32_t row[J], g[J];
  bool isk[J];
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const uint32_t w = it[j * stride];
    row[j] = st + (w & kItemOffMask);
    isk[j] = ((w >> kItemKindShift) & 3) != 0;
    g[j] = isk[j] ? gk : gq;
  }
  float r[J];
  if constexpr (NORM) {
    // first pass: each row's sum of squares, read straight from shared memory, so that only
    // one float a row stays live across the reduction and the reciprocal square root
#pragma unroll
    for (int j = 0; j < J; ++j) {
      float ta[N], tb[N];
      VT::widen(lds_v4(row[j] + cl.ca * EB), ta);
      VT::widen(lds_v4(row[j] + cl.cb * EB), tb);
      // pairs of the two vectors alternately, as two float32 lanes
      float2 acc = __fmul2_rn(make_float2(ta[0], ta[1]), make_float2(ta[0], ta[1]));
      acc = __ffma2_rn(make_float2(tb[0], tb[1]), make_float2(tb[0], tb[1]), acc);
#pragma unroll
      for (int k = 1; k < H2; ++k) {
        acc = __ffma2_rn(make_float2(ta[2 * k], ta[2 * k + 1]),
                         make_float2(ta[2 * k], ta[2 * k + 1]), acc);
        acc = __ffma2_rn(make_float2(tb[2 * k], tb[2 * k + 1]),
                         make_float2(tb[2 * k], tb[2 * k + 1]), acc);
      }
      r[j] = acc.x + acc.y;
    }
#pragma unroll
    for (int msk = L / 2; msk > 0; msk >>= 1)
#pragma unroll
      for (int j = 0; j < J; ++j) r[j] += __shfl_xor_sync(cl.gmask, r[j], msk);
#pragma unroll
    for (int j = 0; j < J; ++j) r[j] = rsqrtf(r[j] * (1.0f / D) + eps);
  }
  // row by row (the second pass with the norm): read the row, scale, rotate, write
  float ga[N], gb[N];  // gamma + weight_offset of the lane's columns, read once per kind
#pragma unroll
  for (int j = 0; j < J; ++j) {
    float2 xa[H2], xb[H2];
    {
      float t[N];
      VT::widen(lds_v4(row[j] + cl.ca * EB), t);
#pragma unroll
      for (int k = 0; k < H2; ++k) xa[k] = make_float2(t[2 * k], t[2 * k + 1]);
      VT::widen(lds_v4(row[j] + cl.cb * EB), t);
#pragma unroll
      for (int k = 0; k < H2; ++k) xb[k] = make_float2(t[2 * k], t[2 * k + 1]);
    }
    float rj = 1.f;
    if constexpr (NORM) {
      if (j == 0 || g[j] != g[j - 1]) {
        lds_f32<N>(g[j] + cl.ca * 4, cl.li, ga);
        lds_f32<N>(g[j] + cl.cb * 4, cl.li, gb);
      }
      if (mbc) {  // x * gamma now; the scalar r after the rotation
#pragma unroll
        for (int k = 0; k < H2; ++k) {
          xa[k] = __fmul2_rn(xa[k], make_float2(ga[2 * k], ga[2 * k + 1]));
          xb[k] = __fmul2_rn(xb[k], make_float2(gb[2 * k], gb[2 * k + 1]));
        }
        rj = r[j];
      } else {  // the normalised value is rounded to the element type, then scaled
        const float2 rr = make_float2(r[j], r[j]);
#pragma unroll
        for (int k = 0; k < H2; ++k) {
          xa[k] = __fmul2_rn(round2<T>(__fmul2_rn(xa[k], rr)),
                                make_float2(ga[2 * k], ga[2 * k + 1]));
          xb[k] = __fmul2_rn(round2<T>(__fmul2_rn(xb[k], rr)),
                                make_float2(gb[2 * k], gb[2 * k + 1]));
        }
      }
    }
    rotate_lane<H2, INTER>(fr, cl, xa, xb);
    if constexpr (NORM) {
      const float2 rr = make_float2(rj, rj);
#pragma unroll
      for (int k = 0; k < H2; ++k) {
        xa[k] = __fmul2_rn(xa[k], rr);
        xb[k] = __fmul2_rn(xb[k], rr);
      }
    }
    float ta[N], tb[N];
#pragma unroll
    for (int k = 0; k < H2; ++k) {
      ta[2 * k] = xa[k].x;
      ta[2 * k + 1] = xa[k].y;
      tb[2 * k] = xb[k].x;
      tb[2 * k + 1] = xb[k].y;
    }
    if constexpr (EXT) {
      const int rb = (int)(row[j] - bo.blk) / (D * EB);  // the row's index in the band block
      if (!isk[j] && bo.q_conv) {  // every lane writes its Q vectors, rounded once
        const uint32_t qrow = bo.qo + (uint32_t)(rb * D * bo.q_eb);
        sts_elems<N>(qrow + cl.ca * bo.q_eb, ta, bo.q_dtype);
        sts_elems<N>(qrow + cl.cb * bo.q_eb, tb, bo.q_dtype);
        continue;
      }
      if (isk[j] && bo.kv8) {  // and its K codes
#pragma unroll
        for (int e = 0; e < N; ++e) {
          ta[e] *= bo.kinv;
          tb[e] *= bo.kinv;
        }
        const uint32_t krow = bo.k8 + (uint32_t)((rb - bo.n_q) * D);
        uint32_t wa[N / 4], wb[N / 4], w1[N / 4], w2[N / 4];
        e4m3_words<N>(ta, wa);
        e4m3_words<N>(tb, wb);
        // the row groups of a warp sit one code row (128 bytes at head_dim 128) apart, on the
        // same banks: odd groups store their b half first, so that each store instruction
        // covers all 32 banks
        const bool odd = (threadIdx.x / L) & 1;
#pragma unroll
        for (int e = 0; e < N / 4; ++e) {
          w1[e] = odd ? wb[e] : wa[e];
          w2[e] = odd ? wa[e] : wb[e];
        }
        sts_words<N>(krow + (odd ? cl.cb : cl.ca), w1);
        sts_words<N>(krow + (odd ? cl.ca : cl.cb), w2);
        continue;
      }
    }
    if (NORM || cl.rot_a) sts_v4(row[j] + cl.ca * EB, VT::narrow(ta));
    if (NORM || cl.rot_b) sts_v4(row[j] + cl.cb * EB, VT::narrow(tb));
  }
}

// The V rows of an FP8 band among a consumer thread's slots [lo, hi): the lane's two
// vectors of each row encoded as E4M3 codes of value / scale, each rounded once (with a
// power-of-two scale the product with its reciprocal is the exact quotient, and one
// conversion rounds it).
template <typename T, int D>
__device__ __forceinline__ void v_rows(const ConsumerLane &cl, const uint32_t *item, int stride,
                                       int lo, int hi, uint32_t st, const BandOut &bo) {
  using VT = Vec<T>;
  constexpr int N = VT::N, EB = (int)sizeof(T);
#pragma unroll 1
  for (int u = lo; u < hi; ++u) {
    const uint32_t row = st + (item[u * stride] & kItemOffMask);
    const int rb = (int)(row - bo.blk) / (D * EB);
    const uint32_t vrow = bo.v8 + (uint32_t)((rb - bo.n_q - bo.n_kv) * D);
    float x[2][N];
    VT::widen(lds_v4(row + cl.ca * EB), x[0]);
    VT::widen(lds_v4(row + cl.cb * EB), x[1]);
    const int odd = (threadIdx.x / (D / (2 * N))) & 1;  // b half first, as for the K codes
#pragma unroll
    for (int h0 = 0; h0 < 2; ++h0) {
      const int h = h0 ^ odd;
      const uint32_t a = vrow + (h ? cl.cb : cl.ca);
      const uint32_t w0 = bo.v_pow2 ? e4m3_scaled4(x[h][0], x[h][1], x[h][2], x[h][3], bo.vinv)
                                    : e4m3_exact4(x[h][0], x[h][1], x[h][2], x[h][3], bo.vinv,
                                                  bo.vs);
      if constexpr (N == 8) {
        const uint32_t w1 =
            bo.v_pow2 ? e4m3_scaled4(x[h][4], x[h][5], x[h][6], x[h][7], bo.vinv)
                      : e4m3_exact4(x[h][4], x[h][5], x[h][6], x[h][7], bo.vinv, bo.vs);
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(w0), "r"(w1) : "memory");
      } else {
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(w0) : "memory");
      }
    }
  }
}

// A band's slots [lo, hi) of a consumer thread's head rows, JM at a time; the token's table
// row is read once here, for every chunk.
template <int JM, typename T, int D, bool NORM, int L, bool INTER, bool EXT>
__device__ __forceinline__ void rows_band(const ConsumerLane &cl, const uint32_t *item, int stride,
                                          int lo, int hi, uint32_t st, uint32_t gq, uint32_t gk,
                                          float eps, int mbc, const unsigned char *F,
                                          const BandOut &bo) {
  static_assert(JM >= 1 && JM <= 3, "the tail below takes at most two rows after the chunks");
  LaneFreqs<Vec<T>::N, INTER> fr;
  load_lane_freqs<Vec<T>::N, INTER>(fr, cl, F);
  int u = lo;
#pragma unroll 1
  for (; u + JM <= hi; u += JM)
    rows_step<JM, T, D, NORM, L, INTER, EXT>(cl, item + u * stride, stride, st, gq, gk, eps,
                                             mbc, fr, bo);
  if constexpr (JM >= 3) {
    if (hi - u == 2)
      rows_step<2, T, D, NORM, L, INTER, EXT>(cl, item + u * stride, stride, st, gq, gk, eps,
                                              mbc, fr, bo);
  }
  if constexpr (JM >= 2) {
    if (hi - u == 1)
      rows_step<1, T, D, NORM, L, INTER, EXT>(cl, item + u * stride, stride, st, gq, gk, eps,
                                              mbc, fr, bo);
  }
}

#ifndef ROPE_LIGHT_MIN_CTAS
#define ROPE_LIGHT_MIN_CTAS 3
#endif
// resident CTAs per SM the register budget is sized for: the light store shape (<= 4
// consumer warps, no norm) and every other one
template <int CW, bool NORM>
__host__ __device__ constexpr int pipe_min_ctas() {
  return CW <= 4 && !NORM ? ROPE_LIGHT_MIN_CTAS : 2;
}

// EXT: built with the extended outputs (a Q output in another element type, FP8 cache rows)
template <typename T, int D, bool NORM, int CW, int LAG, bool EXT>
__global__ void __launch_bounds__(pipe_threads<CW>(), pipe_min_ctas<CW, NORM>())
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
  __shared__ __align__(8) uint64_t s_never;  // no thread ever arrives here

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) grid_dep_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], kConsumerWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&s_never, 1);
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

  if (p.stall_test_ns != 0 && warp >= 2) {
    // A test of the timeout path (stall_test_ns > 0): the consumers wait on a barrier that
    // no thread ever arrives at, for at most stall_test_ns; when the wait runs out they do
    // what a pipeline wait that runs out makes them do.
    if (!mbar_wait(&s_never, 0, &s_abort, p.stall_test_ns) && lane == 0) {
      s_abort = 1;
      raise(p.err, ROPE_DEVERR_TIMEOUT);
    }
  } else if (warp == 0) {
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
    bool marked = false;  // the stop marker went into stage issued % S
    if (!aborted && lane == 0) {
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
      // let the loads issued land before the CTA's shared memory goes away: only the last S
      // can be in flight (a stage is reloaded only once the storer released it); in a run
      // that did not give up the consumers have waited for them already.  The stop marker
      // took the stage of token issued - S one phase further, and that token was stored
      // before the stage was handed back: its phase is not waited for (its parity now names
      // the marker's next, unfinished phase).
      for (int ii = max(0, issued - p.S + (marked ? 1 : 0)); ii < issued; ++ii) {
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
    // vectors.  Interleaved: lane j owns vectors j and j + L.  A thread's head rows of a
    // token are taken up to JM at a time, so that their load -> reduce -> scale -> rotate
    // chains overlap.
    constexpr int JM = chunk_rows<CW, NORM>();
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
    const int fa = inter ? ca - rp.off : 2 * (ca - rp.off);
    const int fb = cb - rp.off;
    const ConsumerLane cl{li, ca, cb, fa, fb, rp.dtype, inter, rot_a, rot_b, gmask};
    // this thread's head rows of a token, decoded once into shared memory: band 0's Q and K
    // rows in slots [0, qk0), its V rows (FP8 caches only) in [qk0, end0); band 1's in
    // [beg1, qk1) and [qk1, end1)
    const int n_items = (p.work_total + G - 1) / G;
    uint32_t *item = s_items + ctid;  // slot u at item[u * kConsumers]
    int qk0 = 0, end0 = 0, beg1 = -1, qk1 = 0, end1 = 0;
    for (int u = 0; u < n_items; ++u) {
      const int j = grp + u * G;
      uint32_t w = 0;
      if (j < p.work_total) {
        const int band = j >= p.work0 ? 1 : 0;
        const BandDev &bd = band ? p.band[1] : p.band[0];
        const int r = j - (band ? p.work0 : 0);  // Q heads, K heads, V heads: stage rows 0..
        const int kind = r < bd.n_q ? 0 : r < bd.n_q + bd.n_kv ? 1 : 2;
        const uint32_t soff = (uint32_t)(bd.smem_off + r * D * EB);
        w = kItemAct | (uint32_t)band << kItemBandShift | (uint32_t)kind << kItemKindShift | soff;
        if (band == 0) {
          if (kind < 2) qk0 = u + 1;
          end0 = u + 1;
        } else {
          if (beg1 < 0) beg1 = qk1 = u;
          if (kind < 2) qk1 = u + 1;
          end1 = u + 1;
        }
      }
      item[u * kConsumers] = w;
    }
    if (beg1 < 0) beg1 = qk1 = end1 = end0;
    const uint32_t stages_a = smem_addr(stages);
    const uint32_t gamma_a = smem_addr(s_gamma);
    // FP8 planes: 1 / scale of K, scale and 1 / scale of V
    float kinv[2] = {1.f, 1.f}, vsc[2] = {1.f, 1.f}, vinv[2] = {1.f, 1.f};
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
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const BandDev &bd = k ? p.band[1] : p.band[0];
          if (k < p.n_bands && bd.kv8) {
            kinv[k] = 1.f / __ldg(bd.k_scale);
            if (bd.n_v) {
              vsc[k] = __ldg(bd.v_scale);
              vinv[k] = 1.f / vsc[k];
            }
          }
        }
      }
      const uint32_t st = stages_a + (uint32_t)(s * p.stage_bytes);
      const int ok0 = meta[s].ok[0], ok1 = meta[s].ok[1];
#pragma unroll 1
      for (int band = 0; band < p.n_bands; ++band) {
        const int lo = band ? beg1 : 0, qk = band ? qk1 : qk0, hi = band ? end1 : end0;
        if (lo >= hi || !(band ? ok1 : ok0)) continue;
        const BandDev &bd = band ? p.band[1] : p.band[0];
        BandOut bo{};
        if constexpr (EXT) {
          bo = BandOut{st + (uint32_t)bd.smem_off, st + (uint32_t)bd.qo_off,
                       st + (uint32_t)bd.k8_off,   st + (uint32_t)bd.v8_off,
                       bd.q_conv, bd.q_dtype, bd.q_eb, bd.kv8, bd.n_q, bd.n_kv,
                       pow2_scale(band ? vsc[1] : vsc[0]), band ? kinv[1] : kinv[0],
                       band ? vinv[1] : vinv[0],
                       band ? vsc[1] : vsc[0]};
          if (qk < hi) v_rows<T, D>(cl, item, kConsumers, qk, hi, st, bo);
        }
        // lanes with nothing to do leave their bytes in place, unless they go elsewhere
        if (lo >= qk || (!busy && !(EXT && (bd.q_conv || bd.kv8)))) continue;
        const unsigned char *F = stages + (size_t)s * p.stage_bytes + bd.f_off;
        const float eps = bd.eps;
        const uint32_t gq = gamma_a + (uint32_t)(band * 2 * D * 4), gk = gq + D * 4;
        if (inter)
          rows_band<JM, T, D, NORM, L, true, EXT>(cl, item, kConsumers, lo, qk, st, gq, gk, eps,
                                                 p.mbc, F, bo);
        else
          rows_band<JM, T, D, NORM, L, false, EXT>(cl, item, kConsumers, lo, qk, st, gq, gk,
                                                  eps, p.mbc, F, bo);
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
