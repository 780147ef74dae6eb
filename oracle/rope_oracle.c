/*
 * rope_oracle.c -- plain double-precision CPU oracle (TEST INFRASTRUCTURE ONLY; see
 * rope_oracle.h for who may load it).  Every function below is the plain definition of one
 * documented operation, evaluated token by token, head by head, column by column.
 *
 * Sources (Modular MAX kernel reference pages):
 *   [P1] "generic_fused_qk_rope_bshd_continuous_batch": description paragraph and Args
 *        (q_proj [batch, seq_len, n_heads, head_dim]; valid_lengths: RoPE only for positions
 *        inside the valid length; output same shape as q_proj).
 *   [P2] "rope_split_store_paged_ragged": one-line description (rotate, split the QKV
 *        columns, store into the paged cache); Args: qkv is the flat projection output
 *        [total_seq_len, q_dim + k_dim + v_dim], input_row_offsets has batch_size + 1
 *        entries, freqs_cis is [max_seq_len, head_dim] with the two parts of each rotation
 *        side by side, q_output is [total_seq_len, q_dim]; Parameters: interleaved (layout of
 *        the rotated pairs).
 *   [P3] "generic_kv_cache_radd_dispatch": description and Args (a is [sum(seq_lens),
 *        2*hidden_size]; its first half of columns goes to K and its second half to V; the
 *        batch index is shifted by batch_offset; the cache length of the sequence gives the
 *        row's position).
 *   [P4] "fused_dual_qk_rms_norm_rope_ragged_paged": signature (gammas, main/index epsilon,
 *        weight_offset, multiply_before_cast) and both description paragraphs (one launch
 *        equals two single-band fused_qk_rms_norm_rope_ragged_paged launches; rope geometry
 *        identical across bands; rope_dim = columns of freqs_cis).
 *   [P5] "MatmulFusedPartialRMSNorm": Args (epsilon sits inside the inverse square root,
 *        with the mean of squares).
 *
 * Readings chosen where the pages leave a step open:
 *   - freqs_cis row p = (cos, sin) pairs of pair i at columns 2i, 2i+1, for both layouts;
 *   - partial RoPE rotates columns [o, o + rope_dim) of each head, o = head_dim - rope_dim
 *     unless the caller names another offset;
 *   - half-split pairs are (o + i, o + i + rope_dim/2) and use pair i's (cos, sin);
 *   - RMSNorm runs over all head_dim columns of one (token, head) row, gamma is [head_dim]
 *     and shared by the heads of its kind; RoPE takes the normed value unrounded;
 *   - position = cache_lengths[seq] + index of the token inside its sequence;
 *   - BSHD tokens at or beyond valid_lengths[b] are copied to the output unchanged and
 *     their K cache rows are left alone;
 *   - a token whose position or page lookup falls outside the tables is skipped (nothing of
 *     it is written) and its error bit is returned.
 */
#include "rope_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ element codecs -- */

static double bf16_bits_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16; /* bfloat16 is the top half of an IEEE binary32 */
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double f16_bits_to_double(uint16_t h) {
  int neg = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  return neg ? -v : v;
}

/* Round a > 0 (finite) to the nearest point, ties to even, of the grid of a binary format
 * with `frac_bits` fraction bits whose smallest normal exponent is `emin` (below 2^emin the
 * grid keeps the spacing 2^(emin - frac_bits): gradual underflow). */
static double round_to_grid(double a, int frac_bits, int emin) {
  int e;
  frexp(a, &e); /* a = f * 2^e, 0.5 <= f < 1: a lies in [2^(e-1), 2^e) */
  int E = e - 1;
  if (E < emin) E = emin;
  double q = ldexp(a, frac_bits - E); /* a measured in grid spacings (exact scaling) */
  double r = nearbyint(q);            /* default environment: round half to even */
  return ldexp(r, E - frac_bits);
}

static uint16_t double_to_bf16_bits(double v) {
  if (isnan(v)) return 0x7FC0;
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (a == 0.0) return sign;
  double r = isinf(a) ? INFINITY : round_to_grid(a, 7, -126);
  if (r >= ldexp(1.0, 128)) return sign | 0x7F80; /* rounds past the largest finite value */
  float f = (float)r;                            /* exact: r is a bfloat16 value */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return sign | (uint16_t)(u >> 16);
}

static uint16_t double_to_f16_bits(double v) {
  if (isnan(v)) return 0x7E00;
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (a == 0.0) return sign;
  double r = isinf(a) ? INFINITY : round_to_grid(a, 10, -14);
  if (r >= 65536.0) return sign | 0x7C00;
  if (r < ldexp(1.0, -14)) return sign | (uint16_t)ldexp(r, 24); /* subnormal */
  int e;
  double f = frexp(r, &e); /* r = (1 + m/1024) * 2^(e-1) */
  uint16_t m = (uint16_t)(ldexp(f, 11) - 1024.0);
  uint16_t ex = (uint16_t)(e - 1 + 15);
  return sign | (uint16_t)(ex << 10) | m;
}

/* OCP 8-bit E4M3 ("fn": no infinities): sign, 4 exponent bits biased by 7, 3 fraction bits;
 * exponent 15 with fraction 7 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448. */
static double e4m3_bits_to_double(uint8_t h) {
  int neg = h >> 7, e = (h >> 3) & 15, m = h & 7;
  double v;
  if (e == 15 && m == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)m, -9); /* subnormal: m * 2^-9 */
  else
    v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return neg ? -v : v;
}

/* nearest E4M3 value, ties to even, saturating: magnitudes past 448 (and infinities)
 * become 448 */
static uint8_t double_to_e4m3_bits(double v) {
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double a = fabs(v);
  if (a == 0.0) return sign;
  double r = isinf(a) ? 448.0 : round_to_grid(a, 3, -6);
  if (r > 448.0) r = 448.0;
  if (r < ldexp(1.0, -6)) return sign | (uint8_t)ldexp(r, 9); /* subnormal */
  int e;
  double f = frexp(r, &e); /* r = (1 + m/8) * 2^(e-1) */
  uint8_t m = (uint8_t)(ldexp(f, 4) - 8.0);
  return sign | (uint8_t)((e - 1 + 7) << 3) | m;
}

double orc_decode(int32_t dtype, const void *base, int64_t i) {
  if (dtype == ORC_BF16) return bf16_bits_to_double(((const uint16_t *)base)[i]);
  if (dtype == ORC_F16) return f16_bits_to_double(((const uint16_t *)base)[i]);
  if (dtype == ORC_FP8_E4M3) return e4m3_bits_to_double(((const uint8_t *)base)[i]);
  return (double)((const float *)base)[i];
}

void orc_encode(int32_t dtype, void *base, int64_t i, double v) {
  if (dtype == ORC_BF16)
    ((uint16_t *)base)[i] = double_to_bf16_bits(v);
  else if (dtype == ORC_F16)
    ((uint16_t *)base)[i] = double_to_f16_bits(v);
  else if (dtype == ORC_FP8_E4M3)
    ((uint8_t *)base)[i] = double_to_e4m3_bits(v);
  else
    ((float *)base)[i] = (float)v; /* C conversion: round to nearest even */
}

/* A cache element: an FP8 cache holds code = e4m3(value / scale) with one float32 scale per
 * plane (the scale_dtype_ / quantization_granularity_ of the pages' cache collections, read
 * as per-tensor scales); other caches hold the value. */
static double cache_scale(const orc_paged_cache *c, int plane) {
  if (c->dtype != ORC_FP8_E4M3) return 1.0;
  return (double)*(plane ? c->v_scale : c->k_scale);
}
static double cache_get(const orc_paged_cache *c, int plane, int64_t i) {
  return orc_decode(c->dtype, plane ? c->v : c->k, i) * cache_scale(c, plane);
}
static void cache_put(const orc_paged_cache *c, int plane, int64_t i, double v) {
  orc_encode(c->dtype, plane ? c->v : c->k, i, v / cache_scale(c, plane));
}

/* the value v takes once stored in `dtype` */
static double requantize(int32_t dtype, double v) {
  unsigned char tmp[8];
  orc_encode(dtype, tmp, 0, v);
  return orc_decode(dtype, tmp, 0);
}

/* ---------------------------------------------------------------- shared definitions -- */

/* input_row_offsets must partition [0, T): starts at 0, never decreases, ends at T ([P2]
 * Args, [P3] Args: "start of each sequence along the ragged sequence dimension"). */
static uint32_t check_row_offsets(const uint32_t *offs, int32_t batch, int32_t T) {
  if (offs[0] != 0) return ORC_ERR_ROW_OFFSETS;
  for (int32_t b = 0; b < batch; ++b)
    if (offs[b + 1] < offs[b]) return ORC_ERR_ROW_OFFSETS;
  if (offs[batch] != (uint32_t)T) return ORC_ERR_ROW_OFFSETS;
  return 0;
}

/* the sequence b with offs[b] <= row < offs[b+1]; plain linear scan */
static int32_t sequence_of_row(const uint32_t *offs, int32_t batch, int64_t row) {
  for (int32_t b = 0; b < batch; ++b)
    if ((int64_t)offs[b] <= row && row < (int64_t)offs[b + 1]) return b;
  return -1;
}

/* Page-table translation of (sequence, position) in a paged cache: page-table column
 * pos / page_size names the page, pos % page_size the slot inside it. */
static uint32_t paged_slot(const orc_paged_cache *c, int64_t seq, int64_t pos, uint32_t layer,
                           int64_t *elem_base, int64_t *flat_slot) {
  int64_t col = pos / c->page_size;
  if (col >= c->max_pages_per_seq) return ORC_ERR_PAGE_INDEX;
  uint32_t page = c->page_table[seq * c->page_table_stride + col];
  if (page >= (uint32_t)c->num_pages) return ORC_ERR_PAGE_ID;
  int64_t slot = pos % c->page_size;
  *elem_base = (int64_t)page * c->page_stride + (int64_t)layer * c->layer_stride +
               slot * c->slot_stride;
  *flat_slot = (int64_t)page * c->page_size + slot;
  return 0;
}

/* cos/sin row of freqs_cis for position pos: cs[2i] = cos, cs[2i+1] = sin of pair i */
static void load_freqs_row(const orc_rope *rope, int64_t pos, double *cs) {
  for (int32_t j = 0; j < rope->rope_dim; ++j)
    cs[j] = orc_decode(rope->dtype, rope->table, pos * rope->rope_dim + j);
}

static int32_t rope_offset(const orc_rope *rope, int32_t head_dim) {
  return rope->rope_col_offset < 0 ? head_dim - rope->rope_dim : rope->rope_col_offset;
}

/* RoPE of one head row y[0..D): pair i is rotated by the angle whose cosine and sine are
 * cs[2i], cs[2i+1]: (a, b) -> (a cos - b sin, a sin + b cos).  Interleaved pairs are
 * adjacent columns; half-split pairs are rope_dim/2 columns apart ([P2] Parameters). */
static void rope_head(double *y, int32_t head_dim, const orc_rope *rope, const double *cs) {
  int32_t o = rope_offset(rope, head_dim), half = rope->rope_dim / 2;
  for (int32_t i = 0; i < half; ++i) {
    int32_t ia = rope->interleaved ? o + 2 * i : o + i;
    int32_t ib = rope->interleaved ? o + 2 * i + 1 : o + i + half;
    double c = cs[2 * i], s = cs[2 * i + 1];
    double a = y[ia], b = y[ib];
    y[ia] = a * c - b * s;
    y[ib] = a * s + b * c;
  }
}

/* Per-head RMSNorm of y[0..D): y_d * rsqrt(mean_d(y^2) + eps) * (gamma_d + weight_offset)
 * ([P4] signature, [P5] epsilon inside the root).  multiply_before_cast = 0 stores the
 * normalised value in the element type before the gamma multiply. */
static void rmsnorm_head(int32_t dtype, double *y, int32_t D, const void *gamma, double eps,
                         double weight_offset, int32_t multiply_before_cast) {
  double ss = 0.0;
  for (int32_t d = 0; d < D; ++d) ss += y[d] * y[d];
  double r = 1.0 / sqrt(ss / D + eps);
  for (int32_t d = 0; d < D; ++d) {
    double g = orc_decode(dtype, gamma, d) + weight_offset;
    y[d] = multiply_before_cast ? y[d] * r * g : requantize(dtype, y[d] * r) * g;
  }
}

/* ------------------------------------------------------------------ banded store op -- */

/* One band: for every token row, optionally RMSNorm then RoPE its Q heads into q_out,
 * its K heads into the band's cache, and copy its V heads into the cache.  With k_col < 0
 * the K heads are not in the input: they are read from the token's cache slot and updated
 * there in place ([P4]: the key caches are updated in place). */
static uint32_t apply_band(int32_t dtype, orc_band *bd, const uint32_t *offs, int32_t batch,
                           int32_t T, const orc_rope *rope, int32_t do_norm,
                           double weight_offset, int32_t mbc, uint32_t layer) {
  orc_paged_cache *c = bd->cache;
  int32_t D = c->head_dim, Hq = bd->n_q_heads, Hk = c->n_kv_heads;
  const double eps = (double)(float)bd->epsilon; /* the epsilons are Float32 scalars ([P4]) */
  double *y = (double *)malloc(sizeof(double) * (size_t)D);
  double *cs = (double *)malloc(sizeof(double) * (size_t)(rope->rope_dim + 2));
  uint32_t err = 0;
  for (int64_t row = 0; row < T; ++row) {
    int32_t b = sequence_of_row(offs, batch, row);
    int64_t t = row - (int64_t)offs[b];
    int64_t pos = (int64_t)c->cache_lengths[b] + t;
    if (pos >= rope->max_seq_len) {
      err |= ORC_ERR_POSITION;
      continue;
    }
    int64_t base, flat;
    uint32_t e = paged_slot(c, b, pos, layer, &base, &flat);
    if (e) {
      err |= e;
      continue;
    }
    load_freqs_row(rope, pos, cs);
    const int64_t in_row = row * bd->input_row_stride;
    for (int32_t h = 0; h < Hq; ++h) { /* Q heads -> q_out */
      for (int32_t d = 0; d < D; ++d) y[d] = orc_decode(dtype, bd->input, in_row + bd->q_col + (int64_t)h * D + d);
      if (do_norm) rmsnorm_head(dtype, y, D, bd->q_gamma, eps, weight_offset, mbc);
      rope_head(y, D, rope, cs);
      for (int32_t d = 0; d < D; ++d)
        orc_encode(bd->q_out_dtype >= 0 ? bd->q_out_dtype : dtype, bd->q_out,
                   row * bd->q_out_row_stride + (int64_t)h * D + d, y[d]);
    }
    for (int32_t h = 0; h < Hk; ++h) { /* K heads -> K cache (k_col < 0: K is the cache's) */
      for (int32_t d = 0; d < D; ++d)
        y[d] = bd->k_col >= 0
                   ? orc_decode(dtype, bd->input, in_row + bd->k_col + (int64_t)h * D + d)
                   : cache_get(c, 0, base + h * c->head_stride + d);
      if (do_norm) rmsnorm_head(dtype, y, D, bd->k_gamma, eps, weight_offset, mbc);
      rope_head(y, D, rope, cs);
      for (int32_t d = 0; d < D; ++d) cache_put(c, 0, base + h * c->head_stride + d, y[d]);
    }
    if (bd->v_col >= 0) /* V heads -> V cache, unchanged */
      for (int32_t h = 0; h < Hk; ++h)
        for (int32_t d = 0; d < D; ++d)
          cache_put(c, 1, base + h * c->head_stride + d,
                    orc_decode(dtype, bd->input, in_row + bd->v_col + (int64_t)h * D + d));
    if (bd->written) bd->written[flat] = 1;
  }
  free(y);
  free(cs);
  return err;
}

static int rope_geometry_ok(const orc_rope *rope, int32_t head_dim) {
  int32_t o = rope_offset(rope, head_dim);
  return rope->rope_dim >= 0 && rope->rope_dim % 2 == 0 && o >= 0 &&
         o + rope->rope_dim <= head_dim;
}

/* [P2]: Q | K | V column blocks of the flat matmul output, Q roped to q_output, K roped and
 * V unchanged into the paged cache of layer_idx. */
uint32_t orc_rope_split_store_paged_ragged(int32_t dtype, const void *qkv, int64_t qkv_row_stride,
                                           int32_t total_tokens, int32_t n_q_heads,
                                           const uint32_t *input_row_offsets, int32_t batch,
                                           const orc_rope *rope, orc_paged_cache *kv,
                                           uint32_t layer_idx, void *q_out,
                                           int64_t q_out_row_stride, int32_t q_out_dtype,
                                           uint8_t *written) {
  if (layer_idx >= (uint32_t)kv->num_layers || batch > kv->n_seqs ||
      !rope_geometry_ok(rope, kv->head_dim) || kv->v == NULL)
    return ORC_ERR_ARGS;
  uint32_t e = check_row_offsets(input_row_offsets, batch, total_tokens);
  if (e) return e;
  int64_t D = kv->head_dim;
  /* [P2] q_out_dtype: the element type of the Q output (the input's by default) */
  orc_band bd = {qkv, qkv_row_stride, 0, n_q_heads * D, (n_q_heads + kv->n_kv_heads) * D,
                 n_q_heads, kv, NULL, NULL, 0.0, q_out, q_out_row_stride, written,
                 q_out_dtype};
  return apply_band(dtype, &bd, input_row_offsets, batch, total_tokens, rope, 0, 0.0, 1,
                    layer_idx);
}

/* The single-band per-head RMSNorm + RoPE op that [P4] fuses twice. */
uint32_t orc_fused_qk_rmsnorm_rope_paged(int32_t dtype, orc_band *band,
                                         const uint32_t *input_row_offsets, int32_t batch,
                                         int32_t total_tokens, const orc_rope *rope,
                                         double weight_offset, int32_t multiply_before_cast,
                                         uint32_t layer_idx) {
  if (layer_idx >= (uint32_t)band->cache->num_layers || batch > band->cache->n_seqs ||
      !rope_geometry_ok(rope, band->cache->head_dim) ||
      (band->v_col >= 0 && band->cache->v == NULL))
    return ORC_ERR_ARGS;
  uint32_t e = check_row_offsets(input_row_offsets, batch, total_tokens);
  if (e) return e;
  /* weight_offset is a scalar of the element type ([P4] signature) */
  double wo = requantize(dtype, weight_offset);
  return apply_band(dtype, band, input_row_offsets, batch, total_tokens, rope, 1, wo,
                    multiply_before_cast, layer_idx);
}

/* [P4]: one launch = the main band's op followed by the index band's op; both bands share
 * offsets, freqs_cis, weight_offset and layer_idx, and must agree on the rope geometry. */
uint32_t orc_fused_dual_qk_rmsnorm_rope_paged(int32_t dtype, orc_band *main_band,
                                              orc_band *index_band,
                                              const uint32_t *input_row_offsets, int32_t batch,
                                              int32_t total_tokens, const orc_rope *rope,
                                              double weight_offset,
                                              int32_t multiply_before_cast, uint32_t layer_idx) {
  /* one input type and head_dim; each cache holds that type or FP8 codes */
  if (main_band->cache->head_dim != index_band->cache->head_dim) return ORC_ERR_ARGS;
  for (int k = 0; k < 2; ++k) {
    int32_t cd = (k ? index_band : main_band)->cache->dtype;
    if (cd != dtype && cd != ORC_FP8_E4M3) return ORC_ERR_ARGS;
  }
  uint32_t e = orc_fused_qk_rmsnorm_rope_paged(dtype, main_band, input_row_offsets, batch,
                                               total_tokens, rope, weight_offset,
                                               multiply_before_cast, layer_idx);
  if (e & (ORC_ERR_ARGS | ORC_ERR_ROW_OFFSETS)) return e;
  return e | orc_fused_qk_rmsnorm_rope_paged(dtype, index_band, input_row_offsets, batch,
                                             total_tokens, rope, weight_offset,
                                             multiply_before_cast, layer_idx);
}

/* [P1]: per (b, s): inside valid_lengths[b], Q is roped into output and K is roped in place
 * in the continuous cache row of slot lookup_table[b] at position cache_lengths[b] + s;
 * beyond it Q is copied unchanged and K is left alone. */
uint32_t orc_qk_rope_bshd_continuous(int32_t dtype, const void *q_proj, int32_t B, int32_t S,
                                     int32_t n_q_heads, int32_t head_dim, orc_cont_cache *kv,
                                     const orc_rope *rope, uint32_t layer_idx,
                                     const uint32_t *valid_lengths, void *output,
                                     uint8_t *written) {
  if (layer_idx >= (uint32_t)kv->num_layers || B > kv->n_seqs || kv->head_dim != head_dim ||
      !rope_geometry_ok(rope, head_dim))
    return ORC_ERR_ARGS;
  int32_t D = head_dim, Hq = n_q_heads, Hk = kv->n_kv_heads;
  double *y = (double *)malloc(sizeof(double) * (size_t)D);
  double *cs = (double *)malloc(sizeof(double) * (size_t)(rope->rope_dim + 2));
  uint32_t err = 0;
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t s = 0; s < S; ++s) {
      int64_t q_row = (b * S + s) * (int64_t)Hq * D;
      if (s >= (int64_t)valid_lengths[b]) { /* outside the valid length: plain copy */
        for (int64_t j = 0; j < (int64_t)Hq * D; ++j)
          orc_encode(dtype, output, q_row + j, orc_decode(dtype, q_proj, q_row + j));
        continue;
      }
      uint32_t slot = kv->lookup_table[b];
      if (slot >= (uint32_t)kv->num_slots) {
        err |= ORC_ERR_BATCH;
        continue;
      }
      int64_t pos = (int64_t)kv->cache_lengths[b] + s;
      if (pos >= rope->max_seq_len || pos >= kv->max_seq_len) {
        err |= ORC_ERR_POSITION;
        continue;
      }
      load_freqs_row(rope, pos, cs);
      for (int32_t h = 0; h < Hq; ++h) {
        for (int32_t d = 0; d < D; ++d) y[d] = orc_decode(dtype, q_proj, q_row + (int64_t)h * D + d);
        rope_head(y, D, rope, cs);
        for (int32_t d = 0; d < D; ++d) orc_encode(dtype, output, q_row + (int64_t)h * D + d, y[d]);
      }
      int64_t base = (int64_t)slot * kv->slot_stride + (int64_t)layer_idx * kv->layer_stride +
                     pos * kv->pos_stride;
      for (int32_t h = 0; h < Hk; ++h) {
        int64_t rb = base + h * kv->head_stride;
        for (int32_t d = 0; d < D; ++d) y[d] = orc_decode(kv->dtype, kv->k, rb + d);
        rope_head(y, D, rope, cs);
        for (int32_t d = 0; d < D; ++d) orc_encode(kv->dtype, kv->k, rb + d, y[d]);
      }
      if (written) written[(int64_t)slot * kv->max_seq_len + pos] = 1;
    }
  }
  free(y);
  free(cs);
  return err;
}

/* [P3]: cache[K or V][seq + batch_offset, cache_len + t] += a[row, K half or V half]. */
uint32_t orc_kv_cache_radd(int32_t dtype, const void *a, int64_t a_row_stride,
                           int32_t total_tokens, orc_paged_cache *kv,
                           const uint32_t *input_row_offsets, int32_t batch,
                           uint32_t batch_offset, uint32_t layer_idx, uint8_t *written) {
  if (layer_idx >= (uint32_t)kv->num_layers || kv->v == NULL) return ORC_ERR_ARGS;
  uint32_t e = check_row_offsets(input_row_offsets, batch, total_tokens);
  if (e) return e;
  int64_t D = kv->head_dim, Hk = kv->n_kv_heads, hidden = Hk * D;
  uint32_t err = 0;
  for (int64_t row = 0; row < total_tokens; ++row) {
    int32_t b = sequence_of_row(input_row_offsets, batch, row);
    int64_t t = row - (int64_t)input_row_offsets[b];
    int64_t seq = (int64_t)b + batch_offset;
    if (seq >= kv->n_seqs) {
      err |= ORC_ERR_BATCH;
      continue;
    }
    int64_t pos = (int64_t)kv->cache_lengths[seq] + t;
    int64_t base, flat;
    uint32_t pe = paged_slot(kv, seq, pos, layer_idx, &base, &flat);
    if (pe) {
      err |= pe;
      continue;
    }
    for (int64_t h = 0; h < Hk; ++h)
      for (int64_t d = 0; d < D; ++d) {
        int64_t ce = base + h * kv->head_stride + d;
        double ak = orc_decode(dtype, a, row * a_row_stride + h * D + d);
        double av = orc_decode(dtype, a, row * a_row_stride + hidden + h * D + d);
        cache_put(kv, 0, ce, cache_get(kv, 0, ce) + ak);
        cache_put(kv, 1, ce, cache_get(kv, 1, ce) + av);
      }
    if (written) written[flat] = 1;
  }
  return err;
}

/* ------------------------------------------------------- GEMV + partial RMSNorm (P5) -- */

/* [P5] MatmulFusedPartialRMSNorm: y = x W^T for one input row (M = 1), W of shape (n, k);
 * the first n_normed entries of y are RMS-normalised over those entries (epsilon inside
 * the root) and scaled by gamma, the remaining n - n_normed pass through unchanged.
 * weight_offset is accepted and not used, as the page states.  y is exact sums of
 * products in double; every output is rounded once. */
uint32_t orc_matmul_fused_partial_rmsnorm(int32_t dtype, const void *input, const void *weight,
                                          int64_t weight_row_stride, int32_t n, int32_t k,
                                          const void *gamma, double epsilon,
                                          double weight_offset, void *normed_output,
                                          int32_t n_normed, void *unnormed_output) {
  (void)weight_offset; /* not consumed ([P5] Args) */
  if (n < 0 || k < 0 || n_normed < 0 || n_normed > n || weight_row_stride < k) return ORC_ERR_ARGS;
  const double eps = (double)(float)epsilon; /* a Float32 argument ([P5]) */
  double *y = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  for (int64_t i = 0; i < n; ++i) {
    double acc = 0.0;
    for (int64_t j = 0; j < k; ++j)
      acc += orc_decode(dtype, input, j) * orc_decode(dtype, weight, i * weight_row_stride + j);
    y[i] = acc;
  }
  double ss = 0.0;
  for (int64_t i = 0; i < n_normed; ++i) ss += y[i] * y[i];
  const double r = n_normed > 0 ? 1.0 / sqrt(ss / n_normed + eps) : 0.0;
  for (int64_t i = 0; i < n_normed; ++i)
    orc_encode(dtype, normed_output, i, y[i] * r * orc_decode(dtype, gamma, i));
  for (int64_t i = n_normed; i < n; ++i) orc_encode(dtype, unnormed_output, i - n_normed, y[i]);
  free(y);
  return 0;
}
