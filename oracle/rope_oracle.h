/*
 * rope_oracle.h -- plain, slow, double-precision CPU oracle for the attention-prologue
 * operations documented on five Modular MAX kernel reference pages:
 *
 *   "rope_split_store_paged_ragged"                (RoPE + split + paged K/V store)
 *   "fused_dual_qk_rms_norm_rope_ragged_paged"     (per-head RMSNorm + RoPE, two caches)
 *   "generic_fused_qk_rope_bshd_continuous_batch"  (BSHD Q/K RoPE, continuous cache)
 *   "generic_kv_cache_radd_dispatch"               (in-place add into the K/V cache)
 *   "MatmulFusedPartialRMSNorm"                    (GEMV + partial RMSNorm)
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or helper with
 * the CUDA library; it has its own element codecs, its own descriptors and its own error
 * constants (numerically equal to the CUDA library's, because they are part of the
 * documented contract the tests compare).
 *
 * Arithmetic: every value is widened to double, every step is evaluated in double in the
 * order the definition states, and each output element is rounded exactly once, with
 * round-to-nearest-even, to the output element type.
 *
 * multiply_before_cast = 0 is parity unpinned: the pages name the flag without defining it.
 * The reading implemented rounds the normalised value to the element type before the gamma
 * multiply (a second rounding ahead of the final one).
 */
#ifndef ROPE_ORACLE_H
#define ROPE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element type codes */
enum { ORC_BF16 = 0, ORC_F16 = 1, ORC_F32 = 2, ORC_FP8_E4M3 = 3 };

/* data-dependent error bits (returned; same meaning as the device error word) */
#define ORC_ERR_ROW_OFFSETS 0x1u /* input_row_offsets is not a partition of [0, T) */
#define ORC_ERR_POSITION 0x2u    /* position >= rows of freqs_cis (or of the cache) */
#define ORC_ERR_PAGE_INDEX 0x4u  /* position / page_size >= page-table row length */
#define ORC_ERR_PAGE_ID 0x8u     /* page-table entry >= num_pages */
#define ORC_ERR_BATCH 0x10u      /* sequence index (+ batch_offset) or slot out of range */
#define ORC_ERR_ARGS 0x80000000u /* the oracle was handed inconsistent arguments */

/* A paged K/V cache: element (page, layer, slot, head, d) of the K plane lives at
 * k[page*page_stride + layer*layer_stride + slot*slot_stride + head*head_stride + d]
 * (the V plane likewise from v; v == NULL for a K-only cache). */
typedef struct {
  void *k, *v;
  int32_t dtype;
  int32_t n_kv_heads, head_dim, page_size, num_pages, num_layers;
  int64_t page_stride, layer_stride, slot_stride, head_stride;
  const uint32_t *page_table; /* [n_seqs, page_table_stride], first max_pages_per_seq used */
  int64_t page_table_stride;
  int32_t max_pages_per_seq;
  const uint32_t *cache_lengths; /* [n_seqs] tokens already cached per sequence */
  int32_t n_seqs;
  /* FP8 (ORC_FP8_E4M3) caches: one float32 scale per plane; an element holds
   * e4m3(value / scale), rounded to nearest even and saturated at +-448.  Parity unpinned:
   * the pages name a scale type and a quantisation granularity without defining them. */
  const float *k_scale, *v_scale;
} orc_paged_cache;

/* A continuous-batching K/V cache: element (slot, layer, pos, head, d) of the K plane at
 * k[slot*slot_stride + layer*layer_stride + pos*pos_stride + head*head_stride + d]. */
typedef struct {
  void *k, *v;
  int32_t dtype;
  int32_t n_kv_heads, head_dim, num_slots, num_layers, max_seq_len;
  int64_t slot_stride, layer_stride, pos_stride, head_stride;
  const uint32_t *lookup_table;  /* [n_seqs] batch entry -> cache slot */
  const uint32_t *cache_lengths; /* [n_seqs] */
  int32_t n_seqs;
} orc_cont_cache;

/* freqs_cis: row p holds rope_dim/2 interleaved (cos, sin) pairs for position p. */
typedef struct {
  const void *table;
  int32_t dtype;       /* ORC_F32 or ORC_BF16 (or ORC_F16) */
  int32_t max_seq_len; /* rows */
  int32_t rope_dim;    /* columns, even, <= head_dim */
  int32_t interleaved; /* 1: pairs (o+2i, o+2i+1); 0: pairs (o+i, o+i+rope_dim/2) */
  int32_t rope_col_offset; /* o: first rotated column of a head; -1 means head_dim - rope_dim */
} orc_rope;

/* One band of the dual launch (or the only band of the single-cache norm op). */
typedef struct {
  const void *input;       /* token-major rows */
  int64_t input_row_stride;
  int64_t q_col, k_col, v_col; /* first column of Q / K / V heads; v_col < 0: K-only;
                                  k_col < 0: K is read from the cache slot (in place) */
  int32_t n_q_heads;
  orc_paged_cache *cache;
  const void *q_gamma, *k_gamma; /* [head_dim] each, element type = dtype */
  double epsilon;
  void *q_out;
  int64_t q_out_row_stride;
  uint8_t *written; /* optional [num_pages*page_size]: set to 1 for each (page, slot) stored */
  int32_t q_out_dtype; /* element type of q_out; < 0: the input's */
} orc_band;

uint32_t orc_rope_split_store_paged_ragged(int32_t dtype, const void *qkv, int64_t qkv_row_stride,
                                           int32_t total_tokens, int32_t n_q_heads,
                                           const uint32_t *input_row_offsets, int32_t batch,
                                           const orc_rope *rope, orc_paged_cache *kv,
                                           uint32_t layer_idx, void *q_out,
                                           int64_t q_out_row_stride, int32_t q_out_dtype,
                                           uint8_t *written);

uint32_t orc_fused_qk_rmsnorm_rope_paged(int32_t dtype, orc_band *band,
                                         const uint32_t *input_row_offsets, int32_t batch,
                                         int32_t total_tokens, const orc_rope *rope,
                                         double weight_offset, int32_t multiply_before_cast,
                                         uint32_t layer_idx);

uint32_t orc_fused_dual_qk_rmsnorm_rope_paged(int32_t dtype, orc_band *main_band,
                                              orc_band *index_band,
                                              const uint32_t *input_row_offsets, int32_t batch,
                                              int32_t total_tokens, const orc_rope *rope,
                                              double weight_offset,
                                              int32_t multiply_before_cast, uint32_t layer_idx);

uint32_t orc_qk_rope_bshd_continuous(int32_t dtype, const void *q_proj, int32_t B, int32_t S,
                                     int32_t n_q_heads, int32_t head_dim, orc_cont_cache *kv,
                                     const orc_rope *rope, uint32_t layer_idx,
                                     const uint32_t *valid_lengths, void *output,
                                     uint8_t *written);

uint32_t orc_kv_cache_radd(int32_t dtype, const void *a, int64_t a_row_stride,
                           int32_t total_tokens, orc_paged_cache *kv,
                           const uint32_t *input_row_offsets, int32_t batch,
                           uint32_t batch_offset, uint32_t layer_idx, uint8_t *written);

/* "MatmulFusedPartialRMSNorm": y = x W^T (one input row, W of shape (n, k), row stride
 * weight_row_stride); normed_output = the first n_normed entries of y RMS-normalised over
 * themselves and scaled by gamma [n_normed]; unnormed_output = the other n - n_normed
 * entries.  weight_offset is not used (as documented). */
uint32_t orc_matmul_fused_partial_rmsnorm(int32_t dtype, const void *input, const void *weight,
                                          int64_t weight_row_stride, int32_t n, int32_t k,
                                          const void *gamma, double epsilon,
                                          double weight_offset, void *normed_output,
                                          int32_t n_normed, void *unnormed_output);

/* element codecs, exported so that the self-tests can pin them */
double orc_decode(int32_t dtype, const void *base, int64_t i);
void orc_encode(int32_t dtype, void *base, int64_t i, double v);

#ifdef __cplusplus
}
#endif
#endif
