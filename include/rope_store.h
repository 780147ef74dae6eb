/*
 * rope_store.h -- attention-prologue kernels for NVIDIA B200 (sm_100a): RoPE, per-head
 * RMSNorm and paged / continuous K/V-cache stores, behind a plain C ABI.
 *
 * The operations follow five Modular MAX kernel reference pages; each entry point below
 * names the page and the part of it that defines the operation.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every pointer argument is a device pointer owned by the caller (destination-
 *           passing style: the caller allocates every output, as the pages' signatures do
 *           for their output tensors).  Descriptor structs (rope_freqs_t,
 *           rope_paged_cache_t, ...) live in host memory and are read only during the call.
 *           The library allocates, frees and synchronises nothing.
 * Streams.  Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *           default stream).  Work on one stream runs in order, which is what orders a
 *           store after the projection that produced its input.
 * Layout.   Rows are token-major; strides are in ELEMENTS.  Within a row, heads are
 *           contiguous blocks of head_dim elements.  All tensor base pointers, row strides
 *           and column offsets must keep every head row 16-byte aligned.
 * Types.    Element types: ROPE_DTYPE_BF16, ROPE_DTYPE_F16, ROPE_DTYPE_F32.  A cache holds
 *           the input's element type, or ROPE_DTYPE_FP8_E4M3 codes (see rope_paged_cache_t).
 *           freqs_cis may be F32, BF16 or F16.  head_dim is 64, 128 or 256 (64 or 128 for
 *           F32 elements).
 * Math.     Values are widened to float32, normalised and rotated in float32, and rounded
 *           once, to nearest even, into the output type.  V heads and columns that are
 *           neither normalised nor rotated are copied bit for bit.
 * Status.   The return value reports argument problems found on the host before any
 *           launch (nothing is written then) and launch failures.  total_tokens == 0 (or
 *           batch*seq_len == 0) returns ROPE_OK at once, without a launch and without
 *           looking at the other arguments (empty tensors may have NULL data).
 * Device errors.  Problems that depend on device data are found by the kernel: it ORs the
 *           ROPE_DEVERR_* bits into *err_word (if err_word is not NULL) and skips the
 *           affected token, writing none of its outputs; other tokens are unaffected.  If
 *           input_row_offsets is not a partition of [0, total_tokens) (first entry 0,
 *           non-decreasing, last entry total_tokens) the whole call writes nothing.  The
 *           kernels never trap and never wait on other blocks.
 * Schedule. The calls that stage token rows (the three paged stores and kv_cache_radd)
 *           take `sched`: NULL, or ROPE_SCHED_WORDS uint32 words of device memory (the
 *           scheduling workspace).  With NULL every CTA processes a fixed strided share of
 *           the tokens.  With a workspace each CTA takes most of its share that way and
 *           then claims the remaining tokens in small chunks from a counter in the
 *           workspace, so that CTAs which get more memory bandwidth take more of the tail;
 *           the results are the same either way.  The words must be zero before the first
 *           call that uses them (e.g. cudaMemsetAsync once after allocating); every call
 *           leaves them zero when it completes.  Calls that can run at the same time (on
 *           different streams) need separate workspaces; calls in one stream may share one.
 * Overlap.  By default (ROPE_OVERLAP_PDL) every kernel is launched as a programmatic
 *           dependent of the previous kernel in its stream: its CTAs may start while that
 *           kernel finishes, and wait for it to complete before they touch global memory.
 *           ROPE_OVERLAP_PDL_EARLY_METADATA additionally reads the descriptor arrays
 *           (input_row_offsets, cache_lengths, page tables, lookup tables, valid_lengths,
 *           gammas) before that wait: only valid when no kernel still running ahead in the
 *           stream writes them (e.g. they were uploaded before the layer's kernels were
 *           queued).  ROPE_OVERLAP_OFF launches plainly.  See rope_set_launch_overlap.
 */
#ifndef ROPE_STORE_H
#define ROPE_STORE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *rope_stream_t; /* same type as cudaStream_t */

typedef enum {
  ROPE_OK = 0,
  ROPE_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, inconsistent geometry */
  ROPE_ERR_UNSUPPORTED = 2, /* dtype / head_dim / rope geometry / alignment not supported */
  ROPE_ERR_CUDA = 3         /* the launch failed (cudaGetLastError() has the cause) */
} rope_status_t;

typedef enum {
  ROPE_DTYPE_BF16 = 0,
  ROPE_DTYPE_F16 = 1,
  ROPE_DTYPE_F32 = 2,
  ROPE_DTYPE_FP8_E4M3 = 3 /* paged caches only: OCP E4M3 codes with per-plane scales */
} rope_dtype_t;

/* bits of *err_word */
#define ROPE_DEVERR_ROW_OFFSETS 0x1u /* input_row_offsets is not a partition of [0, T) */
#define ROPE_DEVERR_POSITION 0x2u    /* position >= rows of freqs_cis (or of the cache) */
#define ROPE_DEVERR_PAGE_INDEX 0x4u  /* position / page_size >= max_pages_per_seq */
#define ROPE_DEVERR_PAGE_ID 0x8u     /* page-table entry >= num_pages */
#define ROPE_DEVERR_BATCH 0x10u      /* sequence (+ batch_offset) >= n_seqs, or slot >= num_slots */
#define ROPE_DEVERR_TIMEOUT 0x20u    /* an internal pipeline wait gave up (the call is incomplete) */

/* uint32 words of a scheduling workspace (see Schedule above) */
#define ROPE_SCHED_WORDS 2

typedef enum {
  ROPE_OVERLAP_OFF = 0,               /* plain launches */
  ROPE_OVERLAP_PDL = 1,               /* programmatic dependent launch (the default) */
  ROPE_OVERLAP_PDL_EARLY_METADATA = 2 /* as PDL, descriptor arrays read before the wait */
} rope_overlap_t;

/* freqs_cis [max_seq_len, rope_dim], row-major, contiguous.  Row p holds rope_dim/2
 * pairs (cos, sin): column 2i is cos and 2i+1 is sin of pair i's angle at position p (the
 * table argument of the rope_split_store_paged_ragged page, Args, stores the two parts of
 * each rotation next to each other).
 * rope_dim = the table's column count (fused_dual_qk_rms_norm_rope_ragged_paged, second
 * paragraph: rope_dim comes from freqs_cis's second dimension); it is even, at most
 * head_dim, and rope_dim < head_dim means partial RoPE.
 * interleaved != 0: pair i of a head is columns (o + 2i, o + 2i + 1): the real and
 *   imaginary parts side by side (rope_split_store_paged_ragged, Parameters, interleaved);
 * interleaved == 0: pair i is columns (o + i, o + i + rope_dim/2) (half-split layout).
 * o = rope_col_offset, or head_dim - rope_dim when rope_col_offset < 0: partial RoPE
 * rotates the last rope_dim columns of each head unless the caller says otherwise.
 * Supported: o and rope_dim multiples of the 16-byte vector width (8 elements for 16-bit
 * types, 4 for F32), and for the half-split layout rope_dim/2 too; a table row
 * (rope_dim * element size) is a multiple of 16 bytes and the table is 16-byte aligned. */
typedef struct {
  const void *data;
  int32_t dtype; /* rope_dtype_t of the table */
  int32_t max_seq_len;
  int32_t rope_dim;
  int32_t interleaved;
  int32_t rope_col_offset;
} rope_freqs_t;

/* A paged K/V cache (PagedKVCacheCollection on the pages).  Element (page, layer, slot,
 * head, d) of the K plane is
 *     k[page*page_stride + layer*layer_stride + slot*slot_stride + head*head_stride + d]
 * and of the V plane likewise from v (v may be NULL for a K-only cache).  A sequence's
 * position p lives in page page_table[seq*page_table_stride + p / page_size] at slot
 * p % page_size.  cache_lengths[seq] = tokens the sequence already holds; new token t of
 * the sequence goes to position cache_lengths[seq] + t.  page_table and cache_lengths are
 * device arrays with n_seqs rows. */
typedef struct {
  void *k;
  void *v;
  int32_t dtype;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t num_pages;
  int32_t num_layers;
  int64_t page_stride, layer_stride, slot_stride, head_stride; /* elements */
  const uint32_t *page_table;
  int64_t page_table_stride; /* elements between consecutive sequences' rows */
  int32_t max_pages_per_seq; /* usable entries of a page-table row */
  const uint32_t *cache_lengths;
  int32_t n_seqs;
  /* dtype == ROPE_DTYPE_FP8_E4M3: one float32 scale per plane (device pointers); an element
   * holds the E4M3 code nearest to value / scale (ties to even, saturating at +-448).  The
   * pages' cache collections carry a scale type and a quantisation granularity without
   * defining them; this per-plane reading is this library's.  FP8 caches are written by the
   * three paged stores (K rotated, V copied; not with K updated in place) and rejected
   * (ROPE_ERR_UNSUPPORTED) by kv_cache_radd.  Ignored for other dtypes (may be NULL). */
  const float *k_scale;
  const float *v_scale;
} rope_paged_cache_t;

/* A continuous-batching K/V cache (ContinuousBatchingKVCacheCollection on the pages).
 * Batch entry b owns slot lookup_table[b]; element (slot, layer, pos, head, d) of the K
 * plane is k[slot*slot_stride + layer*layer_stride + pos*pos_stride + head*head_stride + d].
 * lookup_table and cache_lengths are device arrays with n_seqs entries. */
typedef struct {
  void *k;
  void *v;
  int32_t dtype;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t num_slots;
  int32_t num_layers;
  int32_t max_seq_len;
  int64_t slot_stride, layer_stride, pos_stride, head_stride; /* elements */
  const uint32_t *lookup_table;
  const uint32_t *cache_lengths;
  int32_t n_seqs;
} rope_cont_cache_t;

/* One band of the dual per-head RMSNorm + RoPE launch: its Q heads start at column q_col,
 * its K heads at k_col and its V heads at v_col (v_col < 0: the band's cache is K-only, or
 * its V is not stored) of the token-major `input` (the pages' per-band Q read lambdas become
 * a base pointer, a row stride and column offsets).  k_col < 0: the band's K heads are not
 * in the input; they are read from the token's cache slot, normalised, rotated and written
 * back to that slot (the key cache updated in place, fused_dual_qk_rms_norm_rope_ragged_paged
 * first paragraph).  q_gamma / k_gamma: [head_dim] in the element type, shared by
 * all Q (K) heads of the band.  epsilon: the band's RMSNorm epsilon.  q_out: [T, n_q_heads *
 * head_dim] rows with stride q_out_row_stride. */
typedef struct {
  const void *input;
  int64_t input_row_stride;
  int64_t q_col, k_col, v_col;
  int32_t n_q_heads;
  const rope_paged_cache_t *cache;
  const void *q_gamma;
  const void *k_gamma;
  float epsilon;
  void *q_out;
  int64_t q_out_row_stride;
} rope_norm_band_t;

/* rope_split_store_paged_ragged -- rotate Q and K of a flat ragged QKV batch, write Q
 * out and store K and V into a paged cache (rope_split_store_paged_ragged page: signature,
 * Parameters, Args).
 *   qkv [total_tokens, (n_q_heads + 2*n_kv_heads) * head_dim], row stride qkv_row_stride:
 *       the flat matmul output, columns Q | K | V, of element type qkv_dtype (rope_dtype_t;
 *       < 0: the cache's element type; with an FP8 cache that is ROPE_ERR_UNSUPPORTED).
 *   input_row_offsets [batch + 1]: sequence b owns rows [offs[b], offs[b+1]).
 *   Row r of sequence b sits at position p = kv->cache_lengths[b] + (r - offs[b]).
 *   Q heads are rotated with freqs_cis row p and written to q_out [total_tokens, n_q_heads *
 *   head_dim] (row stride q_out_row_stride, in q_out elements); K heads are rotated and V
 *   heads copied into the cache of layer layer_idx at position p.  kv->v must not be NULL.
 *   q_out_dtype (rope_dtype_t; < 0: the cache's element type) is the element type of q_out
 *   (the page's q_out_dtype parameter, which defaults to dtype): rotated values are rounded
 *   once into it and unrotated columns converted exactly or rounded once. */
rope_status_t rope_split_store_paged_ragged(const void *qkv, int64_t qkv_row_stride,
                                            int32_t qkv_dtype, int32_t total_tokens,
                                            int32_t n_q_heads,
                                            const uint32_t *input_row_offsets, int32_t batch,
                                            const rope_freqs_t *freqs,
                                            const rope_paged_cache_t *kv, uint32_t layer_idx,
                                            void *q_out, int64_t q_out_row_stride,
                                            int32_t q_out_dtype, uint32_t *err_word,
                                            uint32_t *sched, rope_stream_t stream);

/* fused_qk_rmsnorm_rope_paged -- the single-band per-head RMSNorm + RoPE + paged store that
 * the fused_dual_qk_rms_norm_rope_ragged_paged page fuses twice (its first paragraph).
 * As rope_split_store_paged_ragged, but each Q (K) head row x of head_dim elements first
 * becomes x * rsqrt(mean(x^2) + epsilon) * (gamma + weight_offset) with gamma = q_gamma
 * (k_gamma); RoPE then rotates that normalised row (no rounding in between).
 * weight_offset is a scalar of the element type (the page's Scalar[dtype]): it is rounded
 * to the element type first.  multiply_before_cast != 0: the normalised row is multiplied
 * by gamma before any rounding.  multiply_before_cast == 0: the normalised value
 * x * rsqrt(mean(x^2) + epsilon) is rounded to the element type first and then multiplied
 * by (gamma + weight_offset); RoPE follows in float32 and the result is rounded once more
 * (the pages name the flag but do not define it; this is the reading taken). */
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
                                          uint32_t *sched, rope_stream_t stream);

/* fused_dual_qk_rmsnorm_rope_paged -- fused_dual_qk_rms_norm_rope_ragged_paged page
 * (signature and both paragraphs): the main band and the index band in ONE launch.  Both
 * bands share input_row_offsets, total_tokens, freqs_cis, weight_offset,
 * multiply_before_cast and layer_idx; each has its own input columns, cache, gammas,
 * epsilon and Q output, and each band's positions come from its own cache_lengths.  The
 * rope geometry must agree across bands: one input element type input_dtype (< 0: the main
 * cache's) and the same head_dim in both caches, each cache holding that type or FP8 codes
 * (else ROPE_ERR_INVALID_ARG, the runtime form of the page's compile-time assert).  The
 * result equals fused_qk_rmsnorm_rope_paged on the main band followed by the same on the
 * index band.  index_band may be NULL: the launch then has the main band alone (the general
 * single-band form, e.g. for K updated in place). */
rope_status_t fused_dual_qk_rmsnorm_rope_paged(const rope_norm_band_t *main_band,
                                               const rope_norm_band_t *index_band,
                                               int32_t input_dtype,
                                               const uint32_t *input_row_offsets,
                                               int32_t batch, int32_t total_tokens,
                                               const rope_freqs_t *freqs, float weight_offset,
                                               int32_t multiply_before_cast, uint32_t layer_idx,
                                               uint32_t *err_word, uint32_t *sched,
                                               rope_stream_t stream);

/* qk_rope_bshd_continuous -- generic_fused_qk_rope_bshd_continuous_batch page (signature,
 * description, Args).  q_proj and output: [batch, seq_len, n_q_heads, head_dim],
 * contiguous.  For s < valid_lengths[b] (device array [batch]): position p =
 * kv->cache_lengths[b] + s; Q head rows are rotated with freqs_cis row p into output, and
 * the K head rows at (kv->lookup_table[b], layer_idx, p) are rotated IN PLACE in the cache.
 * For s >= valid_lengths[b]: output = q_proj unchanged and the cache is not touched.
 * p must be below both freqs->max_seq_len and kv->max_seq_len (else ROPE_DEVERR_POSITION
 * and the token is skipped). */
rope_status_t qk_rope_bshd_continuous(const void *q_proj, int32_t batch, int32_t seq_len,
                                      int32_t n_q_heads, int32_t head_dim,
                                      const rope_cont_cache_t *kv, const rope_freqs_t *freqs,
                                      uint32_t layer_idx, const uint32_t *valid_lengths,
                                      void *output, uint32_t *err_word, rope_stream_t stream);

/* kv_cache_radd -- generic_kv_cache_radd_dispatch page (description, Args).  a
 * [total_tokens, 2 * n_kv_heads * head_dim], row stride a_row_stride: the first
 * n_kv_heads*head_dim columns are added into K, the rest into V.  Row r of sequence b
 * targets cache sequence b' = b + batch_offset at position kv->cache_lengths[b'] +
 * (r - offs[b]) of layer layer_idx.  Each cache element becomes the float32 sum rounded
 * once to the element type (for 16-bit types this equals the correctly rounded exact sum).
 * kv->v must not be NULL. */
rope_status_t kv_cache_radd(const void *a, int64_t a_row_stride, int32_t total_tokens,
                            const rope_paged_cache_t *kv, const uint32_t *input_row_offsets,
                            int32_t batch, uint32_t batch_offset, uint32_t layer_idx,
                            uint32_t *err_word, uint32_t *sched, rope_stream_t stream);

/* matmul_fused_partial_rmsnorm -- MatmulFusedPartialRMSNorm page (description, execute,
 * Args): the one-row GEMV y = input W^T (M = 1) fused with an RMSNorm over its first
 * n_normed entries.
 *   input [k], weight [n, k] row-major with row stride weight_row_stride (elements) -- the
 *   page's default transpose_b = True; transpose_b = 0 (weight stored [k, n]) returns
 *   ROPE_ERR_UNSUPPORTED.  gamma [n_normed].
 *   normed_output [n_normed] = y[i] * rsqrt(mean(y[0..n_normed)^2) + epsilon) * gamma[i];
 *   unnormed_output [n - n_normed] = y[n_normed..n) unchanged.
 *   weight_offset is accepted and not used, as the page states.
 *   dtype (rope_dtype_t) is the element type of every tensor; y is accumulated in float32
 *   and each output rounded once.  k * element size must be a multiple of 16 bytes, and
 *   input / weight / workspace 16-byte aligned.
 *   err_word: as for the other calls (only ROPE_DEVERR_TIMEOUT can occur here).
 *   workspace: device memory of at least ROPE_GEMV_WORKSPACE_BYTES(n_normed) bytes (may be
 *   NULL when n_normed == 0) whose first word must be zero before the first call that uses
 *   it; every call leaves it zero.  It holds the float32 entries to be normalised until the
 *   last CTA normalises them.  Calls that can run at the same time need separate
 *   workspaces. */
#define ROPE_GEMV_WORKSPACE_BYTES(n_normed) (16 + 4 * (int64_t)(n_normed))
rope_status_t matmul_fused_partial_rmsnorm(const void *input, const void *weight,
                                           int64_t weight_row_stride, int32_t n, int32_t k,
                                           int32_t transpose_b, const void *gamma,
                                           float epsilon, float weight_offset,
                                           void *normed_output, int32_t n_normed,
                                           void *unnormed_output, int32_t dtype,
                                           uint32_t *err_word, void *workspace,
                                           int64_t workspace_bytes, rope_stream_t stream);

/* rope_split_store_paged_ragged_noalloc -- rope_split_store_paged_ragged with the
 * claimed-tail schedule, for callers that cannot allocate device memory: for example a
 * plug-in inside an engine that hands out all device memory from its own pool and allows no
 * other allocation, or code on a latency-critical path that must not call cudaMalloc or
 * cudaFree (either may synchronise the device).  The pages have no counterpart of this
 * call; it is a launch variant, not a different operation.
 * Arguments and results are those of rope_split_store_paged_ragged without `sched`: the
 * scheduling workspace is a 256-byte array inside the library, one per device, of which the
 * schedule uses ROPE_SCHED_WORDS words whatever the call's sizes (so no size is too large
 * for it).  The call allocates nothing; after its argument checks it clears those words
 * on `stream` and launches (a rejected call, or one with nothing to do, queues nothing).
 * The first call in a CUDA context looks up the array's device address in that context
 * (with the device current) and keeps it for later calls in the same context; a context
 * made later on the device (after a device reset) gets a lookup of its own.  Make that
 * first call before any stream capture.  Every call on a device shares the array, so calls
 * that can overlap on the GPU (different streams) race on it and may skip tokens: keep the
 * calls of this entry point in one stream, or use rope_split_store_paged_ragged with a
 * workspace per stream.  ROPE_ERR_CUDA if the lookup or the clearing fails. */
rope_status_t rope_split_store_paged_ragged_noalloc(
    const void *qkv, int64_t qkv_row_stride, int32_t qkv_dtype, int32_t total_tokens,
    int32_t n_q_heads,
    const uint32_t *input_row_offsets, int32_t batch, const rope_freqs_t *freqs,
    const rope_paged_cache_t *kv, uint32_t layer_idx, void *q_out, int64_t q_out_row_stride,
    int32_t q_out_dtype, uint32_t *err_word, rope_stream_t stream);

/* A static, human-readable name of a status code. */
const char *rope_status_string(rope_status_t status);

/* Launch-overlap mode (rope_overlap_t) of every launch that follows, process-wide; not a
 * kernel of the method but a launch option (Overlap above).  Returns ROPE_ERR_INVALID_ARG
 * for an unknown mode, leaving the mode as it was. */
rope_status_t rope_set_launch_overlap(int32_t mode);
int32_t rope_get_launch_overlap(void);

/* A diagnostic of the failure path, not an operation of the pages.  With timeout_us > 0,
 * every launch that follows of the staged kernels (the three paged stores, kv_cache_radd,
 * matmul_fused_partial_rmsnorm) starts with one wait that nothing ever completes (an
 * mbarrier no thread arrives at), bounded by timeout_us instead of the usual 2 s.  When it
 * runs out the kernel does what it does when any of its waits runs out: it sets
 * ROPE_DEVERR_TIMEOUT, every CTA leaves its loops after letting its in-flight copies land
 * (those waits keep the full limit), and the call returns incomplete.  0 (the default) turns
 * it off.  Process-wide; timeout_us above 1000000 is ROPE_ERR_INVALID_ARG. */
rope_status_t rope_set_stall_test(uint32_t timeout_us);
uint32_t rope_get_stall_test(void);

#ifdef __cplusplus
}
#endif
#endif /* ROPE_STORE_H */
