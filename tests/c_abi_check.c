/* A plain C99 program against include/rope_store.h and librope_store.so: the header
 * compiles as C and the library answers from C.  Only calls that return before any CUDA
 * launch are made (empty work and arguments the host checks reject), so no GPU is needed;
 * the pointers below are never dereferenced.  Prints "ok" and exits 0 when every answer is
 * the documented one. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "rope_store.h"

static int failures = 0;

static void expect(const char *what, int got, int want) {
  if (got != want) {
    printf("%s: got %d, want %d\n", what, got, want);
    ++failures;
  }
}

int main(void) {
  /* a non-null, 16-byte aligned address standing for device memory */
  void *fake = (void *)(uintptr_t)(1u << 20);
  rope_freqs_t freqs;
  rope_paged_cache_t kv;
  rope_norm_band_t band;
  rope_cont_cache_t cc;
  const char *s;

  memset(&freqs, 0, sizeof freqs);
  freqs.data = fake;
  freqs.dtype = ROPE_DTYPE_F32;
  freqs.max_seq_len = 64;
  freqs.rope_dim = 64;
  freqs.interleaved = 1;
  freqs.rope_col_offset = -1;

  memset(&kv, 0, sizeof kv);
  kv.k = fake;
  kv.v = fake;
  kv.dtype = ROPE_DTYPE_BF16;
  kv.n_kv_heads = 2;
  kv.head_dim = 64;
  kv.page_size = 16;
  kv.num_pages = 8;
  kv.num_layers = 2;
  kv.page_stride = 4096;
  kv.layer_stride = 2048;
  kv.slot_stride = 128;
  kv.head_stride = 64;
  kv.page_table = (const uint32_t *)fake;
  kv.page_table_stride = 4;
  kv.max_pages_per_seq = 4;
  kv.cache_lengths = (const uint32_t *)fake;
  kv.n_seqs = 2;

  s = rope_status_string(ROPE_ERR_INVALID_ARG);
  if (s == NULL || s[0] == '\0') {
    printf("rope_status_string returned nothing\n");
    ++failures;
  }

  /* empty work: OK without a launch */
  expect("empty store",
         rope_split_store_paged_ragged(fake, 512, ROPE_DTYPE_BF16, 0, 4,
                                       (const uint32_t *)fake, 2, &freqs, &kv, 1, fake, 256,
                                       -1, NULL, NULL, NULL),
         ROPE_OK);
  /* NULL freqs descriptor, layer past num_layers, odd rope_dim */
  expect("null freqs",
         rope_split_store_paged_ragged(fake, 512, ROPE_DTYPE_BF16, 8, 4,
                                       (const uint32_t *)fake, 2, NULL, &kv, 1, fake, 256, -1,
                                       NULL, NULL, NULL),
         ROPE_ERR_INVALID_ARG);
  expect("layer",
         rope_split_store_paged_ragged(fake, 512, ROPE_DTYPE_BF16, 8, 4,
                                       (const uint32_t *)fake, 2, &freqs, &kv, 2, fake, 256,
                                       -1, NULL, NULL, NULL),
         ROPE_ERR_INVALID_ARG);
  freqs.rope_dim = 63;
  expect("odd rope_dim",
         rope_split_store_paged_ragged(fake, 512, ROPE_DTYPE_BF16, 8, 4,
                                       (const uint32_t *)fake, 2, &freqs, &kv, 1, fake, 256,
                                       -1, NULL, NULL, NULL),
         ROPE_ERR_INVALID_ARG);
  freqs.rope_dim = 64;
  /* an FP8 cache does not tell the input's element type */
  kv.dtype = ROPE_DTYPE_FP8_E4M3;
  expect("fp8 cache, input type from the cache",
         rope_split_store_paged_ragged(fake, 512, -1, 8, 4, (const uint32_t *)fake, 2, &freqs,
                                       &kv, 1, fake, 256, -1, NULL, NULL, NULL),
         ROPE_ERR_UNSUPPORTED);
  kv.dtype = ROPE_DTYPE_BF16;
  /* the norm op needs both gammas */
  expect("norm without q_gamma",
         fused_qk_rmsnorm_rope_paged(fake, 512, ROPE_DTYPE_BF16, 8, 4, (const uint32_t *)fake,
                                     2, &freqs, &kv, NULL, fake, 1e-6f, 0.0f, 1, 1, fake, 256,
                                     NULL, NULL, NULL),
         ROPE_ERR_INVALID_ARG);
  /* dual band with no main band */
  memset(&band, 0, sizeof band);
  expect("dual without main band",
         fused_dual_qk_rmsnorm_rope_paged(NULL, &band, ROPE_DTYPE_BF16, (const uint32_t *)fake,
                                          2, 8, &freqs, 0.0f, 1, 1, NULL, NULL, NULL),
         ROPE_ERR_INVALID_ARG);
  /* radd needs a V plane */
  kv.v = NULL;
  expect("radd without V",
         kv_cache_radd(fake, 256, 8, &kv, (const uint32_t *)fake, 2, 0, 1, NULL, NULL, NULL),
         ROPE_ERR_INVALID_ARG);
  kv.v = fake;
  /* BSHD: head_dim must match the cache */
  memset(&cc, 0, sizeof cc);
  cc.k = fake;
  cc.dtype = ROPE_DTYPE_BF16;
  cc.n_kv_heads = 2;
  cc.head_dim = 64;
  cc.num_slots = 4;
  cc.num_layers = 1;
  cc.max_seq_len = 64;
  cc.slot_stride = 8192;
  cc.layer_stride = 8192;
  cc.pos_stride = 128;
  cc.head_stride = 64;
  cc.lookup_table = (const uint32_t *)fake;
  cc.cache_lengths = (const uint32_t *)fake;
  cc.n_seqs = 4;
  expect("bshd head_dim",
         qk_rope_bshd_continuous(fake, 2, 1, 4, 128, &cc, &freqs, 0, (const uint32_t *)fake,
                                 fake, NULL, NULL),
         ROPE_ERR_INVALID_ARG);
  /* GEMV: weight stored [k, n] is not built; workspace smaller than documented */
  expect("gemv transpose_b = 0",
         matmul_fused_partial_rmsnorm(fake, fake, 64, 8, 64, 0, fake, 1e-6f, 0.0f, fake, 8,
                                      NULL, ROPE_DTYPE_BF16, NULL, fake,
                                      ROPE_GEMV_WORKSPACE_BYTES(8), NULL),
         ROPE_ERR_UNSUPPORTED);
  expect("gemv workspace",
         matmul_fused_partial_rmsnorm(fake, fake, 64, 8, 64, 1, fake, 1e-6f, 0.0f, fake, 8,
                                      NULL, ROPE_DTYPE_BF16, NULL, fake, 16, NULL),
         ROPE_ERR_INVALID_ARG);
  /* the no-alloc store: empty work returns before it touches its scratch words */
  expect("noalloc empty",
         rope_split_store_paged_ragged_noalloc(fake, 512, ROPE_DTYPE_BF16, 0, 4,
                                               (const uint32_t *)fake, 2, &freqs, &kv, 1, fake,
                                               256, -1, NULL, NULL),
         ROPE_OK);
  /* launch overlap: an unknown mode is refused and the mode kept */
  expect("overlap default", rope_get_launch_overlap(), ROPE_OVERLAP_PDL);
  expect("overlap unknown", rope_set_launch_overlap(7), ROPE_ERR_INVALID_ARG);
  expect("overlap kept", rope_get_launch_overlap(), ROPE_OVERLAP_PDL);

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
