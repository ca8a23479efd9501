/* The C ABI used from plain C (no Python, no CUDA headers): compiled by the CPU test
 * suite with gcc against include/kv4.h and linked to libkv4.so. It calls only entry
 * points that answer on the host (version, status strings, workspace sizes, argument
 * checks that reject before anything is launched), so it runs without a GPU.
 * Prints "ok" and exits 0 when every check holds, else names the first failure. */
#include <stdio.h>
#include <string.h>

#include "kv4.h"

#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      printf("failed: %s (line %d)\n", #cond, __LINE__);     \
      return 1;                                              \
    }                                                        \
  } while (0)

static kv4_config config(int32_t hq, int32_t hkv, int32_t s, int32_t r, int32_t chunk) {
  kv4_config c;
  memset(&c, 0, sizeof c);
  c.num_q_heads = hq;
  c.num_kv_heads = hkv;
  c.head_dim = 128;
  c.page_size = 16;
  c.group_size = 32;
  c.num_sinks = s;
  c.num_recent = r;
  c.chunk_pages = chunk;
  c.demotion = 0;
  c.prefix_mode = KV4_PREFIX_OFF;
  return c;
}

int main(void) {
  CHECK(kv4_version() >= 500);
  CHECK(strcmp(kv4_status_string(KV4_OK), "ok") == 0);
  CHECK(strstr(kv4_status_string(KV4_ERR_PROTECTED_TOO_LARGE), "144") != NULL);

  /* workspace sizes: positive, growing with the batch, 0 for a rejected config */
  kv4_config c = config(32, 8, 16, 128, 32);
  size_t small = kv4_workspace_size(&c, 64, 2048);
  size_t large = kv4_workspace_size(&c, 1024, 16384);
  CHECK(small > 0 && large > small);
  kv4_config too_wide = config(32, 8, 100, 100, 0);
  CHECK(kv4_workspace_size(&too_wide, 64, 2048) == 0);

  /* chunk lengths: the configured one, an automatic one in 8..64, -1 when rejected */
  CHECK(kv4_chunk_pages_for(&c, 64, 2048) == 32);
  kv4_config autoc = config(32, 8, 16, 128, 0);
  int32_t ch = kv4_chunk_pages_for(&autoc, 64, 2048);
  CHECK(ch >= 8 && ch <= 64);
  CHECK(kv4_chunk_pages_for(&autoc, 1024, 16384) == 64);
  CHECK(kv4_chunk_pages_for(&too_wide, 64, 2048) == -1);

  /* argument checks answer before any launch */
  kv4_int4_pool pool;
  kv4_int8_side side;
  kv4_batch batch;
  memset(&pool, 0, sizeof pool);
  memset(&side, 0, sizeof side);
  memset(&batch, 0, sizeof batch);
  CHECK(kv4_decode_attention(NULL, &pool, &side, &batch, NULL, NULL, NULL, NULL, NULL, 0,
                             NULL, NULL) == KV4_ERR_INVALID_ARG);
  CHECK(kv4_decode_attention(&too_wide, &pool, &side, &batch, NULL, NULL, NULL, NULL, NULL,
                             0, NULL, NULL) == KV4_ERR_PROTECTED_TOO_LARGE);
  kv4_config bad_dim = config(32, 8, 16, 128, 0);
  bad_dim.head_dim = 64;
  CHECK(kv4_quantize_append(&bad_dim, &pool, &side, &batch, NULL, NULL, NULL, 0, NULL,
                            NULL) == KV4_ERR_UNSUPPORTED_SHAPE);
  kv4_config bad_gqa = config(32, 3, 16, 128, 0);
  CHECK(kv4_decode_step(&bad_gqa, &pool, &side, &batch, NULL, NULL, NULL, NULL, NULL, NULL,
                        NULL, 0, NULL, NULL) == KV4_ERR_UNSUPPORTED_SHAPE);
  CHECK(kv4_regional_merge(NULL, NULL, 4, 4, 64, NULL, NULL, NULL, NULL) ==
        KV4_ERR_UNSUPPORTED_SHAPE);
  CHECK(kv4_regional_merge(NULL, NULL, 0, 4, 128, NULL, NULL, NULL, NULL) == KV4_OK);
  printf("ok\n");
  return 0;
}
