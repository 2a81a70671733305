/* The C ABI consumed from plain C99: include/loki.h compiles as C, and the
 * library's host-side validation answers through it without a GPU (every call
 * below fails validation before any CUDA call, or only reports the version). */
#include <stdio.h>
#include <string.h>

#include "loki.h"

static int fails = 0;
#define EXPECT(cond)                                              \
  do {                                                            \
    if (!(cond)) {                                                \
      fprintf(stderr, "line %d: %s failed\n", __LINE__, #cond);  \
      ++fails;                                                    \
    }                                                             \
  } while (0)

int main(void) {
  loki_cache c;
  loki_paged_cache pc;
  size_t bytes = 0;
  void *fake = (void *)(size_t)(1u << 20);

  EXPECT(loki_version() == LOKI_VERSION);
  EXPECT(strstr(loki_status_string(LOKI_ERR_INVALID_ARG), "INVALID_ARG") != NULL);

  memset(&c, 0, sizeof c);
  c.dtype = LOKI_BF16;
  c.batch = 1;
  c.n_kv_heads = 2;
  c.head_dim = 128;
  c.capacity = 64;
  c.k_hat = fake;
  c.v = fake;
  EXPECT(loki_decode_workspace_size(&c, 10, 2, &bytes) == LOKI_OK && bytes > 0);
  EXPECT(loki_decode_workspace_size(&c, 65, 2, &bytes) == LOKI_ERR_INVALID_ARG);
  c.head_dim = 96;
  EXPECT(loki_decode_workspace_size(&c, 10, 2, &bytes) == LOKI_ERR_UNSUPPORTED);
  c.head_dim = 128;
  c.k_lr = fake;
  c.d_lr = 12; /* 24-byte plane rows */
  EXPECT(loki_decode_workspace_size(&c, 10, 2, &bytes) == LOKI_ERR_INVALID_ARG);
  EXPECT(strstr(loki_last_error(), "plane") != NULL);
  c.d_lr = 32;
  EXPECT(loki_decode_workspace_size(&c, 10, 2, &bytes) == LOKI_OK);
  EXPECT(loki_append(&c, 60, 5, fake, fake, (const float *)fake, NULL) == LOKI_ERR_INVALID_ARG);
  EXPECT(loki_decode_attention(&c, 10, 2, NULL, (const float *)fake, 8, 4, 0.f, (float *)fake,
                               (int32_t *)fake, fake, (size_t)1 << 40, NULL) == LOKI_ERR_INVALID_ARG);

  memset(&pc, 0, sizeof pc);
  pc.dtype = LOKI_BF16;
  pc.n_kv_heads = 2;
  pc.head_dim = 128;
  pc.page_size = 24; /* not a power of two */
  pc.num_pages = 10;
  pc.k_hat = fake;
  pc.v = fake;
  {
    loki_seq_table q;
    memset(&q, 0, sizeof q);
    q.batch = 2;
    q.pages_per_seq = 4;
    q.max_seq_len = 50;
    q.block_table = (const int32_t *)fake;
    EXPECT(loki_paged_decode_workspace_size(&pc, &q, 4, &bytes) == LOKI_ERR_INVALID_ARG);
    pc.page_size = 16;
    EXPECT(loki_paged_decode_workspace_size(&pc, &q, 4, &bytes) == LOKI_OK);
  }
  if (fails == 0) printf("c abi ok\n");
  return fails == 0 ? 0 : 1;
}
