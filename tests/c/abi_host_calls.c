/* Plain C99 user of the C ABI: compiles against include/pagedattn.h alone and
 * calls the entry points that need no GPU (planning, layouts, statuses and
 * host-side argument checks). Exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "pagedattn.h"

static int failures = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                \
    }                                                            \
  } while (0)

int main(void) {
  pa_kv_pool_t pool;
  size_t off[7];
  size_t n, n1;
  pa_step_graph_t *graph = (pa_step_graph_t *)1;

  CHECK(pa_abi_version() == PA_ABI_VERSION);
  CHECK(strcmp(pa_status_str(PA_OK), "ok") == 0);
  CHECK(pa_derr_status(0) == PA_OK);
  CHECK(pa_derr_status(PA_DERR_BAD_PAGE | PA_DERR_TIMEOUT) == PA_ERR_TIMEOUT);
  CHECK(pa_derr_status(PA_DERR_BAD_POS) == PA_ERR_BAD_TABLE);

  /* the planner's rule for a B200 (148 SMs x 3 decode CTAs) */
  CHECK(pa_decode_plan_splits(32 * 8, 256, 32, 148, 3, 0) == 1);
  CHECK(pa_decode_plan_splits(8 * 8, 256, 32, 148, 3, 0) == 4);
  CHECK(pa_decode_plan_splits(64 * 8, 256, 16, 148, 3, 0) == 4);
  /* 128 requests x (2000-token prefix + up to 512 own tokens): 3 splits of 11 tiles */
  CHECK(pa_prefix_plan_splits(32, 32, 148, 3, 128.0 * 8 * 2 * 256 * 512 / 2) == 11);
  CHECK(pa_prefix_plan_splits(0, 32, 148, 3, 0.0) <= 0);

  memset(&pool, 0, sizeof pool);
  pool.num_pages = 16;
  pool.page_size = 32;
  pool.num_kv_heads = 8;
  pool.head_dim = 128;
  pool.dtype = PA_KV_BF16;
  pool.k_pool = (void *)0x10000;
  pool.v_pool = (void *)0x20000;

  n = pa_step_packet_layout(&pool, 32, 64, 256, 32, off);
  CHECK(n == 688896);
  CHECK(off[0] == 0 && off[1] == 524288 && off[6] == 688640);
  n1 = pa_step_packet_layout(&pool, 32, 64, 256, PA_STEP_NEWEST_PER_SEQ, off);
  CHECK(n1 > 0 && off[3] == off[4] && off[4] == off[5]);

  /* host-side checks return before any device work */
  CHECK(pa_decode(NULL, NULL, 1, 1, NULL, 1, NULL, 1.f, NULL, NULL, 0, 0, NULL, NULL) ==
        PA_ERR_INVALID_ARG);
  CHECK(strlen(pa_last_error()) > 0);
  CHECK(pa_step_graph_create(NULL, NULL, NULL, 0, 1, 1, 1, 1, 1.f, NULL, NULL, NULL, 0, 0,
                             NULL, &graph) == PA_ERR_INVALID_ARG);
  CHECK(graph == NULL);
  pa_step_graph_destroy(NULL);

  if (failures == 0) printf("c abi host calls: ok\n");
  return failures == 0 ? 0 : 1;
}
