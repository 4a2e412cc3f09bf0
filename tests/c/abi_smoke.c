/* Plain C99 user of the librlscan C ABI (no GPU needed): includes the public
 * header, links the library, and exercises the calls that never touch a
 * device -- version, status strings, plans, options and synchronous argument
 * checks.  Exit status 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "rlscan.h"

static int fails = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++fails;                                                   \
    }                                                            \
  } while (0)

int main(void) {
  CHECK(rlscan_abi_version() == RLSCAN_ABI_VERSION);
  CHECK(strcmp(rlscan_status_string(RLSCAN_ERR_OVERLAP), "RLSCAN_ERR_OVERLAP") == 0);

  rlscan_plan_info info;
  CHECK(rlscan_query_plan(RLSCAN_EST_GAE, 4096, 2048, 1, &info) == RLSCAN_OK);
  CHECK(info.lookback == 0 && info.launches == 1 && info.chunk_steps % 2048 == 0);
  CHECK(rlscan_query_plan(RLSCAN_EST_VTRACE, 256, 16384, 1, &info) == RLSCAN_OK);
  CHECK(info.lookback == 1 && info.workspace_bytes >= 16 * info.chunks);
  CHECK(rlscan_query_plan_tm(RLSCAN_EST_GAE, 4096, 2048, &info) == RLSCAN_OK);
  CHECK(info.lookback == 1 && info.block_threads == 256);
  CHECK(rlscan_query_plan(RLSCAN_EST_GAE, 4, 8, 1, NULL) == RLSCAN_ERR_INVALID_ARG);

  CHECK(rlscan_set_option(RLSCAN_OPT_FORCE_BLOCK, 100) == RLSCAN_ERR_INVALID_ARG);
  CHECK(rlscan_set_option(RLSCAN_OPT_FORCE_BLOCK, 192) == RLSCAN_OK);
  CHECK(rlscan_get_option(RLSCAN_OPT_FORCE_BLOCK) == 192);
  CHECK(rlscan_set_option(RLSCAN_OPT_FORCE_BLOCK, 0) == RLSCAN_OK);

  /* argument checks happen before any device call: fake, never-dereferenced addresses */
  const float *r = (const float *)(uintptr_t)0x10000000u, *v = (const float *)(uintptr_t)0x10010000u;
  const float *b = (const float *)(uintptr_t)0x10020000u;
  float *adv = (float *)(uintptr_t)0x10030000u;
  CHECK(rlscan_gae(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 5, 0.99f, 0.95f, NULL) == RLSCAN_OK);
  CHECK(rlscan_gae(r, v, b, NULL, NULL, NULL, adv, NULL, -1, 5, 0.99f, 0.95f, NULL) == RLSCAN_ERR_INVALID_ARG);
  CHECK(rlscan_gae(r, NULL, b, NULL, NULL, NULL, adv, NULL, 4, 5, 0.99f, 0.95f, NULL) == RLSCAN_ERR_INVALID_ARG);
  CHECK(rlscan_gae(r, v, b, NULL, NULL, NULL, (float *)v, NULL, 4, 5, 0.99f, 0.95f, NULL) == RLSCAN_ERR_OVERLAP);
  CHECK(rlscan_gae_tm(r, v, b, NULL, NULL, NULL, (float *)r, NULL, 4, 5, 0.99f, 0.95f, NULL) == RLSCAN_ERR_OVERLAP);
  CHECK(rlscan_affine_scan(r, v, NULL, NULL, adv, 4, 8, 2, NULL) == RLSCAN_ERR_INVALID_ARG);

  if (fails == 0) printf("abi_smoke ok\n");
  return fails == 0 ? 0 : 1;
}
