/* A plain C caller of libdspark.so: the header compiles as C99, and the
 * host-side paths (version, workspace sizes, status strings, argument errors
 * found before any launch) work without PyTorch and without a GPU. */
#include <stdio.h>
#include <string.h>

#include "dspark.h"

static int fails = 0;
#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      printf("FAIL line %d: %s\n", __LINE__, #c);                  \
      ++fails;                                                     \
    }                                                              \
  } while (0)

int main(void) {
  int32_t i32[8];
  float f32[8];
  unsigned char ws[512];
  uint32_t code = 0;
  int32_t first = 0;

  CHECK((dspark_version() >> 16) == 3);
  /* draft: status block + one (max, sum) pair per request and 256-entry chunk */
  CHECK(dspark_workspace_bytes(DSPARK_OP_DRAFT, 256, 5, 129280, 256, DSPARK_BF16) ==
        256 + (size_t)256 * 505 * 8);
  /* verify: status block, the draft's partials, per-chunk target-row statistics, a counter,
     the verification order */
  CHECK(dspark_workspace_bytes(DSPARK_OP_VERIFY, 256, 5, 129280, 256, DSPARK_BF16) ==
        256 + (size_t)256 * 505 * 8 + (size_t)256 * 6 * 127 * 8 + 256 + 1024);
  CHECK(dspark_workspace_bytes(DSPARK_OP_SCHEDULE, 1024, 8, 0, 0, 0) == 256);
  CHECK(dspark_workspace_bytes(DSPARK_OP_DRAFT, 4, 4, 1001, 16, DSPARK_F32) == 0); /* V % 8 */
  CHECK(dspark_workspace_bytes(DSPARK_OP_VERIFY, 4, 65, 1024, 16, DSPARK_F32) == 0); /* K > 64 */
  CHECK(dspark_workspace_bytes(7, 4, 4, 1024, 16, DSPARK_F32) == 0);

  CHECK(strcmp(dspark_status_string(DSPARK_OK), "ok") == 0);
  CHECK(strstr(dspark_status_string(DSPARK_ERR_WORKSPACE), "workspace") != NULL);

  /* missing pointers and impossible sizes are argument errors (nothing launched) */
  CHECK(dspark_draft_sample(NULL, NULL, NULL, NULL, i32, f32, 4, 4, 1024, 16, DSPARK_F32, 1, 0,
                            i32, NULL, f32, f32, NULL, ws, sizeof ws, NULL) ==
        DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_draft_sample_beside(NULL, NULL, NULL, NULL, NULL, i32, f32, 4, 4, 1024, 16,
                                   DSPARK_F32, 1, 0, i32, NULL, f32, f32, NULL, NULL, 20, ws,
                                   sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_draft_sample_beside(f32, f32, f32, NULL, NULL, i32, f32, 4, 4, 1024, 16,
                                   DSPARK_F32, 1, 0, i32, f32, f32, f32, NULL, NULL, -1, ws,
                                   sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG); /* free_sms < 0 */
  CHECK(dspark_draft_sample_beside(f32, f32, f32, f32, NULL, i32, f32, 4, 4, 1024, 16,
                                   DSPARK_F32, 1, 0, i32, f32, f32, f32, NULL, NULL, 2, ws,
                                   sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG); /* R without h */
  CHECK(dspark_prefix_schedule(NULL, f32, f32, 0.f, 4, 1, DSPARK_CUT_COST, 0.f, i32, f32, ws,
                               sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_prefix_schedule(f32, f32, f32, 0.f, 4, 65, DSPARK_CUT_COST, 0.f, i32, f32, ws,
                               sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_verify(NULL, NULL, i32, f32, NULL, NULL, f32, 4, 4, 1024, DSPARK_F32, 1, 0, i32,
                      i32, i32, ws, sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_verify_target_stats(NULL, NULL, f32, 4, 4, 1024, DSPARK_F32, ws, sizeof ws, NULL) ==
        DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_verify_from_stats(NULL, NULL, i32, f32, NULL, NULL, f32, 4, 4, 1024, DSPARK_F32, 1,
                                 0, i32, i32, i32, ws, sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_sts_fit(NULL, NULL, 10, 5, f32, NULL, NULL, NULL, ws, sizeof ws, NULL) ==
        DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_read_status(NULL, NULL, &code, &first) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_clear_status(NULL, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_selftest_waits(NULL, ws, sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_selftest_waits(i32, NULL, sizeof ws, NULL) == DSPARK_ERR_INVALID_ARG);
  CHECK(dspark_selftest_waits(i32, ws, 64, NULL) == DSPARK_ERR_INVALID_ARG);

  if (fails)
    printf("c abi: %d failures\n", fails);
  else
    printf("c abi: ok\n");
  return fails != 0;
}
