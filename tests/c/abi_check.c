/* Plain C99 client of liblhcal.so: compiles against include/lhcal.h with gcc (no CUDA or C++
 * headers), links the shared library, and exercises the calls that need no GPU: the version,
 * the host-only workspace queries and argument validation with its error strings. Exits 0 on
 * success; prints the first failed check otherwise. */
#include <stdio.h>
#include <string.h>

#include "lhcal.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  size_t bytes = 0;
  CHECK(lhcal_version() == 100);
  CHECK(LHCAL_N_CANDIDATES == 126 && LHCAL_BLOCK == 16 && LHCAL_MAX_MULTIPLIERS == 1024);

  /* Host-only workspace queries. */
  CHECK(lhcal_accumulate_workspace(LHCAL_FULL, LHCAL_BF16, 16384, 2048, 1, &bytes) == LHCAL_OK);
  CHECK(bytes > 0 && bytes % (128 * 4 * 256) == 0);
  CHECK(lhcal_accumulate_workspace(LHCAL_FULL, LHCAL_BF16, 16384, 4096, 1, &bytes) == LHCAL_OK && bytes == 0);
  CHECK(lhcal_accumulate_act_quant_workspace(LHCAL_BF16, 32768, 4096, 1, &bytes) == LHCAL_OK && bytes > 0);
  CHECK(lhcal_accumulate_workspace(LHCAL_FULL, LHCAL_BF16, 100, 24, 1, &bytes) == LHCAL_ERR_INVALID_ARG);
  CHECK(strstr(lhcal_last_error_string(), "multiple of 16") != NULL);
  CHECK(lhcal_accumulate_workspace((lhcal_mode)7, LHCAL_BF16, 100, 32, 1, &bytes) == LHCAL_ERR_UNSUPPORTED);

  /* Validation before any device access. */
  CHECK(lhcal_accumulate(LHCAL_FULL, LHCAL_BF16, NULL, NULL, 10, 33, 33, 1, NULL, NULL, LHCAL_ACCUM_OVERWRITE,
                         NULL, NULL, NULL, 0, NULL) == LHCAL_ERR_INVALID_ARG);
  CHECK(lhcal_act_fake_quant(LHCAL_F32, NULL, 4, 32, 32, NULL, NULL, 32, NULL) == LHCAL_ERR_UNSUPPORTED);
  CHECK(lhcal_accumulate_act_quant(LHCAL_BF16, NULL, 4, 32, 32, 1, NULL, NULL, NULL, 0, NULL, NULL, NULL, 0,
                                   NULL) == LHCAL_ERR_INVALID_ARG);
  CHECK(lhcal_scale_sweep(LHCAL_MSE, LHCAL_BF16, NULL, 1, 4, 32, (const float*)256, NULL, NULL, NULL, NULL, NULL,
                          NULL) == LHCAL_ERR_INVALID_ARG);
  CHECK(lhcal_global_scale_ex(LHCAL_BF16, NULL, 1, 4, 32, 500.0f, NULL, NULL) == LHCAL_ERR_INVALID_ARG);
  CHECK(lhcal_multiplier_search(LHCAL_FULL, LHCAL_BF16, NULL, 1, 4, 32, NULL, NULL, NULL, NULL, 0, NULL, NULL, NULL,
                                NULL) == LHCAL_ERR_INVALID_ARG);
  CHECK(lhcal_apply_scales(LHCAL_BF16, NULL, 1, 4, 33, NULL, NULL, NULL, NULL, NULL, NULL) == LHCAL_ERR_INVALID_ARG);
  CHECK(lhcal_finalize(LHCAL_MSE, 1, 32, NULL, NULL, NULL, NULL) == LHCAL_ERR_UNSUPPORTED);
  CHECK(lhcal_count_tokens(2, 5, NULL, 0, NULL, NULL) == LHCAL_ERR_INVALID_ARG);
  CHECK(lhcal_launch_count(1) >= 0);

  if (failures == 0) printf("abi ok\n");
  return failures == 0 ? 0 : 1;
}
