/* A plain C99 consumer of include/dmu.h: compiles with -std=c99 -pedantic
 * -Werror, links against libdmu.so, and checks the host-side argument
 * validation (no call here reaches the GPU). Exit status 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "dmu.h"

static int failures = 0;

#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++failures;                                                    \
    }                                                                \
  } while (0)

int main(void) {
  dmu_plan plan = NULL;
  dmu_shape shape;
  float mix[4] = {0.5f, 0.5f, 0.5f, 0.5f};
  void* fake[2];
  void* other[2];
  float* fakef[2];
  const float* fakecf[2];
  float* outf[2];

  CHECK(dmu_version() == 100);

  /* plan creation: argument errors come back before any device work */
  CHECK(dmu_plan_create(NULL, 1, DMU_BF16, DMU_PREC_AUTO, 0, &plan) == DMU_ERR_INVALID_ARG);
  CHECK(strlen(dmu_last_error()) > 0);
  shape.rows = 0;
  shape.cols = 4;
  CHECK(dmu_plan_create(&shape, 1, DMU_BF16, DMU_PREC_AUTO, 0, &plan) == DMU_ERR_INVALID_ARG);
  shape.rows = 4;
  CHECK(dmu_plan_create(&shape, 0, DMU_BF16, DMU_PREC_AUTO, 0, &plan) == DMU_ERR_INVALID_ARG);
  CHECK(dmu_plan_create(&shape, 1, (dmu_dtype)7, DMU_PREC_AUTO, 0, &plan) == DMU_ERR_INVALID_ARG);

  /* calls on a NULL plan */
  CHECK(dmu_workspace_bytes(NULL) == 0);
  CHECK(dmu_get_schedule(NULL) == -1);
  CHECK(dmu_set_workspace(NULL, NULL, 0) == DMU_ERR_INVALID_ARG);
  CHECK(dmu_momentum_normalize(NULL, NULL, NULL, 0.9f, 1.0f, 1e-7f, NULL) == DMU_ERR_INVALID_ARG);
  CHECK(dmu_apply_update(NULL, NULL, 0.02f, NULL, NULL) == DMU_ERR_INVALID_ARG);
  dmu_plan_destroy(NULL);

  /* DeMuon entry points: fake, aligned, never dereferenced device pointers */
  fake[0] = (void*)(uintptr_t)0x1000;
  fake[1] = (void*)(uintptr_t)0x2000;
  other[0] = (void*)(uintptr_t)0x3000;
  other[1] = (void*)(uintptr_t)0x4000;
  fakef[0] = (float*)(uintptr_t)0x5000;
  fakef[1] = (float*)(uintptr_t)0x6000;
  fakecf[0] = (const float*)(uintptr_t)0x7000;
  fakecf[1] = (const float*)(uintptr_t)0x8000;
  outf[0] = (float*)(uintptr_t)0x9000;
  outf[1] = (float*)(uintptr_t)0xa000;
  CHECK(dmu_demuon_track(0, 16, mix, 0.1f, (const void* const*)fake, fakef, fakecf, outf, other, NULL) ==
        DMU_ERR_INVALID_ARG);
  CHECK(dmu_demuon_track(DMU_DEMUON_MAX_AGENTS + 1, 16, mix, 0.1f, (const void* const*)fake, fakef, fakecf,
                         outf, other, NULL) == DMU_ERR_INVALID_ARG);
  CHECK(dmu_demuon_track(2, 16, mix, 2.0f, (const void* const*)fake, fakef, fakecf, outf, other, NULL) ==
        DMU_ERR_INVALID_ARG);
  CHECK(dmu_demuon_track(2, 0, mix, 0.1f, (const void* const*)fake, fakef, fakecf, outf, other, NULL) ==
        DMU_OK);
  /* Never call either entry point with valid arguments and numel > 0 here:
   * that would launch a kernel on the fake pointers. */
  CHECK(dmu_demuon_mix(2, 16, NULL, 0.1f, fakecf, fakecf, outf, NULL) == DMU_ERR_INVALID_ARG);
  CHECK(dmu_demuon_mix(2, 0, mix, 0.1f, fakecf, fakecf, outf, NULL) == DMU_OK);

  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("abi_check ok\n");
  return 0;
}
