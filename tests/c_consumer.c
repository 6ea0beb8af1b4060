/* A plain C99 user of libsignmuon.so: plans the nanoGPT-124M weight shapes
 * (12 x {2304x768, 768x768, 3072x768, 768x3072}) for 8 workers and checks the
 * host-only calls (no GPU needed).  Exit status 0 on success; the failing
 * check's number otherwise.  Built and run by tests/test_c_consumer.py. */
#include <stdio.h>
#include <string.h>

#include "signmuon.h"

int main(void) {
  int64_t shapes[96];
  const int64_t layer[8] = {2304, 768, 768, 768, 3072, 768, 768, 3072};
  int64_t info[6];
  int i, rc;
  for (i = 0; i < 48; ++i) {
    shapes[2 * i] = layer[2 * (i % 4)];
    shapes[2 * i + 1] = layer[2 * (i % 4) + 1];
  }
  rc = signmuon_plan(shapes, 48, 8, 5, SIGNMUON_SCALE_SPECTRAL, 2, SIGNMUON_POST_POLAR, info, 6);
  if (rc != SIGNMUON_OK) return 1;
  if (info[0] != 84934656LL || info[1] != 10616832LL || info[3] != 4 || info[4] != 8 || info[5] != 48) return 2;
  if (info[2] <= 0) return 3;
  /* invalid arguments are reported, with text, before any CUDA call */
  rc = signmuon_plan(shapes, 48, 0, 5, SIGNMUON_SCALE_FRO, 1, 0, info, 6);
  if (rc != SIGNMUON_E_INVALID || strlen(signmuon_last_error(NULL)) == 0) return 4;
  rc = signmuon_plan(shapes, 48, 200, 5, SIGNMUON_SCALE_FRO, 1, SIGNMUON_ACC_INT8, info, 6);
  if (rc != SIGNMUON_E_OVERFLOW) return 5;
  rc = signmuon_plan(shapes, 48, 8, 5, SIGNMUON_SCALE_FRO, 1, SIGNMUON_NORMALIZED_SIGN | SIGNMUON_POST_POLAR,
                     info, 6);
  if (rc != SIGNMUON_E_INVALID) return 6;
  if (strcmp(signmuon_status_string(SIGNMUON_OK), "ok") != 0) return 7;
  if (signmuon_kernel_launches() != 0) return 8;
  printf("c consumer ok: d=%lld packed=%lld device_bytes=%lld\n", (long long)info[0], (long long)info[1],
         (long long)info[2]);
  return 0;
}
