/* A C99 caller of the library's C ABI (no C++, no CUDA headers): plans a step, checks
 * the documented argument errors, and frees.  No device is touched, so it runs on a
 * machine without a GPU; it prints "ok" and returns 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "dion.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    printf("FAILED: %s (last error: %s)\n", what, dion_last_error());
    ++failures;
  }
}

int main(void) {
  dion_options o;
  expect(dion_default_options(&o) == DION_OK, "default options");
  expect(o.precision == DION_PREC_BF16 && o.orth_mode == DION_ORTH_AUTO, "defaults");

  dion_bucket_desc b[2];
  memset(b, 0, sizeof(b));
  b[0].count = 4; b[0].m = 256; b[0].n = 128; b[0].r = 32; b[0].scale = 0.f;
  b[1].count = 2; b[1].m = 512; b[1].n = 512; b[1].r = 64; b[1].scale = 0.f;
  dion_handle h = NULL;
  size_t ws = 0;
  expect(dion_init(b, 2, &o, &h, &ws) == DION_OK && h != NULL && ws > 0, "init");
  expect(dion_num_matrices(h) == 6, "matrix count");
  expect(dion_last_launch_count(h) == 0, "no launches before a step");

  b[1].r = 24; /* r % 16 != 0 */
  dion_handle bad = NULL;
  size_t ws2 = 0;
  expect(dion_init(b, 2, &o, &bad, &ws2) == DION_ERR_UNSUPPORTED_SHAPE && bad == NULL,
         "shape check");
  expect(strlen(dion_last_error()) > 0, "error message");

  dion_bucket_ptrs p[2];
  memset(p, 0, sizeof(p));
  expect(dion_step_batched(h, p, 2, 0.01f, NULL, ws, NULL, NULL) == DION_ERR_INVALID_ARG,
         "null workspace");
  expect(dion_step_batched(NULL, p, 2, 0.01f, NULL, ws, NULL, NULL) ==
             DION_ERR_NOT_INITIALIZED, "null handle");

  dion_vec_options vo;
  expect(dion_vec_default_options(DION_VEC_LION, &vo) == DION_OK && vo.rule == DION_VEC_LION,
         "vector defaults");
  vo.beta1 = 1.5f;
  dion_vec_tensor t;
  memset(&t, 0, sizeof(t));
  expect(dion_vec_step(&t, 1, &vo, NULL) == DION_ERR_INVALID_ARG, "vector option check");

  expect(strcmp(dion_status_string(DION_OK), "ok") == 0, "status string");
  expect(dion_free(h) == DION_OK, "free");
  expect(dion_free(NULL) == DION_OK, "free NULL");
  if (failures == 0) printf("ok\n");
  return failures ? 1 : 0;
}
