/* A plain C caller of the library: compiled with gcc against include/pa_attn.h
 * and linked to libpa_attn.so.  It checks the status helpers and that argument
 * errors come back with the documented codes before any CUDA work, so it runs
 * on a machine without a GPU.  Exit status 0 = every check passed. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pa_attn.h"

static int failures = 0;
#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                    \
    }                                                                \
  } while (0)

int main(void) {
  /* 16-byte aligned fake device addresses: never dereferenced, because every
   * call below is refused by a host-side check first. */
  const uintptr_t a = (uintptr_t)1 << 20, mb = (uintptr_t)1 << 24;
  void* q = (void*)a;
  void* k = (void*)(a + mb);
  void* v = (void*)(a + 2 * mb);
  void* o = (void*)(a + 3 * mb);
  float* lse = (float*)(a + 4 * mb);

  CHECK(pa_version() == 200);
  CHECK(strcmp(pa_status_string(PA_OK), "PA_OK") == 0);
  CHECK(strncmp(pa_status_string(PA_ERR_TIMEOUT), "PA_ERR_", 7) == 0);
  CHECK(strncmp(pa_status_string(PA_ERR_BAD_INPUT), "PA_ERR_", 7) == 0);

  CHECK(pa_attn_fwd(NULL, k, v, o, lse, 1, 1, 8, 8, 128, 0.125f, NULL) == PA_ERR_INVALID_ARG);
  CHECK(strlen(pa_last_error()) > 0);
  CHECK(pa_attn_fwd(q, k, v, o, lse, 1, 1, 8, 8, 96, 0.125f, NULL) == PA_ERR_UNSUPPORTED);
  CHECK(pa_attn_fwd((void*)(a + 8), k, v, o, lse, 1, 1, 8, 8, 128, 0.125f, NULL) == PA_ERR_MISALIGNED);
  CHECK(pa_attn_fwd(q, k, v, o, lse, 1, 1, 0, 8, 128, 0.125f, NULL) == PA_OK); /* empty query: no-op */

  const void* ks[2] = {k, (const void*)(a + mb + 4096)};
  const void* vs[2] = {v, (const void*)(a + 2 * mb + 4096)};
  const int nk[2] = {8, 0};
  CHECK(pa_attn_fwd_chunks(q, ks, vs, nk, 2, o, lse, 1, 1, 8, 128, 0.125f, NULL) == PA_ERR_INVALID_ARG);
  CHECK(pa_attn_fwd_chunks(q, ks, vs, nk, 9, o, lse, 1, 1, 8, 128, 0.125f, NULL) == PA_ERR_INVALID_ARG);

  CHECK(pa_attn_merge(o, lse, 0, (void*)(a + 6 * mb), (float*)(a + 7 * mb), 1, 1, 8, 64, NULL) ==
        PA_ERR_INVALID_ARG);
  CHECK(pa_attn_merge(o, lse, 2, (void*)(a + 6 * mb), (float*)(a + 7 * mb), 1, 1, 8, 32, NULL) ==
        PA_ERR_UNSUPPORTED);

  CHECK(pa_attn_fwd_fp8(q, k, v, 0.0f, 1.0f, 1.0f, o, lse, 1, 1, 8, 8, 128, 0.125f, NULL) == PA_ERR_INVALID_ARG);
  CHECK(pa_attn_fwd_fp8(q, k, v, 1.0f, 1.0f, 1.0f, o, lse, 1, 1, 8, 8, 64, 0.125f, NULL) == PA_ERR_UNSUPPORTED);
  CHECK(pa_quantize_e4m3(q, 0, o, lse, NULL) == PA_ERR_INVALID_ARG);
  CHECK(pa_selftest_timeout(0, NULL) == PA_ERR_INVALID_ARG);
  CHECK(pa_set_wait_limit_ms(0) == PA_ERR_INVALID_ARG);

  /* accumulate: the final fold needs o, the others must not get one */
  float* oacc = (float*)(a + 5 * mb);
  CHECK(pa_attn_fwd_accum(q, k, v, oacc, lse, NULL, 1, 1, 8, 8, 128, 0.125f, PA_ACCUM_FINAL, NULL) ==
        PA_ERR_INVALID_ARG);
  CHECK(pa_attn_fwd_accum(q, k, v, oacc, lse, o, 1, 1, 8, 8, 128, 0.125f, PA_ACCUM_FIRST, NULL) ==
        PA_ERR_INVALID_ARG);
  CHECK(pa_attn_fwd_accum(q, k, v, oacc, lse, NULL, 1, 1, 0, 8, 128, 0.125f, 0, NULL) == PA_OK);

  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("C ABI checks passed\n");
  return 0;
}
