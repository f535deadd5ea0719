/* A plain C99 consumer of libcvq: the header must compile as C (no C++ or torch types),
 * the library must link and load, and the host-side calls must behave as cvq.h states.
 * Every call here either needs no device or carries an invalid argument, so nothing is
 * launched and no GPU is needed. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "cvq.h"

#define CHECK(cond)                                                          \
  do {                                                                       \
    if (!(cond)) {                                                           \
      fprintf(stderr, "FAIL %s:%d: %s\n", __FILE__, __LINE__, #cond);        \
      return 1;                                                              \
    }                                                                        \
  } while (0)

static cvq_shape layer(int32_t R, int32_t t_cap) {
  cvq_shape s;
  memset(&s, 0, sizeof s);
  s.batch = 1;
  s.n_q_heads = 32;
  s.n_kv_heads = 8;
  s.head_dim = CVQ_HEAD_DIM;
  s.R = R;
  s.t_cap = t_cap;
  s.rope_base = 500000.0f;
  s.group_dim = 8;
  return s;
}

int main(void) {
  /* an aligned, non-null address that is never dereferenced */
  float* const fake = (float*)(uintptr_t)0x10000;
  const cvq_shape s = layer(2, 1024);
  cvq_shape bad = s;

  CHECK(cvq_abi_version() == CVQ_ABI_VERSION);
  CHECK(strncmp(cvq_status_str(CVQ_OK), "CVQ_OK", 6) == 0);
  CHECK(strncmp(cvq_status_str(CVQ_ERR_ALIGN), "CVQ_ERR_ALIGN", 13) == 0);

  /* sizes: P table [B, Hq, 16, R, 256, 4, 2] fp32; partials 130 floats per (b, hq, split) */
  CHECK(cvq_ptable_bytes(&s) == (size_t)32 * 16 * 2 * 256 * 8 * 4);
  CHECK(cvq_partials_bytes(&s, 5) == (size_t)32 * 5 * 130 * 4);
  CHECK(cvq_split_tokens(&s, 4) == 256);
  CHECK(cvq_attend_workspace_bytes(&s, 5) >= cvq_partials_bytes(&s, 5));

  /* argument errors come back as a status, before any launch */
  CHECK(cvq_combine(&s, 0, fake, fake, fake, fake, fake, NULL) == CVQ_ERR_WORKSPACE);
  CHECK(cvq_combine(NULL, 2, fake, fake, fake, fake, fake, NULL) == CVQ_ERR_NULL);
  CHECK(cvq_attend(&s, NULL, CVQ_F32, fake, 0, (const uint8_t*)fake, (const uint8_t*)fake,
                   (const int32_t*)fake, fake, 0, 4, fake, fake, fake, NULL) == CVQ_ERR_NULL);
  bad.head_dim = 64;
  CHECK(cvq_ptable_bytes(&bad) == 0);
  CHECK(cvq_attend(&bad, fake, CVQ_F32, fake, 0, (const uint8_t*)fake, (const uint8_t*)fake,
                   (const int32_t*)fake, fake, 0, 4, fake, fake, fake, NULL) == CVQ_ERR_UNSUPPORTED);
  bad = s;
  bad.R = 3;
  CHECK(cvq_attend(&bad, fake, CVQ_F32, fake, 0, (const uint8_t*)fake, (const uint8_t*)fake,
                   (const int32_t*)fake, fake, 0, 4, fake, fake, fake, NULL) == CVQ_ERR_UNSUPPORTED);
  CHECK(cvq_fault_status(NULL, 0) == CVQ_ERR_NULL);

  printf("c abi ok\n");
  return 0;
}
