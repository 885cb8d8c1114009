/* A plain C client of libsolattn.so: it includes only include/solattn.h and
 * links the library, and exercises the calls that need no GPU (version,
 * status strings, buffer layout and scratch sizes, argument checks that
 * return before anything touches the device). Exit status 0 = all checks
 * passed; the first failing check is printed. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include "solattn.h"

#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                      \
    }                                                                \
  } while (0)

int main(void) {
  CHECK(solattn_version() >= 10000);
  CHECK(solattn_strerror(SOLATTN_OK) != NULL);
  CHECK(solattn_strerror(SOLATTN_ERR_TIMEOUT) != NULL);

  /* pooled statistics of the 75,600-token, 40-head, d = 128 problem */
  size_t bytes = 0;
  CHECK(solattn_pooled_layout(1, 40, 75600, 128, NULL, NULL, &bytes) == SOLATTN_OK);
  CHECK(bytes > (size_t)40 * 1182 * 128 * 4 * 3);
  solattn_pooled_t p;
  CHECK(solattn_pooled_layout(1, 40, 75600, 128, (void*)(uintptr_t)0x10000000, &p, NULL) == SOLATTN_OK);
  CHECK((uintptr_t)p.qbar == 0x10000000 && ((uintptr_t)p.kcov & 255u) == 0);
  CHECK(solattn_pooled_layout(1, 40, 75600, 80, NULL, NULL, &bytes) == SOLATTN_ERR_UNSUPPORTED);

  /* host-path scratch: workspace + two chunk buffers */
  size_t scratch = 0;
  CHECK(solattn_host_scratch_bytes(1, 40, 75600, 128, 0, &scratch) == SOLATTN_OK);
  CHECK(scratch > SOLATTN_WORKSPACE_BYTES);
  CHECK(solattn_host_scratch_bytes(1, 40, 75600, 128, -1, &scratch) == SOLATTN_ERR_ARG);

  /* argument errors come back before any device work */
  char buf[64];
  void* x = buf;
  CHECK(solattn_forward(NULL, x, x, 1, 2, 256, 64, &p, 0.5f, x, NULL, NULL, x, 256, NULL) == SOLATTN_ERR_ARG);
  CHECK(solattn_forward(x, x, x, 1, 2, 0, 64, &p, 0.5f, x, NULL, NULL, x, 256, NULL) == SOLATTN_ERR_ARG);
  CHECK(solattn_forward(x, x, x, 1, 2, 256, 96, &p, 0.5f, x, NULL, NULL, x, 256, NULL) == SOLATTN_ERR_UNSUPPORTED);
  CHECK(solattn_forward(x, x, x, 1, 2, SOLATTN_MAX_TOKENS + 1, 64, &p, 0.5f, x, NULL, NULL, x, 256, NULL) ==
        SOLATTN_ERR_UNSUPPORTED);
  CHECK(solattn_dense(x, x, x, 1, 2, 256, 64, NULL, NULL, x, 256, NULL) == SOLATTN_ERR_ARG);
  CHECK(solattn_forward_host(x, x, x, 1, 2, 256, 64, NAN, x, NULL, NULL, 0, x, 1u << 30, NULL) == SOLATTN_ERR_ARG);
  CHECK(solattn_forward_host(x, x, x, 1, 2, 256, 64, 0.5f, x, NULL, NULL, 0, NULL, 0, NULL) ==
        SOLATTN_ERR_WORKSPACE);
  printf("c client ok\n");
  return 0;
}
