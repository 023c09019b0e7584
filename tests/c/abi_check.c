/*
 * Host-only use of libqlora from plain C: the header compiles as C11 (and
 * as C++), the library links, and the calls that need no GPU behave.
 * Built and run by tests/test_c_abi.py; prints "ok" and exits 0 on success.
 */
#include <stdio.h>
#include <string.h>

#include "qlora.h"

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                                  \
    }                                                            \
  } while (0)

int main(void) {
  float c[16];
  CHECK(qlora_nf4_codebook(c) == QLORA_OK);
  CHECK(c[0] == -1.0f && c[7] == 0.0f && c[15] == 1.0f);
  for (int k = 0; k < 15; ++k) CHECK(c[k] < c[k + 1]);
  CHECK(qlora_nf4_codebook(NULL) == QLORA_ERR_INVALID_ARG);

  /* 256 x 256 at B = 64, C = 256: 32768 code bytes + 1024 scale codes + 4 t + mu */
  CHECK(qlora_nf4_payload_bytes(65536, 64, 256) == 32768 + 1024 + 4 * 4 + 4);
  CHECK(qlora_nf4_payload_bytes(-1, 64, 256) == 0);
  CHECK(qlora_quantize_nf4_workspace_bytes(65536, 64, 256) >= 256);

  for (int s = 0; s <= QLORA_ERR_WORKSPACE; ++s) CHECK(qlora_status_string((qlora_status)s) != NULL);
  CHECK(strcmp(qlora_status_string(QLORA_OK), "ok") == 0);

  qlora_weight w;
  memset(&w, 0, sizeof w);
  w.fmt = QLORA_FMT_NF4_DQ;
  w.O = 2048;
  w.I = 1024;
  w.block = 64;
  w.group = 256;
  w.bits = 4;
  size_t fwd = qlora_linear_workspace_bytes(&w, 4096, 8, QLORA_OP_FWD, QLORA_COMPUTE_BF16);
  size_t bwd = qlora_linear_workspace_bytes(&w, 4096, 8, QLORA_OP_BWD, QLORA_COMPUTE_BF16);
  CHECK(fwd >= 256 && fwd % 256 == 0 && bwd >= 256 && bwd % 256 == 0);
  CHECK(qlora_linear_workspace_bytes(&w, 4096, 65, QLORA_OP_FWD, QLORA_COMPUTE_BF16) == 0);

  /* rejected before anything is launched */
  CHECK(qlora_merge(NULL, NULL, NULL, 8, 1.0f, NULL, NULL) == QLORA_ERR_INVALID_ARG);
  CHECK(qlora_dequantize(NULL, NULL, NULL) == QLORA_ERR_INVALID_ARG);
  CHECK(qlora_adam_step(NULL, NULL, NULL, NULL, 0, 1, 1e-3f, 0.9f, 0.999f, 1e-8f, 0, NULL) ==
        QLORA_OK);
  CHECK(qlora_adam_step(NULL, NULL, NULL, NULL, 4, 0, 1e-3f, 0.9f, 0.999f, 1e-8f, 0, NULL) ==
        QLORA_ERR_SHAPE);
  CHECK(qlora_kernel_timing_enable(-1) == QLORA_ERR_INVALID_ARG);
  printf("ok\n");
  return 0;
}
