/* A plain C consumer of the library's ABI: include/fqa.h must compile as C99
 * and libfqa.so must link and answer the calls that need no GPU (versions,
 * status strings, sizes, argument validation before any launch). */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fqa.h"

int main(void) {
  int fails = 0;
#define CHECK(cond)                                   \
  do {                                                \
    if (!(cond)) {                                    \
      printf("FAIL %s:%d %s\n", __FILE__, __LINE__, #cond); \
      ++fails;                                        \
    }                                                 \
  } while (0)
  printf("version %d.%d\n", fqa_version() >> 16, fqa_version() & 0xFFFF);
  CHECK(strcmp(fqa_status_string(FQA_OK), "") != 0);
  CHECK(fqa_status_string(FQA_ERR_TIMEOUT) != fqa_status_string(FQA_OK));
  /* B*H*(N/64)*d*4 rounded up to 256, plus 256 bytes of counters */
  CHECK(fqa_quantize_workspace_bytes(1, 24, 8704, 128) == 1671168 + 256);
  CHECK(fqa_quantize_workspace_bytes(1, 1, 100, 128) == 1024 + 256); /* a short last block */
  CHECK(fqa_quantize_workspace_bytes(1, 1, 100, 64) == 0);
  /* 8 MiB of partial sums plus the 256 counter bytes: exactly 16384 blocks fit */
  CHECK(fqa_quantize_noalloc_max_workspace_bytes() == ((size_t)8 << 20) + 256);
  CHECK(fqa_quantize_workspace_bytes(1, 16, 65536, 128) == fqa_quantize_noalloc_max_workspace_bytes());
  /* argument errors come back before anything is launched */
  void* p = (void*)(uintptr_t)0x10000;
  float* f = (float*)p;
  CHECK(fqa_quantize(NULL, p, p, 1, 1, 128, 128, p, p, p, f, f, f, f, f, p, 1 << 20, NULL) ==
        FQA_ERR_INVALID_ARG);
  CHECK(fqa_quantize(p, p, p, 1, 1, 128, 64, p, p, p, f, f, f, f, f, p, 1 << 20, NULL) ==
        FQA_ERR_UNSUPPORTED);
  CHECK(fqa_attention_fp8(p, p, p, f, f, f, f, 1, 1, 192, 64, 0.088f, p, FQA_OUT_BF16, NULL) ==
        FQA_ERR_UNSUPPORTED);
  CHECK(fqa_attention_bf16(p, p, p, 1, 1, 128, 128, -1.0f, p, FQA_OUT_BF16, NULL) ==
        FQA_ERR_INVALID_ARG);
  CHECK(fqa_e4m3_encode(NULL, (uint8_t*)p, 4, NULL) == FQA_ERR_INVALID_ARG);
  uint8_t* u = (uint8_t*)p;
  CHECK(fqa_attention_nvfp4(u, u, u, u, f, f, p, f, f, 1, 1, 200, 64, 0.088f, p, FQA_OUT_BF16, NULL) ==
        FQA_ERR_UNSUPPORTED);
  CHECK(fqa_quantize_nvfp4_qk(p, p, f, 1, 1, 128, 128, NULL, u, u, u, f, f, NULL) == FQA_ERR_INVALID_ARG);
  CHECK(fqa_e2m1_encode(NULL, u, 4, NULL) == FQA_ERR_INVALID_ARG);
  printf("%s (%d failed)\n", fails ? "FAILED" : "OK", fails);
  return fails ? 1 : 0;
}
