/* Plain C99 client of the C ABI: compiled by tests/test_abi_host.py with
 * gcc -std=c99 -pedantic against include/fp8lin.h and linked against libfp8lin.so.
 * It checks that the header is valid C and its size macros evaluate as documented,
 * and calls entry points with bad arguments, which are refused before any CUDA call,
 * so it runs without a GPU. */
#include <stdio.h>
#include <string.h>
#include "fp8lin.h"
int main(void) {
  if (strcmp(fp8_status_string(FP8_OK), "ok") != 0) return 1;
  /* bad arguments are refused before any CUDA call, so this runs without a GPU */
  if (fp8_act_quant((const void*)0, -1, 128, 128, 128, FP8_E4M3, FP8_SCALE_FP32, (void*)0, (float*)0, (void*)0) != FP8_ERR_INVALID_ARG) return 2;
  if (fp8_block_gemm((const void*)0, (const float*)0, (const void*)0, (const float*)0, 4, 256, 200, FP8_OUT_BF16, (void*)0, (void*)0) == FP8_OK) return 3;
  if (FP8_MOE_ROUTE_WS_BYTES(4096, 8, 256) != (int64_t)65 * 256 * 4) return 4;
  if (FP8_MX_SF_BYTES(300, 1024) != (int64_t)3 * 8 * 512) return 5;
  printf("c abi ok\n");
  return 0;
}
