/* A C11 program against include/mxq.h and libmxq.so: the header compiles as
 * plain C, the library links from C, and calls that fail validation return
 * their status without touching the (fake) device pointers or needing a GPU.
 * Prints "abi_check: all N checks passed" and exits 0, else lists failures
 * and exits 1. Built and run by tests/test_abi.py. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mxq.h"

static int checks, failures;

static void expect(const char* what, long long got, long long want) {
  ++checks;
  if (got != want) {
    ++failures;
    printf("FAIL %s: got %lld, want %lld\n", what, got, want);
  }
}

int main(void) {
  /* a 16-byte-aligned fake device address: never dereferenced, because every
     call below is rejected (or has nothing to do) before any launch */
  void* A = (void*)(uintptr_t)0x10000;
  uint8_t* B = (uint8_t*)A;
  const mxq_stream_t s = 0;

  expect("abi version", mxq_abi_version(), MXQ_ABI_VERSION);
  for (int st = MXQ_OK; st <= MXQ_ERR_ARG; ++st)
    expect("status string present", mxq_status_string(st) != NULL && strlen(mxq_status_string(st)) > 0, 1);

  /* size helpers: 130 rows pad to 256, 5 scale columns to 8 */
  expect("swizzled scale bytes", mxq_swizzled_scale_bytes(130, 5), 256 * 8);
  expect("swizzled scale bytes, negative", mxq_swizzled_scale_bytes(-1, 5), -1);
  expect("nvfp4 workspace bytes", mxq_nvfp4_workspace_bytes(8192, 8192) > 0, 1);

  /* MXFP8 */
  expect("quantize N % 32", mxfp8_quantize(A, MXQ_BF16, 4, 48, 48, B, B, NULL, s), MXQ_ERR_SHAPE);
  expect("quantize dtype", mxfp8_quantize(A, 7, 4, 64, 64, B, B, NULL, s), MXQ_ERR_DTYPE);
  expect("quantize ld_x < N", mxfp8_quantize(A, MXQ_BF16, 4, 64, 32, B, B, NULL, s), MXQ_ERR_SHAPE);
  expect("quantize NULL x", mxfp8_quantize(NULL, MXQ_BF16, 4, 64, 64, B, B, NULL, s), MXQ_ERR_NULL);
  expect("quantize misaligned x", mxfp8_quantize(B + 2, MXQ_BF16, 4, 64, 64, B, B, NULL, s),
         MXQ_ERR_ALIGN);
  expect("quantize empty", mxfp8_quantize(NULL, MXQ_BF16, 0, 64, 64, NULL, NULL, NULL, s), MXQ_OK);
  expect("dequantize N % 32", mxfp8_dequantize(B, B, 4, 48, A, MXQ_BF16, s), MXQ_ERR_SHAPE);
  expect("dequantize NULL y", mxfp8_dequantize(B, B, 4, 64, NULL, MXQ_BF16, s), MXQ_ERR_NULL);

  /* grouped, stacked */
  const int64_t* offs = (const int64_t*)(uintptr_t)0x10100;
  expect("grouped E = 0", mxfp8_quantize_grouped(A, MXQ_BF16, 0, offs, 64, 64, B, B, s), MXQ_ERR_SHAPE);
  expect("grouped NULL offsets", mxfp8_quantize_grouped(A, MXQ_BF16, 4, NULL, 64, 64, B, B, s),
         MXQ_ERR_NULL);
  expect("grouped swizzled negative bytes",
         mxfp8_quantize_grouped_swizzled(A, MXQ_BF16, 4, offs, 64, 64, B, B, B, -1, s), MXQ_ERR_SHAPE);

  /* columnwise, MXFP4, fake quantize */
  expect("columnwise N % 16", mxfp8_quantize_columnwise(A, MXQ_BF16, 64, 24, 24, B, B, NULL, NULL, s),
         MXQ_ERR_SHAPE);
  expect("mxfp4 N % 32", mxfp4_quantize(A, MXQ_BF16, 4, 48, 48, B, B, NULL, s), MXQ_ERR_SHAPE);
  expect("fake quantize format", mx_fake_quantize(9, A, MXQ_BF16, 4, 64, 64, A, MXQ_BF16, s), MXQ_ERR_ARG);

  /* GEMM */
  expect("gemm K % 32", mxfp8_gemm(B, B, B, B, 128, 128, 48, A, MXQ_BF16, NULL, s), MXQ_ERR_SHAPE);
  expect("gemm NULL output", mxfp8_gemm(B, B, B, B, 128, 128, 64, NULL, MXQ_BF16, NULL, s), MXQ_ERR_NULL);
  expect("bounded wait limit below 1 us", mxq_check_bounded_wait(999, (int64_t*)A, s), MXQ_ERR_ARG);
  expect("bounded wait limit above 1 s", mxq_check_bounded_wait(1000000001, (int64_t*)A, s), MXQ_ERR_ARG);
  expect("bounded wait NULL result", mxq_check_bounded_wait(2000000, NULL, s), MXQ_ERR_NULL);
  expect("bounded wait misaligned result", mxq_check_bounded_wait(2000000, (int64_t*)(B + 4), s),
         MXQ_ERR_ALIGN);

  /* NVFP4 */
  float* g = (float*)A;
  expect("nvfp4 N % 16", nvfp4_quantize(A, MXQ_BF16, 4, 24, 24, B, B, g, NULL, 0, A, 1 << 20, s),
         MXQ_ERR_SHAPE);
  expect("nvfp4 missing workspace", nvfp4_quantize(A, MXQ_BF16, 4, 64, 64, B, B, g, NULL, 0, NULL, 0, s),
         MXQ_ERR_WORKSPACE);
  expect("nvfp4 given scale and amax", nvfp4_quantize(A, MXQ_BF16, 4, 64, 64, B, B, g, g,
                                                      MXQ_NVFP4_GLOBAL_GIVEN, NULL, 0, s),
         MXQ_ERR_ARG);
  expect("nvfp4 dequantize N % 16", nvfp4_dequantize(B, B, g, 4, 24, A, MXQ_BF16, s), MXQ_ERR_SHAPE);

  if (failures) {
    printf("abi_check: %d of %d checks failed\n", failures, checks);
    return 1;
  }
  printf("abi_check: all %d checks passed\n", checks);
  return 0;
}
