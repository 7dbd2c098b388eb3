/* The C ABI driven from plain C on the GPU, with no Python or torch in the
 * process: reads two [M, N] bf16 tensors (raw little-endian bit patterns)
 * from files, quantizes the first to MXFP8 (compact and swizzled scales),
 * dequantizes its codes to bf16 and quantizes the second to NVFP4 with the
 * no-alloc entry point, on the legacy default stream, then writes every
 * output to <prefix>.{q,s,z,y,p4,b4,g4}. Exit status 0 when every call
 * returned MXQ_OK and the CUDA runtime reported no error. Built and run by
 * tests/test_gpu_c_abi.py, which checks the outputs against the oracle and
 * the hand-worked groups.
 *
 * usage: gpu_roundtrip M N mxfp8_input.bin nvfp4_input.bin output_prefix */
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "mxq.h"

static int fail(const char* what, const char* detail) {
  fprintf(stderr, "gpu_roundtrip: %s: %s\n", what, detail);
  return 1;
}

static int write_back(const char* prefix, const char* ext, const void* dev, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s.%s", prefix, ext);
  void* host = malloc(bytes ? bytes : 1);
  if (!host) return fail("malloc", ext);
  if (cudaMemcpy(host, dev, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) {
    free(host);
    return fail("cudaMemcpy to host", ext);
  }
  FILE* f = fopen(path, "wb");
  const int ok = f && fwrite(host, 1, bytes, f) == bytes;
  if (f) fclose(f);
  free(host);
  return ok ? 0 : fail("write", path);
}

int main(int argc, char** argv) {
  if (argc != 6)
    return fail("usage", "gpu_roundtrip M N mxfp8_input.bin nvfp4_input.bin output_prefix");
  const int64_t M = atoll(argv[1]), N = atoll(argv[2]);
  if (M <= 0 || N <= 0 || N % 32 != 0) return fail("arguments", "M > 0 and N a multiple of 32");
  const size_t elems = (size_t)M * (size_t)N;

  uint16_t* xh = malloc(2 * elems * sizeof *xh);  /* both inputs, one after the other */
  if (!xh) return fail("malloc", "input");
  for (int i = 0; i < 2; i++) {
    FILE* in = fopen(argv[3 + i], "rb");
    if (!in || fread(xh + i * elems, sizeof *xh, elems, in) != elems) return fail("read", argv[3 + i]);
    fclose(in);
  }

  const size_t s_bytes = elems / 32, z_bytes = (size_t)mxq_swizzled_scale_bytes(M, N / 32);
  void *x, *xn, *q, *s, *z, *y, *p4, *b4, *g4;
  if (cudaMalloc(&x, elems * 2) || cudaMalloc(&xn, elems * 2) || cudaMalloc(&q, elems) ||
      cudaMalloc(&s, s_bytes) || cudaMalloc(&z, z_bytes) || cudaMalloc(&y, elems * 2) || cudaMalloc(&p4, elems / 2) ||
      cudaMalloc(&b4, elems / 16) || cudaMalloc(&g4, sizeof(float)))
    return fail("cudaMalloc", cudaGetErrorString(cudaGetLastError()));
  if (cudaMemcpy(x, xh, elems * 2, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(xn, xh + elems, elems * 2, cudaMemcpyHostToDevice) != cudaSuccess)
    return fail("cudaMemcpy to device", cudaGetErrorString(cudaGetLastError()));
  free(xh);

  mxq_status st = mxfp8_quantize(x, MXQ_BF16, M, N, N, q, s, z, 0);
  if (st != MXQ_OK) return fail("mxfp8_quantize", mxq_status_string(st));
  st = mxfp8_dequantize(q, s, M, N, y, MXQ_BF16, 0);
  if (st != MXQ_OK) return fail("mxfp8_dequantize", mxq_status_string(st));
  st = nvfp4_quantize_noalloc(xn, MXQ_BF16, M, N, N, p4, b4, g4, NULL, 0, 0);
  if (st != MXQ_OK) return fail("nvfp4_quantize_noalloc", mxq_status_string(st));
  const cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail("cudaDeviceSynchronize", cudaGetErrorString(e));

  const char* pre = argv[5];
  if (write_back(pre, "q", q, elems) || write_back(pre, "s", s, s_bytes) ||
      write_back(pre, "z", z, z_bytes) || write_back(pre, "y", y, elems * 2) ||
      write_back(pre, "p4", p4, elems / 2) || write_back(pre, "b4", b4, elems / 16) ||
      write_back(pre, "g4", g4, sizeof(float)))
    return 1;
  cudaFree(x); cudaFree(xn); cudaFree(q); cudaFree(s); cudaFree(z); cudaFree(y);
  cudaFree(p4); cudaFree(b4); cudaFree(g4);
  printf("gpu_roundtrip: ok\n");
  return 0;
}
