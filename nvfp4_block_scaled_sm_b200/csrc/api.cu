// api.cu -- library-wide entry points of libmxq: version, status strings,
// CUDA error reporting and output-size helpers.
#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace mxq {

namespace {
thread_local char g_last_cuda_error[256] = "";
}

void record_cuda_error(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
}

mxq_status check_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return MXQ_ERR_CUDA;
  }
  return MXQ_OK;
}

}  // namespace mxq

extern "C" {

int mxq_abi_version(void) { return MXQ_ABI_VERSION; }

const char* mxq_status_string(int status) {
  switch (status) {
    case MXQ_OK: return "ok";
    case MXQ_ERR_NULL: return "a required pointer is NULL";
    case MXQ_ERR_SHAPE: return "invalid shape (negative size, N not a multiple of the group, ld_x < N, or size limit)";
    case MXQ_ERR_DTYPE: return "unknown dtype";
    case MXQ_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case MXQ_ERR_WORKSPACE: return "workspace missing or too small";
    case MXQ_ERR_CUDA: return "CUDA launch failed";
    case MXQ_ERR_ARG: return "inconsistent arguments";
    default: return "unknown status";
  }
}

const char* mxq_last_cuda_error(void) { return mxq::g_last_cuda_error; }

int64_t mxq_swizzled_scale_bytes(int64_t M, int64_t S) {
  if (M < 0 || S < 0) return -1;
  return ((M + 127) / 128 * 128) * ((S + 3) / 4 * 4);
}

int64_t mxq_grouped_swizzled_scale_bytes_max(int32_t E, int64_t M_total, int64_t S) {
  if (E < 0 || M_total < 0 || S < 0) return -1;
  // each expert pads its rows to a multiple of 128, adding at most 127 rows
  return ((M_total + 127 * int64_t(E)) / 128 * 128) * ((S + 3) / 4 * 4);
}

}  // extern "C"
