// gemm_dispatch.cu -- picks the GEMM kernel family for a problem.
//
//   SIMT    generic CUDA-core kernel: any shape, stride, block size.
#include <cstdio>

#include "../../include/bq.h"
#include "gemm_paths.h"

namespace bq {

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t, int) { return 0; }

size_t grouped_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t, int64_t, int) {
  return 0;
}

static int run_simt(const GemmArgs& a, cudaStream_t st, char* why, size_t n) {
  cudaError_t e = launch_gemm_simt(a, st);
  if (e != cudaSuccess) {
    snprintf(why, n, "SIMT GEMM launch: %s", cudaGetErrorString(e));
    return kRunCuda;
  }
  return kRunOk;
}

int run_gemm(const GemmArgs& a, int path, void* ws, size_t ws_bytes, cudaStream_t st, char* why,
             size_t why_len) {
  (void)ws;
  (void)ws_bytes;
  switch (path) {
    case BQ_PATH_AUTO:
    case BQ_PATH_SIMT:
      return run_simt(a, st, why, why_len);
    default:
      snprintf(why, why_len, "kernel path %d is not available in this build", path);
      return kRunUnsupported;
  }
}

int run_grouped_gemm(const GemmArgs& a, int path, void* ws, size_t ws_bytes, cudaStream_t st,
                     char* why, size_t why_len) {
  (void)ws;
  (void)ws_bytes;
  switch (path) {
    case BQ_PATH_AUTO:
    case BQ_PATH_SIMT:
      return run_simt(a, st, why, why_len);
    default:
      snprintf(why, why_len, "kernel path %d is not available for grouped GEMM", path);
      return kRunUnsupported;
  }
}

}  // namespace bq
