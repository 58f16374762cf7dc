// gemm_dispatch.cu -- picks the GEMM kernel family for a problem.
//
//   SIMT     generic CUDA-core kernel: any shape, stride, block size.
//   TCGEN05  TMA + tcgen05 kernel: block_n = block_k = 128, 16-byte strides.
// AUTO takes the tensor-core kernel whenever it applies and M is large
// enough to fill an MMA tile, else the CUDA-core kernel.
#include <cstdio>

#include "../../include/bq.h"
#include "gemm_paths.h"
#include "gemm_tc.h"

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

static int run_tc(const GemmArgs& a, cudaStream_t st, char* why, size_t n) {
  cudaError_t e = launch_gemm_tc(a, st);
  if (e != cudaSuccess) {
    snprintf(why, n, "tcgen05 GEMM launch: %s", cudaGetErrorString(e));
    return kRunCuda;
  }
  return kRunOk;
}

constexpr int64_t kTcMinRows = 65;

int run_gemm(const GemmArgs& a, int path, void* ws, size_t ws_bytes, cudaStream_t st, char* why,
             size_t why_len) {
  (void)ws;
  (void)ws_bytes;
  switch (path) {
    case BQ_PATH_AUTO:
      if (a.M >= kTcMinRows && tc_supported(a, nullptr, 0)) return run_tc(a, st, why, why_len);
      return run_simt(a, st, why, why_len);
    case BQ_PATH_SIMT:
      return run_simt(a, st, why, why_len);
    case BQ_PATH_TCGEN05:
      if (!tc_supported(a, why, why_len)) return kRunUnsupported;
      return run_tc(a, st, why, why_len);
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
      if (tc_supported(a, nullptr, 0)) return run_tc(a, st, why, why_len);
      return run_simt(a, st, why, why_len);
    case BQ_PATH_SIMT:
      return run_simt(a, st, why, why_len);
    case BQ_PATH_TCGEN05:
      if (!tc_supported(a, why, why_len)) return kRunUnsupported;
      return run_tc(a, st, why, why_len);
    default:
      snprintf(why, why_len, "kernel path %d is not available for grouped GEMM", path);
      return kRunUnsupported;
  }
}

}  // namespace bq
