// gemm_dispatch.cu -- picks the GEMM kernel family for a problem.
//
//   SIMT     generic CUDA-core kernel: any shape, stride, block size.
//   TCGEN05  TMA + tcgen05 kernel: block_n = block_k = 128, 16-byte strides.
//   DECODE   swap-AB split-K weight-streaming tcgen05 kernels, M <= 128: the
//            cluster kernel of gemm_decode_cluster.cu (split-K reduced over
//            distributed shared memory, no workspace) where it applies,
//            else the workspace split-K kernel of gemm_decode.cu.
// AUTO: M <= 128 -> DECODE, larger M -> TCGEN05, when they apply; otherwise
// the generic CUDA-core kernel.
#include <cstdio>

#include "bq.h"
#include "gemm_paths.h"
#include "gemm_decode.h"
#include "gemm_tc.h"
#include "gemm_decode_cluster.h"

namespace bq {

constexpr int64_t kDecodeMaxRows = 128;

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t bn, int64_t bk, int) {
  if (M < 1 || M > kDecodeMaxRows || N < 1 || K < 1 || bn != 128 || bk != 128) return 0;
  return decode_plan(M, N, K).ws_bytes;
}

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

static int run_tc(const GemmArgs& a0, int path, cudaStream_t st, char* why, size_t n) {
  GemmArgs a = a0;
  a.tc_shape = path == BQ_PATH_TCGEN05_1CTA ? 1 : path == BQ_PATH_TCGEN05_PAIR ? 2 : 0;
  cudaError_t e = launch_gemm_tc(a, st);
  if (e != cudaSuccess) {
    snprintf(why, n, "tcgen05 GEMM launch: %s", cudaGetErrorString(e));
    return kRunCuda;
  }
  return kRunOk;
}

static int run_decode(const GemmArgs& a, void* ws, size_t ws_bytes, bool pdl, cudaStream_t st,
                      char* why, size_t n) {
  const size_t need = decode_plan(a.M, a.N, a.K).ws_bytes;
  if (need > 0 && (ws == nullptr || ws_bytes < need)) {
    snprintf(why, n, "decode path needs %zu workspace bytes, got %zu", need, ws_bytes);
    return kRunUnsupported;
  }
  cudaError_t e = launch_gemm_decode(a, ws, pdl, st);
  if (e != cudaSuccess) {
    snprintf(why, n, "decode GEMM launch: %s", cudaGetErrorString(e));
    return kRunCuda;
  }
  return kRunOk;
}

// The cluster decode kernel.  Launched as a programmatic dependent of the
// preceding kernel: it requests its weights before waiting for that kernel,
// which therefore must not write them.
static bool cluster_decode_args(const GemmArgs& a, DecClusterArgs* d) {
  *d = DecClusterArgs{};
  d->qa = a.qa; d->lda = a.lda; d->sa = a.sa;
  d->qw = a.qw; d->ldw = a.ldw; d->sw = a.sw;
  d->M = a.M; d->N = a.N; d->K = a.K; d->bn = a.bn; d->bk = a.bk;
  d->dtype = a.dtype; d->bias = a.bias; d->out = a.out; d->ldo = a.ldo;
  d->out_f32 = a.out_f32;
  d->status = a.status; d->pdl = true;
  return !a.offsets && a.sa_rows == a.M && gemm_decode_cluster_supported(*d, nullptr, 0);
}

static int run_cluster_decode(const DecClusterArgs& d, cudaStream_t st, char* why, size_t n) {
  cudaError_t e = launch_gemm_decode_cluster(d, st);
  if (e != cudaSuccess) {
    snprintf(why, n, "decode GEMM launch: %s", cudaGetErrorString(e));
    return kRunCuda;
  }
  return kRunOk;
}

static int dispatch_dense(const GemmArgs& a, int path, void* ws, size_t ws_bytes, bool pdl,
                          cudaStream_t st, char* why, size_t why_len) {
  switch (path) {
    case BQ_PATH_AUTO: {
      DecClusterArgs d;
      if (a.M <= kDecodeMaxRows && cluster_decode_args(a, &d))
        return run_cluster_decode(d, st, why, why_len);
      if (a.M <= kDecodeMaxRows && !a.out_f32 && decode_supported(a, nullptr, 0))
        return run_decode(a, ws, ws_bytes, pdl, st, why, why_len);
      if (a.M > kDecodeMaxRows && tc_supported(a, nullptr, 0)) return run_tc(a, path, st, why, why_len);
      return run_simt(a, st, why, why_len);
    }
    case BQ_PATH_DECODE: {
      DecClusterArgs d;
      if (a.M <= kDecodeMaxRows && cluster_decode_args(a, &d))
        return run_cluster_decode(d, st, why, why_len);
      if (a.out_f32) {
        snprintf(why, why_len, "decode path: fp32 partial output needs the cluster kernel");
        return kRunUnsupported;
      }
      if (!decode_supported(a, why, why_len)) return kRunUnsupported;
      return run_decode(a, ws, ws_bytes, pdl, st, why, why_len);
    }
    case BQ_PATH_SIMT:
      return run_simt(a, st, why, why_len);
    case BQ_PATH_TCGEN05:
    case BQ_PATH_TCGEN05_1CTA:
    case BQ_PATH_TCGEN05_PAIR:
      if (!tc_supported(a, why, why_len)) return kRunUnsupported;
      return run_tc(a, path, st, why, why_len);
    default:
      snprintf(why, why_len, "kernel path %d is not available in this build", path);
      return kRunUnsupported;
  }
}

int run_gemm(const GemmArgs& a, int path, void* ws, size_t ws_bytes, cudaStream_t st, char* why,
             size_t why_len) {
  return dispatch_dense(a, path, ws, ws_bytes, false, st, why, why_len);
}

int run_gemm_after_quant(const GemmArgs& a, int path, void* ws, size_t ws_bytes,
                         cudaStream_t st, char* why, size_t why_len) {
  return dispatch_dense(a, path, ws, ws_bytes, true, st, why, why_len);
}

int run_grouped_gemm(const GemmArgs& a, int path, void* ws, size_t ws_bytes, cudaStream_t st,
                     char* why, size_t why_len) {
  (void)ws;
  (void)ws_bytes;
  switch (path) {
    case BQ_PATH_AUTO:
      if (tc_supported(a, nullptr, 0)) return run_tc(a, path, st, why, why_len);
      return run_simt(a, st, why, why_len);
    case BQ_PATH_SIMT:
      return run_simt(a, st, why, why_len);
    case BQ_PATH_TCGEN05:
    case BQ_PATH_TCGEN05_1CTA:
    case BQ_PATH_TCGEN05_PAIR:
      if (!tc_supported(a, why, why_len)) return kRunUnsupported;
      return run_tc(a, path, st, why, why_len);
    default:
      snprintf(why, why_len, "kernel path %d is not available for grouped GEMM", path);
      return kRunUnsupported;
  }
}

}  // namespace bq
