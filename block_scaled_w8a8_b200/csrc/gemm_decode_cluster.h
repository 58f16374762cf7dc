// gemm_decode_cluster.h -- the few-token (decode) block-scaled GEMM whose
// split-K partials are reduced inside thread-block clusters.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace bq {

struct DecClusterArgs {
  const void* qa; int64_t lda;         // activation codes [M, lda]
  const float* sa;                     // activation scales [Kb][M]
  const void* qw; int64_t ldw;         // weight codes [N, ldw]
  const float* sw;                     // weight scales [ceil(N/128)][Kb]
  int64_t M, N, K, bn, bk;
  int dtype;
  const void* bias;                    // bf16 [N] or nullptr
  void* out; int64_t ldo;              // bf16 [M, ldo]
  float* out_f32;                      // or: unrounded fp32 [M, ldo], no bias
  unsigned* status;
  bool pdl;                            // programmatic dependent launch
};

struct DecClusterPlan {
  int nt;          // token tile (MMA N): 16, 32, 64 or 128
  int64_t tiles;   // 128-row weight tiles (one cluster each)
  int S;           // K-splits per tile (CTAs per cluster)
  bool ok;         // the split fits the kernel's per-CTA K-block limit
};

DecClusterPlan gemm_decode_cluster_plan(int64_t M, int64_t N, int64_t K);
bool gemm_decode_cluster_supported(const DecClusterArgs& a, char* why, size_t n);
// pdl: the kernel requests its weights (codes and scales) before it waits
// for the preceding kernel on the stream, which therefore must not write them.
cudaError_t launch_gemm_decode_cluster(const DecClusterArgs& a, cudaStream_t st);

}  // namespace bq
