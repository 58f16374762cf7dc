// gemm_mx.h -- MXFP8 quantisers and the block-scaled tensor-core GEMM.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace bq {

struct MxArgs {
  const void* qa; int64_t lda; const void* sfa;   // e4m3 [M, K], scale atoms
  const void* qw; int64_t ldw; const void* sfw;   // e4m3 [N, K], scale atoms
  int64_t M, N, K;                                 // K a multiple of 128
  const void* bias;                                // bf16 [N] or nullptr
  void* out; int64_t ldo;                          // bf16 [M, N]
  unsigned* status;
};

// Bytes of the scale atoms of R rows: ceil(R / 128) * (K / 128) * 512.
size_t mx_scale_bytes(int64_t R, int64_t K);
cudaError_t launch_mx_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, void* q,
                                int64_t ldq, void* sf, cudaStream_t st);
cudaError_t launch_mx_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw, void* q,
                                   int64_t ldq, void* sf, cudaStream_t st);
cudaError_t launch_gemm_mx(const MxArgs& a, cudaStream_t st);

}  // namespace bq
