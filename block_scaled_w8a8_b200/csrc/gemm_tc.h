// gemm_tc.h -- the tcgen05 tensor-core GEMM (dense and grouped).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "bq_internal.h"

namespace bq {

// True if the tensor-core kernel can run this problem; otherwise writes why.
bool tc_supported(const GemmArgs& a, char* why, size_t n);
// The fused form for a gate/up weight (N = 2I, seam = I): the single-CTA
// kernel's epilogue computes h = bf16(silu(g) * u) and writes h's 1 x 128
// codes and scales (q_out, ldq, s_out) instead of the bf16 GEMM output.
bool tc_silu_supported(const GemmArgs& a, char* why, size_t n);
cudaError_t launch_gemm_tc_silu(const GemmArgs& a, cudaStream_t st);
// Single-CTA kernel: 128 x 256 tiles (128 x 128 for N <= 128).
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st);

}  // namespace bq
