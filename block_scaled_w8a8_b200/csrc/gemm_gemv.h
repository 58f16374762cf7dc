// gemm_gemv.h -- the CUDA-core block-scaled INT8 GEMM for 1..8 tokens.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "bq_internal.h"

namespace bq {

constexpr int64_t kGemvMaxRows = 8;

bool gemv_supported(const GemmArgs& a, char* why, size_t n);
// pdl: launch as a programmatic dependent of the preceding kernel (which must
// not write the weights).
cudaError_t launch_gemm_gemv(const GemmArgs& a, bool pdl, cudaStream_t st);

}  // namespace bq
