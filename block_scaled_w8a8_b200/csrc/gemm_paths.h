// gemm_paths.h -- kernel-family choice and workspace sizing for the GEMMs.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "bq_internal.h"

namespace bq {

enum RunCode : int { kRunOk = 0, kRunUnsupported = 1, kRunAlignment = 2, kRunCuda = 3 };

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t bn, int64_t bk, int dtype);
size_t grouped_workspace_bytes(int64_t R, int64_t N, int64_t K, int64_t E, int64_t bn,
                               int64_t bk, int dtype);

// Runs a dense GEMM with the forced path (or the automatic choice).  On
// failure writes a reason into `why`.
int run_gemm(const GemmArgs& a, int path, void* ws, size_t ws_bytes, cudaStream_t st,
             char* why, size_t why_len);
// The GEMM half of bq_linear: like run_gemm, but a decode-path launch may
// start as a programmatic dependent of the activation quantiser before it.
int run_gemm_after_quant(const GemmArgs& a, int path, void* ws, size_t ws_bytes,
                         cudaStream_t st, char* why, size_t why_len);
int run_grouped_gemm(const GemmArgs& a, int path, void* ws, size_t ws_bytes, cudaStream_t st,
                     char* why, size_t why_len);

}  // namespace bq
