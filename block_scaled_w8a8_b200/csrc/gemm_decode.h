// gemm_decode.h -- the few-token (decode) weight-streaming GEMM.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "bq_internal.h"

namespace bq {

// Arrival counters occupy the first 64 KiB of a decode workspace (one per
// 128-row weight tile, so N <= 2^21 rows); the split partials follow.
constexpr size_t kDecodeCounterBytes = 65536;

struct DecodePlan {
  int nt;              // token tile (MMA N): 16, 32, 64 or 128
  int64_t tiles;       // 128-row weight tiles
  int splits;          // K splits per tile (cluster mode: chosen at launch)
  bool cluster;        // splits reduce over distributed shared memory
  size_t part_bytes;   // fp32 split partials
  size_t ws_bytes;     // counter region + partials (0 unless workspace mode)
};

DecodePlan decode_plan(int64_t M, int64_t N, int64_t K);
bool decode_supported(const GemmArgs& a, char* why, size_t n);
// Fixed scratch of bq_gemm_decode_noalloc (counter region included).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxScratchDevices = 64;
// Device address of that scratch on the current device (cudaGetSymbolAddress;
// looked up on every call made outside stream capture).
cudaError_t noalloc_scratch(void** ptr, cudaStream_t st);

// pdl: launch as a programmatic dependent of the preceding kernel (which must
// not write the weights).  ws: zero-filled workspace of plan.ws_bytes.
cudaError_t launch_gemm_decode(const GemmArgs& a, void* ws, bool pdl, cudaStream_t st);

}  // namespace bq
