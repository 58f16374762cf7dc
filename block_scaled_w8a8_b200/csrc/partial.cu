// partial.cu -- the last step of a linear layer whose K dimension is split
// over several GPUs (row-parallel tensor parallelism, block-wise INT8 page,
// section 3): after the fp32 partials of all K shards have been summed, add
// the bias once and round once to bf16, so that the sharded layer rounds
// exactly as often as the unsharded one.
#include <cuda_runtime.h>
#include <stdint.h>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {

namespace {

// out[m, n] = bf16(part[m, n] + bias[n]); 4 columns per thread when the
// rows allow 16-byte loads and 8-byte stores.
__global__ void __launch_bounds__(256)
finish_bf16_kernel(const float* __restrict__ part, int64_t ldp, int64_t M, int64_t N,
                   const uint16_t* __restrict__ bias, uint16_t* __restrict__ out, int64_t ldo,
                   bool vec) {
  const int64_t nq = vec ? N / 4 : N;
  const int64_t total = M * nq;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / nq, c = i - m * nq;
    if (vec) {
      const float4 v = *reinterpret_cast<const float4*>(part + m * ldp + 4 * c);
      float x[4] = {v.x, v.y, v.z, v.w};
      uint16_t h[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (bias) x[e] += bf16_bits_to_float(bias[4 * c + e]);
        h[e] = float_to_bf16_bits(x[e]);
      }
      *reinterpret_cast<uint2*>(out + m * ldo + 4 * c) =
          make_uint2((uint32_t)h[0] | ((uint32_t)h[1] << 16),
                     (uint32_t)h[2] | ((uint32_t)h[3] << 16));
    } else {
      float x = part[m * ldp + c];
      if (bias) x += bf16_bits_to_float(bias[c]);
      out[m * ldo + c] = float_to_bf16_bits(x);
    }
  }
}

}  // namespace

cudaError_t launch_finish_bf16(const float* part, int64_t ldp, int64_t M, int64_t N,
                               const void* bias, void* out, int64_t ldo, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  const bool vec = N % 4 == 0 && ldp % 4 == 0 && ldo % 4 == 0 &&
                   (reinterpret_cast<uintptr_t>(part) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) & 7) == 0;
  const int64_t work = M * (vec ? N / 4 : N);
  const int64_t blocks = (work + 255) / 256;
  const unsigned grid = (unsigned)(blocks < 148 * 16 ? (blocks < 1 ? 1 : blocks) : 148 * 16);
  finish_bf16_kernel<<<grid, 256, 0, st>>>(part, ldp, M, N,
                                           static_cast<const uint16_t*>(bias),
                                           static_cast<uint16_t*>(out), ldo, vec);
  return cudaGetLastError();
}

}  // namespace bq
