// bq_common.cuh -- device helpers shared by the libbq kernels (sm_100a).
//
// Quantisation rule (block-wise INT8 page, sections 2 and 4; e4m3 layout of the
// FP8 section of the LLM-quantization overview page), with the readings taken
// where the pages are silent:
//   s = amax / Q, one IEEE fp32 division (Q = 127 INT8, 448 FP8 e4m3)
//   INT8: q = clamp(round_half_even(x / s), -128, 127)
//   FP8 : q = cvt.rn.satfinite.e4m3(x / s)
//   s == 0 (all-zero group): every code is 0.
// The division is __fdiv_rn (IEEE round-to-nearest); the library is built
// without fast-math and without flush-to-zero so subnormal scales behave
// like the CPU.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bq {

enum : int { kInt8 = 0, kFp8 = 1 };

// ---- device status word -------------------------------------------------
// Layout: bits [0,8) kind, bits [8,32) site.  The first error wins (CAS).
enum : unsigned { kStatusTimeout = 1u, kStatusBadInput = 2u };

__device__ __forceinline__ void record_status(unsigned* status, unsigned kind, unsigned site) {
  if (status) atomicCAS(status, 0u, (site << 8) | kind);
}

// ---- scalar quantisation --------------------------------------------------
template <int DT>
__device__ __forceinline__ float qmax_of() { return DT == kInt8 ? 127.0f : 448.0f; }

// Scale of a group from its amax: one IEEE fp32 division.
template <int DT>
__device__ __forceinline__ float group_scale(float amax) {
  return __fdiv_rn(amax, qmax_of<DT>());
}

// INT8 code of x for scale s > 0: IEEE quotient, round half to even, clamp.
__device__ __forceinline__ int int8_code(float x, float s) {
  int r = __float2int_rn(__fdiv_rn(x, s));   // cvt.rni: ties to even
  return max(-128, min(127, r));
}

// INT8 code of x for scale s > 0 from rs = 1/s (correctly rounded), equal to
// int8_code(x, s): for |x/s| < 128, q1 = fl(x * rs) is within 2^-16 of the
// exact quotient and the IEEE quotient within 2^-18, so the two lie on the same
// side of every rounding boundary n + 1/2 unless q1 is within 2^-13 of one;
// there the IEEE division decides.  Larger |x/s| clamp either way.
__device__ __forceinline__ int int8_code_recip(float x, float s, float rs) {
  const float q1 = x * rs;
  const float fr = q1 - floorf(q1);
  if (fabsf(q1) < 128.0f && fabsf(fr - 0.5f) > 0x1p-13f)
    return max(-128, min(127, __float2int_rn(q1)));
  return int8_code(x, s);
}

// Two e4m3 codes (lo = x0, hi = x1) for scale s > 0, packed in 16 bits.
__device__ __forceinline__ uint32_t e4m3x2_code(float x0, float x1, float s) {
  float c0 = __fdiv_rn(x0, s), c1 = __fdiv_rn(x1, s);
  unsigned short r;
  // the first source operand lands in the upper byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(c1), "f"(c0));
  return (uint32_t)r;
}

// Four codes packed little-endian (byte i = code of v[i]).
template <int DT>
__device__ __forceinline__ uint32_t pack4_codes(const float v[4], float s) {
  if (s == 0.0f) return 0u;
  if (DT == kInt8) {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) w |= ((uint32_t)(uint8_t)(int8_t)int8_code(v[i], s)) << (8 * i);
    return w;
  } else {
    return e4m3x2_code(v[0], v[1], s) | (e4m3x2_code(v[2], v[3], s) << 16);
  }
}

template <int DT>
__device__ __forceinline__ uint8_t one_code(float v, float s) {
  if (s == 0.0f) return 0;
  if (DT == kInt8) return (uint8_t)(int8_t)int8_code(v, s);
  return (uint8_t)(e4m3x2_code(v, 0.0f, s) & 0xFFu);
}

// Exact fp32 value of an e4m3 code (for the CUDA-core paths): hardware
// e4m3 -> f16 conversion (exact), then f16 -> f32 (exact).
__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  unsigned r;
  unsigned short in = (unsigned short)c;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(in));
  __half_raw hr;
  hr.x = (unsigned short)(r & 0xFFFFu);
  return __half2float(__half(hr));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

// bf16 bits of silu(g) * u, silu(g) = g / (1 + exp(-g)) in fp32 with the
// hardware exp2 and reciprocal (relative error ~1e-6, far below bf16's
// half-ulp of 2^-9), rounded once to bf16.  Both the fused w13 epilogue and
// the stand-alone SiLU kernel use this, so their h are identical.
__device__ __forceinline__ uint16_t silu_mul_bf16(float g, float u) {
  const float sg = __fdividef(g, 1.0f + __expf(-g));
  return float_to_bf16_bits(sg * u);
}

}  // namespace bq
