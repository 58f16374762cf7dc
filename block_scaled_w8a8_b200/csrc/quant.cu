// quant.cu -- activation and weight quantisation kernels.
//
// Activation quantisation (block-wise INT8 page, section 4: the activation
// scale is computed at run time, per token, inside the kernel): each 1 x
// group_k group of a row gets s = amax / Q and codes q = code(x / s).
// Many rows with 128-element groups on 16-byte-aligned data: a half warp per
// group, two groups per warp instruction and several in flight per warp
// (quant_g128_kernel, bandwidth-bound).  Otherwise one warp per group; for
// group_k <= 128 every lane holds its (up to) four elements in registers,
// loaded as one 8-byte vector when aligned, and the amax is a 5-step shuffle
// reduction.  Consecutive warps take consecutive rows of the same K-block so
// the K-block-major scale stores coalesce.
//
// Weight quantisation (structure diagram and section 2): one CTA per
// [bn, bk] block; amax by a block reduction, then codes.
#include <algorithm>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {

namespace {

constexpr int kWarpsPerCta = 8;

// Loads the (up to 4) elements [k0, k0+4) of a row restricted to [0, L).
__device__ __forceinline__ void load4(const uint16_t* row, int64_t k0, int64_t L, bool vec,
                                      float v[4]) {
  if (vec && k0 + 4 <= L) {
    uint2 u = *reinterpret_cast<const uint2*>(row + k0);
    v[0] = bf16_bits_to_float((uint16_t)(u.x & 0xFFFFu));
    v[1] = bf16_bits_to_float((uint16_t)(u.x >> 16));
    v[2] = bf16_bits_to_float((uint16_t)(u.y & 0xFFFFu));
    v[3] = bf16_bits_to_float((uint16_t)(u.y >> 16));
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (k0 + i < L) ? bf16_bits_to_float(row[k0 + i]) : 0.0f;
  }
}

__device__ __forceinline__ void store4(uint8_t* row, int64_t k0, int64_t L, bool vec,
                                       uint32_t w) {
  if (vec && k0 + 4 <= L) {
    *reinterpret_cast<uint32_t*>(row + k0) = w;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (k0 + i < L) row[k0 + i] = (uint8_t)(w >> (8 * i));
  }
}

// Source of the elements of one group: either a bf16 row, or (SILU) the
// gate/up halves of a bf16 row combined as bf16(silu(g) * u).
template <bool SILU>
struct RowSource {
  const uint16_t* row;   // start of the group (gate half for SILU)
  const uint16_t* up;    // SILU only: start of the group in the up half
  uint16_t* h_out;       // SILU only: optional bf16 copy of h
  bool vec;
  __device__ __forceinline__ void get4(int64_t k0, int64_t L, float v[4]) const {
    if (!SILU) {
      load4(row, k0, L, vec, v);
    } else {
      float g[4], u[4];
      load4(row, k0, L, vec, g);
      load4(up, k0, L, vec, u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint16_t hb = silu_mul_bf16(g[i], u[i]);
        v[i] = (k0 + i < L) ? bf16_bits_to_float(hb) : 0.0f;
      }
      if (h_out) {
        if (vec && k0 + 4 <= L) {
          uint2 w;
          w.x = (uint32_t)float_to_bf16_bits(v[0]) | ((uint32_t)float_to_bf16_bits(v[1]) << 16);
          w.y = (uint32_t)float_to_bf16_bits(v[2]) | ((uint32_t)float_to_bf16_bits(v[3]) << 16);
          *reinterpret_cast<uint2*>(h_out + k0) = w;
        } else {
          for (int i = 0; i < 4; ++i)
            if (k0 + i < L) h_out[k0 + i] = float_to_bf16_bits(v[i]);
        }
      }
    }
  }
};

// One warp quantises one group.  Groups of <= 128 elements stay in
// registers (one read); longer groups are read twice (amax, then codes).
template <int DT, bool SILU>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
quant_rows_kernel(const uint16_t* __restrict__ x, int64_t M_out, int64_t K, int64_t ldx,
                  const int32_t* __restrict__ perm, int64_t topk, int64_t gk, int64_t I_half,
                  uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ s,
                  uint16_t* __restrict__ h_out, bool vec_in, bool vec_out) {
  // Programmatic dependent launch: let the next kernel (a GEMM that streams
  // its weights first) be scheduled now, then wait until the kernel before
  // this one has finished and its writes are visible before touching memory.
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t Kb = (K + gk - 1) / gk;
  const int64_t n_groups = M_out * Kb;
  const int64_t warp0 = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int64_t wstride = (int64_t)gridDim.x * kWarpsPerCta;
  for (int64_t w = warp0; w < n_groups; w += wstride) {
    const int64_t g = w / M_out, m = w - g * M_out;
    const int64_t src = perm ? (int64_t)perm[m] / topk : m;
    const int64_t k0 = g * gk;
    const int64_t L = min(gk, K - k0);
    RowSource<SILU> srcrow;
    srcrow.row = x + src * ldx + k0;
    srcrow.up = SILU ? x + src * ldx + I_half + k0 : nullptr;
    srcrow.h_out = (SILU && h_out) ? h_out + m * K + k0 : nullptr;
    srcrow.vec = vec_in;
    uint8_t* qrow = q + m * ldq + k0;
    if (gk <= 128) {
      float v[4];
      srcrow.get4(4 * lane, L, v);
      float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
      amax = warp_max(amax);
      const float sc = group_scale<DT>(amax);
      if (4 * lane < L) store4(qrow, 4 * lane, L, vec_out, pack4_codes<DT>(v, sc));
      if (lane == 0) s[g * M_out + m] = sc;
    } else {
      float amax = 0.0f;
      for (int64_t k = 4 * lane; k < L; k += 128) {
        float v[4];
        if (SILU) {
          // h is only materialised in the second pass
          RowSource<SILU> tmp = srcrow;
          tmp.h_out = nullptr;
          tmp.get4(k, L, v);
        } else {
          srcrow.get4(k, L, v);
        }
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
      }
      amax = warp_max(amax);
      const float sc = group_scale<DT>(amax);
      for (int64_t k = 4 * lane; k < L; k += 128) {
        float v[4];
        srcrow.get4(k, L, v);
        store4(qrow, k, L, vec_out, pack4_codes<DT>(v, sc));
      }
      if (lane == 0) s[g * M_out + m] = sc;
    }
  }
}

// Fast path for 128-element groups on 16-byte-aligned rows (K a multiple of
// 8): a half warp per group, 8 elements per lane from one 16-byte load per
// source row, so one warp instruction covers two groups; each warp issues the
// loads of kPairs group pairs before reducing any of them, keeping several
// loads in flight per warp.  Same arithmetic, element for element, as
// quant_rows_kernel: amax over the group, s = amax / Q, codes of x / s, and
// for SILU h = bf16(silu(g) * u) first.
template <int DT, bool SILU>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
quant_g128_kernel(const uint16_t* __restrict__ x, int64_t M_out, int64_t K, int64_t ldx,
                  const int32_t* __restrict__ perm, int64_t topk, int64_t I_half,
                  uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ s,
                  uint16_t* __restrict__ h_out) {
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kPairs = 2;
  const int lane = threadIdx.x & 31, half = lane >> 4, hl = lane & 15;
  const int64_t Kb = (K + 127) / 128;
  const int64_t n_groups = M_out * Kb;
  const int64_t n_pairs = (n_groups + 1) / 2;
  const int64_t warp0 = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int64_t wstride = (int64_t)gridDim.x * kWarpsPerCta;
  for (int64_t p0 = warp0 * kPairs; p0 < n_pairs; p0 += wstride * kPairs) {
    uint4 a[kPairs], b[kPairs];
    int64_t gm[kPairs], gkb[kPairs];
    bool act[kPairs];                      // this lane's 8 elements exist
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
      const int64_t g = 2 * (p0 + j) + half;
      const bool gv = (p0 + j) < n_pairs && g < n_groups;
      const int64_t kb = gv ? g / M_out : 0, m = gv ? g - kb * M_out : 0;
      const int64_t k = kb * 128 + 8 * hl;
      gm[j] = m;
      gkb[j] = gv ? kb : -1;
      act[j] = gv && k < K;
      a[j] = make_uint4(0u, 0u, 0u, 0u);
      b[j] = make_uint4(0u, 0u, 0u, 0u);
      if (act[j]) {
        const int64_t src = perm ? (int64_t)perm[m] / topk : m;
        const uint16_t* row = x + src * ldx;
        a[j] = __ldg(reinterpret_cast<const uint4*>(row + k));
        if (SILU) b[j] = __ldg(reinterpret_cast<const uint4*>(row + I_half + k));
      }
    }
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
      const uint32_t wa[4] = {a[j].x, a[j].y, a[j].z, a[j].w};
      float v[8];
      if (!SILU) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[2 * e] = __uint_as_float(wa[e] << 16);
          v[2 * e + 1] = __uint_as_float(wa[e] & 0xFFFF0000u);
        }
      } else {
        const uint32_t wb[4] = {b[j].x, b[j].y, b[j].z, b[j].w};
        uint32_t hw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint16_t hb[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float g = __uint_as_float(h ? (wa[e] & 0xFFFF0000u) : (wa[e] << 16));
            const float u = __uint_as_float(h ? (wb[e] & 0xFFFF0000u) : (wb[e] << 16));
            hb[h] = silu_mul_bf16(g, u);
            v[2 * e + h] = act[j] ? bf16_bits_to_float(hb[h]) : 0.0f;
          }
          hw[e] = (uint32_t)hb[0] | ((uint32_t)hb[1] << 16);
        }
        if (h_out && act[j])
          *reinterpret_cast<uint4*>(h_out + gm[j] * K + gkb[j] * 128 + 8 * hl) =
              make_uint4(hw[0], hw[1], hw[2], hw[3]);
      }
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float sc = group_scale<DT>(amax);
      if (act[j]) {
        const uint32_t c0 = pack4_codes<DT>(v, sc), c1 = pack4_codes<DT>(v + 4, sc);
        *reinterpret_cast<uint2*>(q + gm[j] * ldq + gkb[j] * 128 + 8 * hl) = make_uint2(c0, c1);
      }
      if (gkb[j] >= 0 && hl == 0) s[gkb[j] * M_out + gm[j]] = sc;
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(256)
quant_weight_kernel(const float* __restrict__ w, int64_t N, int64_t K, int64_t ldw, int64_t bn,
                    int64_t bk, uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ s) {
  __shared__ float red[8];
  const int64_t Kb = (K + bk - 1) / bk;
  const int64_t i = blockIdx.y, j = blockIdx.x;
  const int64_t n0 = i * bn, k0 = j * bk;
  const int64_t Ln = min(bn, N - n0), Lk = min(bk, K - k0);
  const int64_t cnt = Ln * Lk;
  float amax = 0.0f;
  for (int64_t e = threadIdx.x; e < cnt; e += blockDim.x) {
    int64_t r = e / Lk, c = e - r * Lk;
    amax = fmaxf(amax, fabsf(w[(n0 + r) * ldw + k0 + c]));
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
    v = warp_max(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float sc = group_scale<DT>(red[0]);
  for (int64_t e = threadIdx.x; e < cnt; e += blockDim.x) {
    int64_t r = e / Lk, c = e - r * Lk;
    q[(n0 + r) * ldq + k0 + c] = one_code<DT>(w[(n0 + r) * ldw + k0 + c], sc);
  }
  if (threadIdx.x == 0) s[i * Kb + j] = sc;
  // the decode kernels read weights before their dependency wait: make
  // these codes visible GPU-wide before this CTA exits
  __threadfence();
}

inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int grid_for_groups(int64_t n_groups) {
  int64_t ctas = (n_groups + kWarpsPerCta - 1) / kWarpsPerCta;
  const int64_t cap = 148 * 16;  // persistent-style cap: 16 CTAs per SM
  return (int)std::max<int64_t>(1, std::min<int64_t>(ctas, cap));
}

}  // namespace

cudaError_t launch_quant_act(const void* x, int64_t M_out, int64_t K, int64_t ldx,
                             const int32_t* perm, int64_t topk, int64_t group_k, int dtype,
                             void* q, int64_t ldq, float* s, cudaStream_t st) {
  if (M_out == 0 || K == 0) return cudaSuccess;
  const int64_t Kb = (K + group_k - 1) / group_k;
  const bool vec_in = aligned(x, 8) && ldx % 4 == 0 && group_k % 4 == 0;
  const bool vec_out = aligned(q, 4) && ldq % 4 == 0 && group_k % 4 == 0;
  auto xs = static_cast<const uint16_t*>(x);
  auto qs = static_cast<uint8_t*>(q);
  // the four-groups-per-warp path pays off for bandwidth (many rows); a few
  // tokens (decode) want the most warps in flight for latency instead
  const bool g128 = M_out >= 128 && group_k == 128 && K % 8 == 0 && aligned(x, 16) &&
                    ldx % 8 == 0 && aligned(q, 8) && ldq % 8 == 0;
  const int grid = g128 ? grid_for_groups((M_out * Kb + 3) / 4) : grid_for_groups(M_out * Kb);
  // launched as a programmatic dependent of the preceding kernel: it waits on
  // the GPU (griddepcontrol.wait) before reading or writing any memory, so
  // only its launch latency overlaps the predecessor
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kWarpsPerCta * 32);
  cfg.stream = st;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  if (g128) {
    if (dtype == kInt8)
      return cudaLaunchKernelEx(&cfg, quant_g128_kernel<kInt8, false>, xs, M_out, K, ldx, perm,
                                topk, (int64_t)0, qs, ldq, s, (uint16_t*)nullptr);
    return cudaLaunchKernelEx(&cfg, quant_g128_kernel<kFp8, false>, xs, M_out, K, ldx, perm,
                              topk, (int64_t)0, qs, ldq, s, (uint16_t*)nullptr);
  }
  if (dtype == kInt8)
    return cudaLaunchKernelEx(&cfg, quant_rows_kernel<kInt8, false>, xs, M_out, K, ldx, perm,
                              topk, group_k, (int64_t)0, qs, ldq, s, (uint16_t*)nullptr, vec_in,
                              vec_out);
  return cudaLaunchKernelEx(&cfg, quant_rows_kernel<kFp8, false>, xs, M_out, K, ldx, perm, topk,
                            group_k, (int64_t)0, qs, ldq, s, (uint16_t*)nullptr, vec_in,
                            vec_out);
}

cudaError_t launch_silu_mul_quant(const void* y, int64_t ldy, int64_t R, int64_t I,
                                  int64_t group_k, int dtype, void* q, int64_t ldq, float* s,
                                  void* h_out, cudaStream_t st) {
  if (R == 0 || I == 0) return cudaSuccess;
  const int64_t Kb = (I + group_k - 1) / group_k;
  const bool vec_in = aligned(y, 8) && ldy % 4 == 0 && group_k % 4 == 0 && I % 4 == 0 &&
                      (h_out == nullptr || aligned(h_out, 8));
  const bool vec_out = aligned(q, 4) && ldq % 4 == 0 && group_k % 4 == 0;
  auto ys = static_cast<const uint16_t*>(y);
  auto qs = static_cast<uint8_t*>(q);
  auto hs = static_cast<uint16_t*>(h_out);
  const bool g128 = R >= 128 && group_k == 128 && I % 8 == 0 && aligned(y, 16) &&
                    ldy % 8 == 0 && aligned(q, 8) && ldq % 8 == 0 &&
                    (h_out == nullptr || aligned(h_out, 16));
  if (g128) {
    const int grid = grid_for_groups((R * Kb + 3) / 4);
    if (dtype == kInt8)
      quant_g128_kernel<kInt8, true><<<grid, kWarpsPerCta * 32, 0, st>>>(
          ys, R, I, ldy, nullptr, 1, I, qs, ldq, s, hs);
    else
      quant_g128_kernel<kFp8, true><<<grid, kWarpsPerCta * 32, 0, st>>>(
          ys, R, I, ldy, nullptr, 1, I, qs, ldq, s, hs);
    return cudaGetLastError();
  }
  const int grid = grid_for_groups(R * Kb);
  if (dtype == kInt8)
    quant_rows_kernel<kInt8, true><<<grid, kWarpsPerCta * 32, 0, st>>>(
        ys, R, I, ldy, nullptr, 1, group_k, I, qs, ldq, s, hs, vec_in, vec_out);
  else
    quant_rows_kernel<kFp8, true><<<grid, kWarpsPerCta * 32, 0, st>>>(
        ys, R, I, ldy, nullptr, 1, group_k, I, qs, ldq, s, hs, vec_in, vec_out);
  return cudaGetLastError();
}

cudaError_t launch_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw,
                                int64_t bn, int64_t bk, int dtype, void* q, int64_t ldq,
                                float* s, cudaStream_t st) {
  if (N == 0 || K == 0) return cudaSuccess;
  const int64_t Nb = (N + bn - 1) / bn, Kb = (K + bk - 1) / bk;
  if (Nb > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid((unsigned)Kb, (unsigned)Nb);
  auto qs = static_cast<uint8_t*>(q);
  if (dtype == kInt8)
    quant_weight_kernel<kInt8><<<grid, 256, 0, st>>>(w, N, K, ldw, bn, bk, qs, ldq, s);
  else
    quant_weight_kernel<kFp8><<<grid, 256, 0, st>>>(w, N, K, ldw, bn, bk, qs, ldq, s);
  return cudaGetLastError();
}

}  // namespace bq
