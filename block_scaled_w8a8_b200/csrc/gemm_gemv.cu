// gemm_gemv.cu -- block-scaled INT8 GEMM for 1..8 tokens on CUDA cores.
//
// out[m, n] = bf16( sum_kb P_kb[m, n] * sa[kb][m] * sw[n/128][kb] + bias[n] )
// (block-wise INT8 page, sections 2 and 4), block_n = block_k = 128.
//
// With a handful of tokens the layer is a weight stream: 16.8 MB of codes
// for N = K = 4096 against at most 8 x 4096 activation bytes.  The
// tensor-core decode kernel needs split-K (too few 128-row weight tiles to
// fill the GPU) and pays TMEM/cluster set-up and a cross-CTA reduction per
// launch; here there is neither:
//  * one warp per weight row over the full K (no split, no cross-CTA
//    reduction), N/8 CTAs of 8 warps so every SM keeps loads in flight;
//  * lane l reads bytes [16 l + 512 c, +16) of the row for c = 0, 1, ...:
//    every load instruction is one contiguous 512-byte run (weights streamed
//    past L1, activation codes shared by all warps through L1), and the
//    first eight chunks (4 KB) are requested up front;
//  * a K-block (128 bytes) spans 8 lanes: each lane forms its exact int32
//    dp4a partial for every token, a butterfly reduce-scatter over the 8
//    lanes (MT-1 shuffles for MT tokens, exact integer sums) leaves each lane
//    holding one token's complete P_kb, which it promotes with
//    sa[kb][m] * sw[n/128][kb];
//  * two more shuffles add the four lane groups (different K-blocks); lanes
//    0..MT-1 add the bias and write bf16;
//  * programmatic dependent launch: the first weight chunks are requested
//    before griddepcontrol.wait, so they overlap the activation quantiser.
#include <algorithm>
#include <cstdio>

#include "bq_common.cuh"
#include "bq_internal.h"
#include "gemm_gemv.h"

namespace bq {

namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ uint4 ldg_stream(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ int dot16(uint4 w, uint4 a, int acc) {
  acc = __dp4a((int)w.x, (int)a.x, acc);
  acc = __dp4a((int)w.y, (int)a.y, acc);
  acc = __dp4a((int)w.z, (int)a.z, acc);
  return __dp4a((int)w.w, (int)a.w, acc);
}

// Butterfly reduce-scatter of MT per-token integer sums over the 8 lanes of
// a group: afterwards v[0] holds, in every lane, the group total of token
// own_token(lane).  Exact (integer adds).
template <int MT>
__device__ __forceinline__ int group_reduce_scatter(int (&v)[MT], int lane) {
  int cnt = MT;
  int tok = 0;
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) {
    if (cnt > 1) {
      const int half = cnt / 2;
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < MT / 2; ++i) {
        if (i < half) {
          const int send = upper ? v[i] : v[i + half];
          const int keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      if (upper) tok += half;
      cnt = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return tok;
}

// MT: token count rounded up to a power of two (1..8).
template <int MT>
__global__ void __launch_bounds__(kWarps * 32)
gemv_kernel(const uint8_t* __restrict__ qa, int64_t lda, const float* __restrict__ sa,
            const uint8_t* __restrict__ qw, int64_t ldw, const float* __restrict__ sw,
            int M, int64_t N, int64_t K, const uint16_t* __restrict__ bias,
            uint16_t* __restrict__ out, int64_t ldo) {
  constexpr int kDepth = 8;                        // 512-byte chunks requested ahead
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t Kb = (K + 127) / 128;
  const int64_t nchunks = (K + 511) / 512;
  const bool row_ok = n < N;
  const uint8_t* wrow = qw + (row_ok ? n : 0) * ldw;
  const float* swrow = sw + ((row_ok ? n : 0) >> 7) * Kb;
  const int g = lane >> 3;                         // K-block within a 512-byte chunk

  // chunks are processed in groups of kDepth: the group's weights (and their
  // block scales) are requested first, then its activation scales in one
  // batch, so no load latency sits inside the dot-product loop
  uint4 w[kDepth];
  float swv[kDepth];
  auto fetch_weights = [&](int64_t c0) {
#pragma unroll
    for (int c = 0; c < kDepth; ++c) {
      const int64_t ci = c0 + c;
      const int64_t k = 512 * ci + 16 * lane;
      const int64_t kb = 4 * ci + g;
      w[c] = (row_ok && ci < nchunks && k < K) ? ldg_stream(wrow + k) : make_uint4(0, 0, 0, 0);
      swv[c] = (row_ok && ci < nchunks && kb < Kb) ? __ldg(swrow + kb) : 0.f;
    }
  };
  fetch_weights(0);
  // weights are independent of the kernel that produced the activation
  // codes: let the next kernel launch, then wait for the codes
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // token owned by this lane after the butterfly (lanes of a group split the
  // tokens by the bits of lane & 7, from bit 2 down)
  int own = 0;
  {
    int cnt = MT;
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) {
      if (cnt > 1) {
        if (lane & o) own += cnt / 2;
        cnt /= 2;
      }
    }
  }
  float acc = 0.f;
  for (int64_t c0 = 0; c0 < nchunks; c0 += kDepth) {
    float sav[kDepth];
#pragma unroll
    for (int c = 0; c < kDepth; ++c) {
      const int64_t kb = 4 * (c0 + c) + g;
      sav[c] = (own < M && c0 + c < nchunks && kb < Kb) ? __ldg(sa + kb * M + own) : 0.f;
    }
#pragma unroll
    for (int c = 0; c < kDepth; ++c) {
      const int64_t ci = c0 + c;
      if (ci < nchunks) {                          // warp-uniform
        const int64_t k = 512 * ci + 16 * lane;
        int P[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          P[m] = 0;
          if (m < M && k < K) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(qa + m * lda + k));
            P[m] = dot16(w[c], a, 0);
          }
        }
        group_reduce_scatter<MT>(P, lane);
        acc = fmaf((float)P[0], sav[c] * swv[c], acc);
      }
    }
    if (c0 + kDepth < nchunks) fetch_weights(c0 + kDepth);
  }
  // add the four lane groups (lanes l, l^8, l^16, l^24 hold the same token)
  acc += __shfl_xor_sync(0xffffffffu, acc, 8);
  acc += __shfl_xor_sync(0xffffffffu, acc, 16);
  if (lane < 8 && row_ok && own < M && (lane & (8 / MT - 1)) == 0) {
    const float b = bias ? bf16_bits_to_float(bias[n]) : 0.f;
    out[(int64_t)own * ldo + n] = float_to_bf16_bits(acc + b);
  }
}

template <int MT>
cudaError_t launch_mt(const GemmArgs& a, bool pdl, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((a.N + kWarps - 1) / kWarps));
  cfg.blockDim = dim3(kWarps * 32);
  cfg.stream = st;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<MT>, static_cast<const uint8_t*>(a.qa), a.lda,
                            a.sa, static_cast<const uint8_t*>(a.qw), a.ldw, a.sw, (int)a.M, a.N,
                            a.K, static_cast<const uint16_t*>(a.bias),
                            static_cast<uint16_t*>(a.out), a.ldo);
}

}  // namespace

bool gemv_supported(const GemmArgs& a, char* why, size_t n) {
  auto no = [&](const char* msg) {
    if (why) snprintf(why, n, "CUDA-core decode path: %s", msg);
    return false;
  };
  if (a.offsets) return no("dense problems only");
  if (a.dtype != kInt8) return no("INT8 only");
  if (a.M > kGemvMaxRows) return no("at most 8 tokens");
  if (a.bn != 128 || a.bk != 128) return no("needs block_n = block_k = 128");
  if (a.K % 16 != 0 || a.lda % 16 != 0 || a.ldw % 16 != 0)
    return no("K and the row strides must be multiples of 16 bytes");
  if ((reinterpret_cast<uintptr_t>(a.qa) & 15) || (reinterpret_cast<uintptr_t>(a.qw) & 15))
    return no("operands must be 16-byte aligned");
  if ((a.N + kWarps - 1) / kWarps > 0x7fffffff) return no("N too large");
  return true;
}

cudaError_t launch_gemm_gemv(const GemmArgs& a, bool pdl, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  if (a.M <= 1) return launch_mt<1>(a, pdl, st);
  if (a.M <= 2) return launch_mt<2>(a, pdl, st);
  if (a.M <= 4) return launch_mt<4>(a, pdl, st);
  return launch_mt<8>(a, pdl, st);
}

}  // namespace bq
