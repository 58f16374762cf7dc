// gemm_simt.cu -- generic block-scaled GEMM on CUDA cores.
//
// out[m, n] = bf16( sum_kb P_kb[m, n] * sa[kb][m] * sw[nb(n)][kb] + bias[n] )
// (block-wise INT8 page, sections 2 and 4; blockwise FP8 of the SGLang
// quantization doc).  This kernel accepts any M, N, K, block sizes, strides
// and alignments; it is the path for shapes the tensor-core kernels do not
// take (K not a multiple of 16 bytes, odd block sizes, ...).
//
// Tiling: 64 x 64 outputs per CTA, 256 threads, 4 x 4 outputs per thread.
// The K loop walks chunks of at most 32 elements that never straddle a
// K-block; bytes past the chunk are zero-filled in shared memory.  INT8
// partials use dp4a into int32 (exact); FP8 decodes codes to fp32 (exact) and
// accumulates the block partial in fp32.  When a K-block ends, each partial
// is rescaled by sa * sw and added to the fp32 accumulator.
//
// Grouped (MoE) problems: blockIdx.z is the expert; its rows are
// [offsets[e], offsets[e+1]) and CTAs past the expert's rows exit at once.
#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {

namespace {

constexpr int BM = 64, BN = 64, BKC = 32;

__device__ __forceinline__ int64_t wrow_block(int64_t n, int64_t bn, int64_t seam, int64_t N) {
  if (seam <= 0 || seam >= N || n < seam) return n / bn;
  return (seam + bn - 1) / bn + (n - seam) / bn;
}

template <int DT>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(GemmArgs a) {
  // INT8: codes packed 4 per word; FP8: decoded floats.
  __shared__ __align__(16) uint32_t As_i[BM][BKC / 4 + 1];
  __shared__ __align__(16) uint32_t Ws_i[BN][BKC / 4 + 1];
  __shared__ float As_f[DT == kFp8 ? BM : 1][BKC + 1];
  __shared__ float Ws_f[DT == kFp8 ? BN : 1][BKC + 1];

  const int e = blockIdx.z;
  int64_t row0 = 0, rows = a.M;
  if (a.offsets) {
    row0 = a.offsets[e];
    rows = (int64_t)a.offsets[e + 1] - row0;
  }
  const int64_t mt = (int64_t)blockIdx.y * BM;
  if (mt >= rows) return;
  const int64_t nt = (int64_t)blockIdx.x * BN;
  const uint8_t* qa = static_cast<const uint8_t*>(a.qa) + row0 * a.lda;
  const uint8_t* qw = static_cast<const uint8_t*>(a.qw) + (int64_t)e * a.w_expert_stride;
  const float* sw = a.sw + (int64_t)e * a.sw_expert_stride;
  const int64_t Kb = (a.K + a.bk - 1) / a.bk;

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
  int32_t pi[4][4];
  float pf[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) { acc[i][j] = 0.f; pi[i][j] = 0; pf[i][j] = 0.f; }

  for (int64_t kb = 0; kb < Kb; ++kb) {
    const int64_t kb0 = kb * a.bk, kb1 = min(a.K, kb0 + a.bk);
    for (int64_t k0 = kb0; k0 < kb1; k0 += BKC) {
      const int64_t kc = (kb1 - k0 < BKC) ? (kb1 - k0) : (int64_t)BKC;
      __syncthreads();
      // each thread loads 8 bytes of A and 8 of W (64 rows x 32 bytes each)
      for (int idx = threadIdx.x; idx < BM * BKC; idx += 256) {
        const int r = idx / BKC, c = idx % BKC;
        const int64_t gm = mt + r, gn = nt + r;
        uint8_t va = 0, vw = 0;
        if (c < kc && gm < rows) va = qa[gm * a.lda + k0 + c];
        if (c < kc && gn < a.N) vw = qw[gn * a.ldw + k0 + c];
        if constexpr (DT == kInt8) {
          reinterpret_cast<uint8_t*>(&As_i[r][0])[c] = va;
          reinterpret_cast<uint8_t*>(&Ws_i[r][0])[c] = vw;
        } else {
          As_f[r][c] = e4m3_to_float(va);
          Ws_f[r][c] = e4m3_to_float(vw);
        }
      }
      __syncthreads();
      if constexpr (DT == kInt8) {
#pragma unroll
        for (int w = 0; w < BKC / 4; ++w) {
          int av[4], wv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) av[i] = (int)As_i[ty + 16 * i][w];
#pragma unroll
          for (int j = 0; j < 4; ++j) wv[j] = (int)Ws_i[tx + 16 * j][w];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) pi[i][j] = __dp4a(av[i], wv[j], pi[i][j]);
        }
      } else {
        for (int c = 0; c < BKC; ++c) {
          float av[4], wv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) av[i] = As_f[ty + 16 * i][c];
#pragma unroll
          for (int j = 0; j < 4; ++j) wv[j] = Ws_f[tx + 16 * j][c];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) pf[i][j] = fmaf(av[i], wv[j], pf[i][j]);
        }
      }
    }
    // K-block done: promote partials with sa * sw
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t gm = mt + ty + 16 * i;
      const float sav = gm < rows ? a.sa[kb * a.sa_rows + row0 + gm] : 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t gn = nt + tx + 16 * j;
        const float swv =
            gn < a.N ? sw[wrow_block(gn, a.bn, a.seam, a.N) * Kb + kb] : 0.f;
        const float p = (DT == kInt8) ? (float)pi[i][j] : pf[i][j];
        acc[i][j] = fmaf(p * sav, swv, acc[i][j]);
        pi[i][j] = 0;
        pf[i][j] = 0.f;
      }
    }
  }
  uint16_t* out = static_cast<uint16_t*>(a.out) + row0 * a.ldo;
  const uint16_t* bias = static_cast<const uint16_t*>(a.bias);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gm = mt + ty + 16 * i;
    if (gm >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t gn = nt + tx + 16 * j;
      if (gn >= a.N) continue;
      float v = acc[i][j];
      if (a.out_f32) {
        a.out_f32[(row0 + gm) * a.ldo + gn] = v;
        continue;
      }
      if (bias) v += bf16_bits_to_float(bias[gn]);
      out[gm * a.ldo + gn] = float_to_bf16_bits(v);
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmArgs& a, cudaStream_t st) {
  const int64_t max_rows = a.M;  // dense: M; grouped: total rows R (upper bound per expert)
  if (max_rows == 0 || a.N == 0) return cudaSuccess;
  const int64_t gy = (max_rows + BM - 1) / BM, gx = (a.N + BN - 1) / BN;
  if (gy > 65535 || a.E > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid((unsigned)gx, (unsigned)gy, (unsigned)a.E);
  if (a.dtype == kInt8)
    gemm_simt_kernel<kInt8><<<grid, 256, 0, st>>>(a);
  else
    gemm_simt_kernel<kFp8><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace bq
