// gemm_mx.cu -- MXFP8 dense linear on the block-scaled tensor cores (sm_100a).
//
// The SGLang quantization doc ("GEMM backends for FP4/FP8") lists an MXFP8
// dense linear next to the blockwise FP8 GEMM.  The format is the
// microscaling one the name refers to: groups of 32 consecutive elements
// along K share a power-of-two scale 2^(E - 127) held as an 8-bit exponent E
// (E8M0), the elements are e4m3 codes, and
//   out[m, n] = bf16( sum_g 2^(Ea[m,g]-127) 2^(Ew[n,g]-127) sum_{k in g} a[m,k] w[n,k] + bias[n] ).
// Unlike the 128 x 128 block-scaled path, the scale is applied inside the
// MMA (tcgen05.mma kind::mxf8f6f4.block_scale), so the whole K accumulates
// in TMEM and the epilogue only converts.
//
// Quantisation (one group): se = clamp(floor(log2 amax) - 8, -127, 127), where
// 8 is the largest exponent of an e4m3 normal; E = se + 127; each element is
// x * 2^-se (exact) converted once to e4m3 with round-to-nearest-even and
// saturation to +-448.  An all-zero group gets E = 0 and zero codes.
//
// Scale-factor layout ("tensor-core layout"), shared by the quantisers, the
// GEMM and the C ABI: rows are cut into blocks of 128 and K into blocks of
// 128 (4 groups); each (row block, K block) pair is one 512-byte atom, atoms
// ordered row block major, K block minor.  Inside an atom, row r and group g
// sit at byte 16 * (r % 32) + 4 * ((r % 128) / 32) + g % 4.  An atom is then
// exactly what one tcgen05.cp.32x128b.warpx4 moves into TMEM: lane r % 32
// of every lane quadrant receives 16 bytes, column (r % 128) / 32, byte g % 4.
//
// GEMM design (persistent, one CTA per SM, 640 threads):
//   warp 0      TMA producer of the A tile (128 x 128 codes) and a bulk copy of
//               its 512-byte scale atom, per K-block;
//   warp 2      TMA producer of the W tile (256 x 128) and its two scale atoms;
//   warp 1      MMA issuer: per K-block, three tcgen05.cp (scale atoms ->
//               TMEM columns of that ring stage) then four block-scaled MMAs
//               (K = 32 each; scale-factor id j selects byte j of each column);
//   warps 4-19  epilogue: once per tile, read the 128 x 256 fp32 accumulator
//               (64 columns per warp), free it, add the bias, store bf16.
// TMEM: columns [0, 256) accumulator; [256 + 16 s, +12) the scale factors of
// ring stage s (4 columns for A, 8 for the 256 rows of W).
//
// Every mbarrier wait is bounded (2 s); on expiry the CTA records a timeout
// in the device status word, drains its in-flight copies and MMAs, frees its
// tensor memory and exits.
#include <cuda.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>

#include "bq_common.cuh"
#include "bq_internal.h"
#include "gemm_mx.h"
#include "gemm_tc_common.cuh"
#include "sm100.cuh"

namespace bq {
namespace {

using namespace sm100;
using tc::make_tmap;
using tc::sm_count;

constexpr int MX_BM = 128, MX_BN = 256, MX_BK = 128, MX_S = 4;
constexpr int kMxThreads = 640;
constexpr int kMxEpiWarps = 16;
constexpr uint32_t kMxA = MX_BM * MX_BK, kMxB = MX_BN * MX_BK;
constexpr uint32_t kAtom = 512;                 // one scale atom: 128 rows x 4 groups
constexpr uint32_t kMxStages = MX_S * (kMxA + kMxB);
constexpr uint32_t kMxSf = MX_S * 3 * kAtom;    // per stage: A atom, two W atoms
constexpr uint32_t kMxBars = (2 * MX_S + 3) * 8;
constexpr uint32_t kMxTotal = 1024 + kMxStages + kMxSf + kMxBars + 16;
constexpr uint32_t kSfCol0 = 256;               // first TMEM column of the scale factors
static_assert(kMxTotal <= 227u * 1024u, "shared memory budget");

struct MxParams {
  const uint8_t* sfa;    // activation scale atoms
  const uint8_t* sfw;    // weight scale atoms
  int64_t M, N, K, Kb;   // Kb = K / 128
  int mblk, nblk;
  const uint16_t* bias;
  uint16_t* out; int64_t ldo;
  unsigned* status;
};

// 1-D bulk copy global -> shared, completing on an mbarrier (16-byte aligned,
// size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Shared-memory descriptor of one scale atom for tcgen05.cp: 32 rows of 16
// bytes, no swizzle, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(kAtom >> 4) << 16;       // leading byte offset (one 16-byte chunk per row)
  d |= (uint64_t)(128u >> 4) << 32;        // stride byte offset: 8 rows x 16 bytes
  d |= (uint64_t)1u << 46;                 // descriptor version for tcgen05
  return d;                                // layout type 0: no swizzle
}

// 32 lanes x 128 bits from shared memory into TMEM, replicated to the four
// lane quadrants.
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Instruction descriptor of the block-scaled MMA: e4m3 x e4m3 -> f32,
// both K-major, M = 128, N = 256, E8M0 scales; scale-factor id j (byte j of
// the scale columns) for both operands.
__device__ __forceinline__ uint32_t mx_idesc(uint32_t j) {
  return (j << 4) |                               // B scale-factor id
         ((uint32_t)(MX_BN >> 3) << 17) |          // N
         (1u << 23) |                              // scale format E8M0
         ((uint32_t)(MX_BM >> 4) << 24) |          // M
         (j << 29);                                // A scale-factor id
}

__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__global__ void __launch_bounds__(kMxThreads, 1)
gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const MxParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + MX_S * kMxA;
  uint8_t* sSf = smem + kMxStages;                 // [stage][A atom, W atom 0, W atom 1]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kMxStages + kMxSf);
  uint64_t* full = bars;
  uint64_t* empty = bars + MX_S;
  uint64_t* tfull = bars + 2 * MX_S;
  uint64_t* tempty = bars + 2 * MX_S + 1;
  uint64_t* drain = bars + 2 * MX_S + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * MX_S + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.mblk * p.nblk;
  const int nrb = (int)((p.N + 127) / 128);        // 128-row blocks of W (scale atoms)

  if (threadIdx.x == 0) {
    for (int s = 0; s < MX_S; ++s) {
      mbar_init(smem_u32(&full[s]), 2);            // the A producer and the W producer
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(&tfull[0]), 1);
    mbar_init(smem_u32(&tempty[0]), kMxEpiWarps);
    mbar_init(smem_u32(&drain[0]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmA);
  if (warp == 2 && lane == 0) tma_prefetch_desc(&tmB);
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == 2) {
    // ---------------- producers ----------------
    const bool is_a = warp == 0;
    int stage = 0;
    uint32_t phase = 0;
    int issued_parity[MX_S];
#pragma unroll
    for (int s = 0; s < MX_S; ++s) issued_parity[s] = -1;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int mb = t % p.mblk, nb = t / p.mblk;  // m-blocks fastest: CTAs share W tiles
      for (int kb = 0; kb < (int)p.Kb; ++kb) {
        if (!warp_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.status, 0x501u)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* sf = sSf + stage * 3 * kAtom;
          const uint32_t bar = smem_u32(&full[stage]);
          if (is_a) {
            mbar_arrive_expect_tx(bar, kMxA + kAtom);
            tma_load_2d(smem_u32(sA + stage * kMxA), &tmA, kb * MX_BK, mb * MX_BM, bar);
            bulk_g2s(smem_u32(sf), p.sfa + ((int64_t)mb * p.Kb + kb) * kAtom, kAtom, bar);
          } else {
            // the second 128-row scale atom exists unless N ends inside this tile
            const bool two = 2 * nb + 1 < nrb;
            mbar_arrive_expect_tx(bar, kMxB + (two ? 2 : 1) * kAtom);
            tma_load_2d(smem_u32(sB + stage * kMxB), &tmB, kb * MX_BK, nb * MX_BN, bar);
            bulk_g2s(smem_u32(sf + kAtom), p.sfw + ((int64_t)(2 * nb) * p.Kb + kb) * kAtom,
                     kAtom, bar);
            if (two)
              bulk_g2s(smem_u32(sf + 2 * kAtom),
                       p.sfw + ((int64_t)(2 * nb + 1) * p.Kb + kb) * kAtom, kAtom, bar);
          }
        }
        issued_parity[stage] = (int)phase;
        if (++stage == MX_S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok) {
      for (int s = 0; s < MX_S; ++s) {
        if (issued_parity[s] < 0) continue;
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(&full[s]), (uint32_t)issued_parity[s]) &&
               globaltimer() - t0 < 100000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    int stage = 0;
    uint32_t phase = 0, tcount = 0;
    bool ok = true, issued_any = false;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      // the single accumulator is free once the epilogue has read the last tile
      if (!warp_wait(smem_u32(&tempty[0]), (tcount & 1) ^ 1, abort_flag, p.status, 0x502u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kb = 0; kb < (int)p.Kb; ++kb) {
        if (!warp_wait(smem_u32(&full[stage]), phase, abort_flag, p.status, 0x503u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sfa_t = tmem_base + kSfCol0 + 16u * (uint32_t)stage;
          const uint32_t sfb_t = sfa_t + 4u;
          const uint32_t sf = smem_u32(sSf + stage * 3 * kAtom);
          tmem_cp_atom(sfa_t, sf_desc(sf));
          tmem_cp_atom(sfb_t, sf_desc(sf + kAtom));
          tmem_cp_atom(sfb_t + 4u, sf_desc(sf + 2 * kAtom));
          const uint64_t a0 = smem_desc_k128(smem_u32(sA + stage * kMxA));
          const uint64_t b0 = smem_desc_k128(smem_u32(sB + stage * kMxB));
#pragma unroll
          for (uint32_t j = 0; j < MX_BK / 32; ++j)
            mma_mx(tmem_base, a0 + 2ull * j, b0 + 2ull * j, mx_idesc(j), sfa_t | (j << 30),
                   sfb_t | (j << 30), (kb > 0 || j > 0) ? 1u : 0u);
          mma_commit(smem_u32(&empty[stage]));
          if (kb == (int)p.Kb - 1) mma_commit(smem_u32(&tfull[0]));
        }
        __syncwarp();
        issued_any = true;
        if (++stage == MX_S) {
          stage = 0;
          phase ^= 1;
        }
      }
      ++tcount;
    }
    if (!ok && issued_any) {
      if (lane == 0) mma_commit(smem_u32(&drain[0]));
      __syncwarp();
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(&drain[0]), 0) && globaltimer() - t0 < 100000000ull) {
      }
    }
  } else if (warp >= 4) {
    // ---------------- epilogue ----------------
    constexpr int CW = MX_BN / 4;                  // 64 columns per warp
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int rit = 32 * q + lane;
    const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(CW * half);
    uint32_t tcount = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const int mb = t % p.mblk, nb = t / p.mblk;
      if (!warp_wait(smem_u32(&tfull[0]), tcount & 1, abort_flag, p.status, 0x504u)) break;
      tc_fence_after();
      float v[CW];
#pragma unroll
      for (int c = 0; c < CW / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(taddr + 16u * c, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 * c + i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[0]));   // accumulator free for the MMA
      ++tcount;
      const int64_t m = (int64_t)mb * MX_BM + rit;
      const int64_t n0 = (int64_t)nb * MX_BN + CW * half;
      if (m >= p.M || n0 >= p.N) continue;
      uint16_t* orow = p.out + m * p.ldo + n0;
      const bool vec = n0 + CW <= p.N && ((reinterpret_cast<uintptr_t>(orow) & 15) == 0);
      if (vec) {
#pragma unroll
        for (int j = 0; j < CW; j += 8) {
          uint32_t w[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            float v0 = v[j + 2 * h], v1 = v[j + 2 * h + 1];
            if (p.bias) {
              v0 += bf16_bits_to_float(__ldg(p.bias + n0 + j + 2 * h));
              v1 += bf16_bits_to_float(__ldg(p.bias + n0 + j + 2 * h + 1));
            }
            w[h] = (uint32_t)float_to_bf16_bits(v0) | ((uint32_t)float_to_bf16_bits(v1) << 16);
          }
          *reinterpret_cast<uint4*>(orow + j) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          if (n0 + j < p.N) {
            float x = v[j];
            if (p.bias) x += bf16_bits_to_float(__ldg(p.bias + n0 + j));
            orow[j] = float_to_bf16_bits(x);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------- MX quantisation ----------------

// A warp quantises a chunk of 256 consecutive elements of a row (8 groups of
// 32, or the last 128 of a row); lane l holds elements 8l .. 8l + 7, so
// lanes 4g .. 4g + 3 form group g.  Each warp keeps two chunks in flight.
template <typename T>
__device__ __forceinline__ void mx_load8(const T* __restrict__ src, bool vec, bool valid,
                                         float (&v)[8]) {
  if (!valid) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    return;
  }
  if constexpr (sizeof(T) == 2) {
    if (vec) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = bf16_bits_to_float(src[i]);
    }
  } else {
    if (vec) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(src));
      const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = src[i];
    }
  }
}

__device__ __forceinline__ void mx_finish8(const float (&v)[8], int64_t r, int64_t k0, bool valid,
                                           int64_t K, uint8_t* __restrict__ q, int64_t ldq,
                                           uint8_t* __restrict__ sf, int lane) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  if (!valid) return;
  // floor(log2 amax) is the unbiased exponent of a normal amax; a zero or
  // subnormal amax clamps to the smallest scale
  const int ef = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
  const int se = (ef == 0) ? -127 : max(-127, min(127, ef - 127 - 8));
  const float inv = __uint_as_float((uint32_t)(127 - se) << 23);   // 2^-se, exact
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    unsigned short lo, hi;
    // the first source operand lands in the upper byte
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
        : "=h"(lo) : "f"(v[4 * h + 1] * inv), "f"(v[4 * h] * inv));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
        : "=h"(hi) : "f"(v[4 * h + 3] * inv), "f"(v[4 * h + 2] * inv));
    w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  uint32_t* dst = reinterpret_cast<uint32_t*>(q + r * ldq + k0);
  dst[0] = w[0];
  dst[1] = w[1];
  if ((lane & 3) == 0) {
    const int64_t gk = k0 / 32;                       // group index in the row
    const int64_t atom = (r / 128) * (K / 128) + gk / 4;
    sf[atom * kAtom + 16 * (r % 32) + 4 * ((r % 128) / 32) + gk % 4] = (uint8_t)(se + 127);
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
mx_quant_kernel(const T* __restrict__ x, int64_t R, int64_t K, int64_t ldx, bool vec,
                uint8_t* __restrict__ q, int64_t ldq, uint8_t* __restrict__ sf) {
  const int64_t kc = (K + 255) / 256;                 // chunks per row
  const int64_t total = R * kc;
  const int lane = threadIdx.x & 31;
  const int64_t nw = (int64_t)gridDim.x * 8;
  for (int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); w < total; w += 2 * nw) {
    const int64_t w2 = w + nw;
    const int64_t r = w / kc, k0 = (w - r * kc) * 256 + 8 * lane;
    const bool ok0 = k0 < K;
    float a[8], b[8];
    mx_load8(x + r * ldx + k0, vec, ok0, a);
    int64_t r2 = 0, k2 = 0;
    bool ok1 = false;
    if (w2 < total) {
      r2 = w2 / kc;
      k2 = (w2 - r2 * kc) * 256 + 8 * lane;
      ok1 = k2 < K;
      mx_load8(x + r2 * ldx + k2, vec, ok1, b);
    }
    mx_finish8(a, r, k0, ok0, K, q, ldq, sf, lane);
    if (w2 < total) mx_finish8(b, r2, k2, ok1, K, q, ldq, sf, lane);
  }
}

template <typename T>
cudaError_t launch_mx_quant_t(const T* x, int64_t R, int64_t K, int64_t ldx, void* q,
                              int64_t ldq, void* sf, cudaStream_t st) {
  const int64_t warps = R * ((K + 255) / 256);
  if (warps == 0) return cudaSuccess;
  const bool vec = ldx % 8 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0;
  const int64_t blocks = std::min<int64_t>((warps + 7) / 8, (int64_t)sm_count() * 8);
  mx_quant_kernel<T><<<(unsigned)blocks, 256, 0, st>>>(x, R, K, ldx, vec,
                                                        static_cast<uint8_t*>(q), ldq,
                                                        static_cast<uint8_t*>(sf));
  return cudaGetLastError();
}

}  // namespace

size_t mx_scale_bytes(int64_t R, int64_t K) {
  return (size_t)((R + 127) / 128) * (size_t)(K / 128) * kAtom;
}

cudaError_t launch_mx_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, void* q,
                                int64_t ldq, void* sf, cudaStream_t st) {
  return launch_mx_quant_t(static_cast<const uint16_t*>(x), M, K, ldx, q, ldq, sf, st);
}

cudaError_t launch_mx_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw, void* q,
                                   int64_t ldq, void* sf, cudaStream_t st) {
  return launch_mx_quant_t(w, N, K, ldw, q, ldq, sf, st);
}

cudaError_t launch_gemm_mx(const MxArgs& a, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_mx_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kMxTotal);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tA, tB;
  if (!make_tmap(&tA, a.qa, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.lda, MX_BM) ||
      !make_tmap(&tB, a.qw, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.ldw, MX_BN))
    return cudaErrorInvalidValue;
  MxParams p;
  p.sfa = static_cast<const uint8_t*>(a.sfa);
  p.sfw = static_cast<const uint8_t*>(a.sfw);
  p.M = a.M; p.N = a.N; p.K = a.K; p.Kb = a.K / MX_BK;
  p.mblk = (int)((a.M + MX_BM - 1) / MX_BM);
  p.nblk = (int)((a.N + MX_BN - 1) / MX_BN);
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.out = static_cast<uint16_t*>(a.out); p.ldo = a.ldo;
  p.status = a.status;
  const int64_t tiles = (int64_t)p.mblk * p.nblk;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, sm_count()));
  gemm_mx_kernel<<<grid, kMxThreads, kMxTotal, st>>>(tA, tB, p);
  return cudaGetLastError();
}

}  // namespace bq
