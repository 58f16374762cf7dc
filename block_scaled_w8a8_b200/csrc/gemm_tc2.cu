// gemm_tc2.cu -- block-scaled GEMM on CTA pairs (tcgen05 cta_group::2), sm_100a.
//
// out[m, n] = bf16( sum_kb P_kb[m, n] * sa[kb][m] * sw[nb(n)][kb] + bias[n] )
// (block-wise INT8 page, sections 2 and 4; blockwise FP8 of the SGLang
// quantization doc), for block_n = block_k = 128.
//
// Why pairs: with one CTA per 128x128 tile each K-block of 128 needs 32 KB
// of operands from L2 per 2 M MACs, and measured on B200 that feed (about
// 8 TB/s of L2 -> shared memory traffic, ~3 us load latency under load)
// caps the tensor pipe at ~30%.  A pair of CTAs on two SMs computes a
// 256 x TN tile (TN = 128 or 256): each CTA stages its own 128 rows of A and
// TN/2 rows of W per K-block, and the pair MMA (M = 256, N = TN) uses both
// CTAs' operands, so the L2 traffic per output drops to 3/4 (TN = 128) or
// 1/2 (TN = 256) of the single-CTA kernel's.
//
// Roles (persistent; one pair per two SMs; 19 warps per CTA):
//   warps 0, 18 TMA producers of each CTA: warp 0 its A rows [128r, 128r+128)
//               and warp 18 its W rows [TN/2 r, TN/2 (r+1)) of the pair tile,
//               into an 8- or 6-stage ring; completion is counted on the
//               LEADER CTA's stage barrier (cta_group::2 loads, no multicast).
//   warp 1      leader: issues the pair MMAs (4 x K = 32 per K-block) into one
//               of 512/TN TMEM buffers of TN columns and commits to the stage
//               and TMEM barriers of both CTAs at once; both CTAs' warp 1 own
//               the pair's TMEM allocation (all 512 columns).
//   warps 2-17  epilogue of each CTA: warp w reads TMEM lanes 32*(w%4).. of
//               its own CTA (one output row per thread) and TN/4 columns
//               (w-2)/4; per K-block it promotes acc += P_kb * sa * sw in fp32
//               (INT8: exact int->float by the 1.5 * 2^23 offset trick on the
//               ALU and FMA pipes; scalar FADD/FFMA), releases the buffer to
//               the leader, and
//               after the last K-block adds the bias and stores bf16.
// The tile scheduler is the one of the single-CTA kernel with 256-row tiles:
// dense problems are one expert, grouped (MoE) problems read their expert
// row ranges from device memory.  Rows of a tile past the expert's range are
// computed but never stored.
//
// Every wait is bounded (2 s).  On expiry the CTA records a timeout, the
// leader drains the loads counted on its barriers and the issued MMAs, both
// CTAs meet at a final cluster barrier, and the pair frees its TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstdio>

#include "bq_common.cuh"
#include "bq_internal.h"
#include "gemm_tc.h"
#include "gemm_tc_common.cuh"
#include "sm100.cuh"

namespace bq {

namespace {

using namespace sm100;
using tc::BK;
using tc::kMaxE;
using tc::kMagic;
using tc::kMagicBits;
using tc::TcParams;

constexpr int TM = 256;            // pair tile rows (128 per CTA)
constexpr int kThreads = 608;      // 19 warps: A producer, MMA, 16 epilogue, W producer
constexpr int kWProducerWarp = 18;
constexpr int kEpiWarps = 16;

// Pair tile of 256 x TN: each CTA stages 128 rows of A and TN/2 rows of W
// per K-block; TMEM holds NBUF buffers of TN columns (NBUF * TN = 512).
template <int TN>
struct Pair {
  static constexpr int kNBuf = 512 / TN;
  static constexpr int kStages = TN == 128 ? 8 : 6;
  static constexpr int kEpiCols = TN / 4;                      // per epilogue warp
  static constexpr uint32_t kA = 128 * BK, kB = (TN / 2) * BK;  // per CTA per stage
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kRing = kStages * kStage;
  static constexpr uint32_t kBars = (2 * kStages + 2 * kNBuf + 1) * 8;
  static constexpr uint32_t kMisc = 16 + 2 * (kMaxE + 1) * 4;
  static constexpr uint32_t kTotal = 1024 + kRing + kBars + kMisc;
};

template <int DT, int TN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const TcParams p) {
  using L = Pair<TN>;
  constexpr int kStages = L::kStages, kNBuf = L::kNBuf, kEpiCols = L::kEpiCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                          // stage s: sA + s * kStage
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kRing);
  uint64_t* full = bars;                       // leader: loads of both CTAs
  uint64_t* empty = bars + kStages;            // each CTA: stage consumed by the MMA
  uint64_t* tfull = bars + 2 * kStages;        // each CTA: TMEM buffer holds a partial
  uint64_t* tempty = tfull + kNBuf;            // leader: both CTAs drained a buffer
  uint64_t* drain = tempty + kNBuf;            // leader: issued MMAs finished (abort)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* off_s = reinterpret_cast<int*>(tmem_slot + 4);
  int* tp_s = off_s + (kMaxE + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();        // 0 = leader, 1 = peer
  const int E = p.E;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < kNBuf; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(&drain[0]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmA);
  if (warp == kWProducerWarp && lane == 0) tma_prefetch_desc(&tmB);
  if (threadIdx.x == 32) tc::load_expert_ranges<TM>(p, off_s, tp_s);
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), 512);
  // both CTAs' barriers exist before any load or commit can signal them
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tp_s[E];
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  bool leader_drain = false;
  int issued_parity[kStages];
#pragma unroll
  for (int s = 0; s < kStages; ++s) issued_parity[s] = -1;

  if (warp == 0 || warp == kWProducerWarp) {
    // ---------------- TMA producers (both CTAs): warp 0 the A rows, warp 18
    // the W rows (one issuing thread alone cannot sustain the L2 -> shared
    // memory rate a K-block needs) ----------------
    const bool is_a = warp == 0;
    const uint32_t leader_full0 = mapa_shared(smem_u32(&full[0]), 0);
    int stage = 0;
    uint32_t phase = 0;
    int e_hint = 0;
    bool ok = true;
    for (int t = pair; t < total && ok; t += npairs) {
      int e, mb, nb;
      tc::decode_tile<TM>(t, tp_s, off_s, E, e_hint, e, mb, nb);
      const int a_row = off_s[e] + mb * TM + 128 * (int)rank;
      const int b_row = e * (int)p.N + nb * TN + (TN / 2) * (int)rank;
      for (int kb = 0; kb < p.Kb; ++kb) {
        if (!warp_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.status, 0x501u)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          // the leader expects the bytes of both CTAs on its stage barrier
          if (rank == 0 && is_a) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * L::kStage);
          const uint32_t bar = leader_full0 + 8u * (uint32_t)stage;
          uint8_t* st = sA + stage * L::kStage;
          if (is_a) tma_load_2d_pair(smem_u32(st), &tmA, kb * BK, a_row, bar);
          else tma_load_2d_pair(smem_u32(st + L::kA), &tmB, kb * BK, b_row, bar);
        }
        issued_parity[stage] = (int)phase;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (is_a) leader_drain = !ok;
  } else if (warp == 1) {
    // ---------------- pair MMA issuer (leader only) ----------------
    if (rank == 0) {
      constexpr uint32_t idesc = instr_desc<DT>(TM, TN);
      int stage = 0;
      uint32_t phase = 0, kcount = 0;
      bool ok = true, issued_any = false;
      for (int t = pair; t < total && ok; t += npairs) {
        for (int kb = 0; kb < p.Kb; ++kb) {
          const uint32_t buf = kcount % kNBuf, tround = kcount / kNBuf;
          if (!warp_wait(smem_u32(&tempty[buf]), (tround & 1) ^ 1, abort_flag, p.status,
                         0x502u) ||
              !warp_wait(smem_u32(&full[stage]), phase, abort_flag, p.status, 0x503u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t d = tmem_base + buf * TN;
            const uint64_t a0 = smem_desc_k128(smem_u32(sA + stage * L::kStage));
            const uint64_t b0 = smem_desc_k128(smem_u32(sA + stage * L::kStage + L::kA));
#pragma unroll
            for (int j = 0; j < BK / 32; ++j)
              mma_pair<DT>(d, a0 + (uint64_t)(2 * j), b0 + (uint64_t)(2 * j), idesc,
                           j > 0 ? 1u : 0u);
            mma_commit_pair(smem_u32(&empty[stage]), (uint16_t)0x3);
            mma_commit_pair(smem_u32(&tfull[buf]), (uint16_t)0x3);
          }
          __syncwarp();
          issued_any = true;
          ++kcount;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && issued_any) {
        if (lane == 0) mma_commit_pair(smem_u32(&drain[0]), (uint16_t)0x1);
        __syncwarp();
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(&drain[0]), 0) && globaltimer() - t0 < 100000000ull) {
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..17 of both CTAs) ----------------
    const int q = warp & 3;                       // TMEM lane quadrant of this warp
    const int g = (warp - 2) >> 2;                // 64-column group
    const int rit = 32 * q + lane;                // row inside this CTA's 128 rows
    const uint32_t tcol = (uint32_t)(kEpiCols * g);
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    uint32_t kcount = 0;
    int e_hint = 0;
    bool ok = true;
    for (int t = pair; t < total && ok; t += npairs) {
      int e, mb, nb;
      tc::decode_tile<TM>(t, tp_s, off_s, E, e_hint, e, mb, nb);
      const int row0 = off_s[e] + mb * TM + 128 * (int)rank;
      const int64_t m = (int64_t)row0 + rit;
      const bool row_ok = row0 + rit < off_s[e + 1];
      const int64_t n0 = (int64_t)nb * TN + kEpiCols * g;
      const float* sw_e = p.sw + (int64_t)e * p.sw_expert_stride;
      const int64_t swrow = n0 < p.N ? tc::wrow_block(n0, p.seam, p.N) * p.Kb : 0;
      float accf[kEpiCols];
#pragma unroll
      for (int i = 0; i < kEpiCols; ++i) accf[i] = 0.f;
      float sa_next = row_ok ? p.sa[m] : 0.f;      // K-block 0
      float sw_next = n0 < p.N ? __ldg(sw_e + swrow) : 0.f;
      for (int kb = 0; kb < p.Kb; ++kb) {
        const uint32_t buf = kcount % kNBuf, tround = kcount / kNBuf;
        const float f = sa_next * sw_next;
        if (kb + 1 < p.Kb) {
          sa_next = row_ok ? p.sa[(int64_t)(kb + 1) * p.sa_rows + m] : 0.f;
          sw_next = n0 < p.N ? __ldg(sw_e + swrow + kb + 1) : 0.f;
        }
        if (!warp_wait(smem_u32(&tfull[buf]), tround & 1, abort_flag, p.status, 0x504u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_base + buf * TN + tcol;
        // 16 columns per TMEM load: with kEpiCols accumulators live, larger
        // chunks would not fit the register budget of 18 warps per SM
#pragma unroll
        for (int c = 0; c < kEpiCols / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(taddr + 16 * c, r);
          tmem_ld_wait();
          if (c == kEpiCols / 16 - 1) {
            // every column of this warp is in registers: hand the buffer back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty0 + 8u * buf);
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float xv;
            if constexpr (DT == kInt8) xv = __uint_as_float(r[i] + kMagicBits) - kMagic;  // exact
            else xv = __uint_as_float(r[i]);
            accf[16 * c + i] = fmaf(xv, f, accf[16 * c + i]);
          }
        }
        ++kcount;
      }
      if (!ok) break;
      if (row_ok && n0 < p.N) {
        uint16_t* orow = p.out + m * p.ldo + n0;
        const bool vec = (n0 + kEpiCols <= p.N) && ((reinterpret_cast<uintptr_t>(orow) & 15) == 0);
        if (vec) {
#pragma unroll
          for (int j = 0; j < kEpiCols; j += 8) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              float v0 = accf[j + 2 * h];
              float v1 = accf[j + 2 * h + 1];
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
          for (int j = 0; j < kEpiCols; ++j) {
            if (n0 + j < p.N) {
              float x = accf[j];
              if (p.bias) x += bf16_bits_to_float(__ldg(p.bias + n0 + j));
              orow[j] = float_to_bf16_bits(x);
            }
          }
        }
      }
    }
  }

  if (warp == 0 && rank == 0 && (leader_drain || *abort_flag)) {
    // wait (bounded) for the loads counted on the leader's stage barriers
    for (int s = 0; s < kStages; ++s) {
      if (issued_parity[s] < 0) continue;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(&full[s]), (uint32_t)issued_parity[s]) &&
             globaltimer() - t0 < 100000000ull) {
      }
    }
  }
  // neither CTA leaves (freeing shared memory a pair MMA or peer arrive may
  // still address) before the other is done
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// Clusters of two CTAs of this kernel the device can hold at once.
template <int DT, int TN>
int max_active_pairs() {
  static int cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return tc::sm_count() / 2;
  if (cache[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Pair<TN>::kTotal;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 2;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<DT, TN>, &cfg) != cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = tc::sm_count() / 2;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

template <int DT, int TN>
cudaError_t launch_pair_typed(const GemmArgs& a, cudaStream_t st) {
  using L = Pair<TN>;
  auto kern = gemm_tc2_kernel<DT, TN>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kTotal);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tA, tB;
  if (!tc::make_tmap(&tA, a.qa, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.lda, 128) ||
      !tc::make_tmap(&tB, a.qw, (uint64_t)a.K, (uint64_t)(a.N * a.E), (uint64_t)a.ldw, TN / 2))
    return cudaErrorInvalidValue;
  TcParams p;
  p.sa = a.sa; p.sa_rows = a.sa_rows;
  p.sw = a.sw; p.sw_expert_stride = a.sw_expert_stride;
  p.M = a.M; p.N = a.N; p.K = a.K; p.Kb = (a.K + BK - 1) / BK; p.Kmma = p.Kb; p.bn = 128; p.seam = a.seam;
  p.offsets = a.offsets; p.E = (int)a.E;
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.out = static_cast<uint16_t*>(a.out); p.ldo = a.ldo;
  p.nblk = (int)((a.N + TN - 1) / TN);
  p.status = a.status;
  const int64_t mblk_bound = (a.M + TM - 1) / TM + (a.offsets ? a.E : 0);
  const int64_t tiles_bound = mblk_bound * p.nblk;
  const int64_t npairs =
      std::max<int64_t>(1, std::min<int64_t>(tiles_bound, max_active_pairs<DT, TN>()));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * npairs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kTotal;
  cfg.stream = st;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeClusterDimension;
  at.val.clusterDim.x = 2;
  at.val.clusterDim.y = 1;
  at.val.clusterDim.z = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tA, tB, p);
}

}  // namespace

cudaError_t launch_gemm_tc_pair(const GemmArgs& a, int tile_n, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  if (tile_n == 128)
    return a.dtype == kInt8 ? launch_pair_typed<kInt8, 128>(a, st)
                            : launch_pair_typed<kFp8, 128>(a, st);
  return a.dtype == kInt8 ? launch_pair_typed<kInt8, 256>(a, st)
                          : launch_pair_typed<kFp8, 256>(a, st);
}

}  // namespace bq
