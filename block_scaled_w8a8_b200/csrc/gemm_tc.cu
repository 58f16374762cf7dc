// gemm_tc.cu -- block-scaled GEMM on the 5th-generation tensor cores (sm_100a).
//
// out[m, n] = bf16( sum_kb P_kb[m, n] * sa[kb][m] * sw[nb(n)][kb] + bias[n] )
// (block-wise INT8 page, sections 2 and 4; blockwise FP8 of the SGLang
// quantization doc, "GEMM backends for FP4/FP8"), for block_n = block_k = 128.
//
// Design (persistent, warp-specialised, one CTA per SM or one CTA pair per
// two SMs):
//   warps 0, 2, 3  TMA producers: K-block j of the CTA's sequence goes to
//               producer j % 3, which loads its 128x128 A tile and its W
//               tile (BN x 128, or BN/2 x 128 per CTA of a pair; K-major,
//               128-byte swizzle) into an S-stage ring.  One issuing thread
//               sustains about one TMA tile per 270 ns on B200.
//   warp 1      MMA issuer (lane 0 alone): 4 x tcgen05.mma (K = 32 each) per
//               K-block into a TMEM buffer; the buffer holds exactly one
//               K-block's partial P_kb (int32 for kind::i8, fp32 for
//               kind::f8f6f4).  512 / BN TMEM buffers (all 512 columns)
//               rotate.  Also owns the TMEM allocation.
//   warps 4-19  epilogue: warp w reads TMEM lanes 32*(w%4).. (one output row
//               per thread) and columns [BN/4*h, BN/4*(h+1)), h = (w-4)/4; it
//               promotes acc += P_kb * (sa[kb][m] * sw[nb][kb]) in fp32
//               registers (scalar FADD/FFMA: measured faster here than the
//               packed f32x2 forms), frees the buffer, and after the last
//               K-block adds the bias and stores bf16 with 32-byte stores.
//   registers   setmaxnreg moves registers from the control warpgroup (56
//               each) to the epilogue (104 each): no spills in the
//               promotion loop (+5% INT8, +3% FP8 measured).
// INT8 promotion without an integer add or the int->float conversion unit:
// each TMEM buffer is pre-filled with the bits 0x4B400000 (the float
// 1.5 * 2^23), so the MMA's int32 sum 0x4B400000 + P_kb (|P_kb| <=
// 128 * 127 * 127 < 2^22) is the float 12582912 + P_kb exactly; one FADD
// recovers P_kb exactly and one FFMA promotes it.  The epilogue refills
// the buffer (tcgen05.st) as it frees it.
// A tile scheduler walks (expert, m-block, n-block) tiles; a dense problem is
// one expert.  The grouped (MoE) problem reads its expert row ranges from
// device memory, so no host read-back is needed.  Rows of a tile past the
// expert's range are computed but never stored.
//
// Every mbarrier wait is bounded (2 s); on expiry the CTA records a timeout
// in the device status word, drains its in-flight TMA loads and MMAs, frees
// its tensor memory and exits.
#include <cuda.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "bq_common.cuh"
#include "bq_internal.h"
#include "gemm_tc.h"
#include "gemm_tc_common.cuh"
#include "sm100.cuh"

namespace bq {

namespace {

using namespace sm100;

constexpr int BM = 128;
using tc::BK;
using tc::kMaxE;
using tc::kMagic;
using tc::kMagicBits;
using tc::TcParams;
using tc::decode_tile;
using tc::wrow_block;
using tc::bf16_round;
using tc::red_add_v4;
using tc::make_tmap;
using tc::sm_count;
using tc::encode_fn;
constexpr int kThreads = 640;        // 20 warps: A producer, MMA, W producer, idle, 16 epilogue
constexpr int kEpiWarps = 16;
// Register split (setmaxnreg): the control warpgroup (warps 0-3) gives up
// registers, the four epilogue warpgroups take them, so that 64 fp32
// accumulators and a 16-column TMEM chunk live in registers without spills.
// The epilogue warpgroups' increase waits until the control warpgroup has
// released enough: the split must fit the registers the CTA launched with,
// which launch_typed checks against the compiled kernel before launching.
constexpr int kCtrlRegs = 56;
constexpr int kEpiRegs = 104;
constexpr int kSplitRegs = 128 * kCtrlRegs + 32 * kEpiWarps * kEpiRegs;   // 60416
static_assert(kSplitRegs <= 65536, "register split exceeds the SM's register file");
// TMEM accumulators of BN columns: all 512 columns (4 x 128 or 2 x 256)
template <int BN>
constexpr int tbufs() { return 512 / BN; }
// TMA producer warps (0, 2 and 3), each issuing whole K-blocks in turn
constexpr int kProducers = 3;

// Per CTA: an S-stage ring of one 128-row A tile and the CTA's W rows (all
// BN of them, or BN / 2 for a CTA pair, which splits the MMA's N between its
// two CTAs' shared memory).
template <int BN, int S, bool PAIR = false>
struct Smem {
  static constexpr uint32_t kA = BM * BK, kB = (PAIR ? BN / 2 : BN) * BK;
  static constexpr uint32_t kStages = S * (kA + kB);
  static constexpr uint32_t kBars = (2 * S + 2 * tbufs<BN>() + 6) * 8;
  static constexpr uint32_t kMisc = 8 + 2 * (kMaxE + 1) * 4;
  // SILU: group amax of each tile row from its four column warps, two tiles
  static constexpr uint32_t kAmax = 2 * 4 * BM * 4;
  static constexpr uint32_t kTotal = 1024 + kStages + kBars + kMisc + kAmax;
};

// ONEK: the scale grid has a single K-block (block_k >= K: per-token
// activation scales, per-channel or per-row-block weight scales).  The MMAs
// then accumulate a tile's whole K in TMEM and the epilogue promotes once per
// tile, out = P * sa[m] * sw[n / block_n], instead of once per K-block.
//
// PAIR: a cluster of two CTAs on two SMs computes a 256 x BN tile with
// tcgen05.mma.cta_group::2 (M = 256).  Each CTA stages its own 128 rows of A
// and BN / 2 rows of W per K-block (the MMA reads the other half of W from
// the peer's shared memory), so a K-block moves half the W bytes per SM of
// the single-CTA kernel: L2 -> shared memory traffic per output falls by a
// third at BN = 256.  Each CTA's TMEM receives its own 128 rows of the
// accumulator, so the epilogue is the single-CTA one.  The leader (cluster
// rank 0) issues the MMAs; loads of both CTAs complete on the leader's stage
// barriers (cta_group::2 loads, no multicast); MMA completions are committed
// to both CTAs' barriers; both CTAs' epilogues release a TMEM buffer on the
// leader's barrier.
template <int DT, int BN, int S, bool ONEK, bool SILU, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const TcParams p) {
  using L = Smem<BN, S, PAIR>;
  constexpr int kTBufs = tbufs<BN>();
  constexpr int TM = PAIR ? 2 * BM : BM;           // rows of a scheduled tile
  constexpr int BNL = PAIR ? BN / 2 : BN;          // W rows this CTA stages
  // INT8 K-block partials land on a TMEM buffer pre-filled with the bits of
  // 1.5 * 2^23: the int32 sum 0x4B400000 + P_kb is then the float
  // 12582912 + P_kb exactly (|P_kb| <= 128 * 127 * 127 < 2^22), so the
  // epilogue needs one FADD and one FFMA per element and no integer add; it
  // refills the buffer with the bias as it frees it.  Measured on B200: +8%
  // on the block-wise INT8 GEMM (1176 -> 1268 TOPS at 4096 x 14336 x 4096).
  // The fused SiLU kernel adds the bias with an integer add, as before
  constexpr bool kBias = DT == kInt8 && !ONEK && !SILU;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * L::kA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kStages);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + kTBufs;
  uint64_t* drain = bars + 2 * S + 2 * kTBufs;
  uint64_t* xbar = bars + 2 * S + 2 * kTBufs + 1;   // SILU: amax exchange, per quadrant
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 2 * kTBufs + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* off_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* tp_s = off_s + (kMaxE + 1);
  float* amax_s = reinterpret_cast<float*>(smem + L::kStages + L::kBars + L::kMisc);
  static_assert(!SILU || (BN == 256 && !ONEK), "the fused SiLU epilogue uses 128 x 256 tiles");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);            // the (leader's) producer of the K-block
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < kTBufs; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), (PAIR ? 2 : 1) * kEpiWarps);   // (leader's) epilogues
    }
    mbar_init(smem_u32(&drain[0]), 1);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&xbar[i]), kEpiWarps / 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp != 1 && warp < 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  // expert row ranges (sanitised: clamped to [0, M] and nondecreasing)
  if (threadIdx.x == 32) tc::load_expert_ranges<TM>(p, off_s, tp_s);
  if (warp == 1) {
    if constexpr (PAIR) tmem_alloc_pair(smem_u32(tmem_slot), kTBufs * BN);
    else tmem_alloc(smem_u32(tmem_slot), kTBufs * BN);
  }
  tc_fence_before();
  // a pair's barriers all exist before any load, commit or arrive signals them
  if constexpr (PAIR) cluster_sync_all();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tp_s[E];
  const uint32_t rank = PAIR ? cluster_rank() : 0u;      // 0: the pair's leader
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int nunits = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kCtrlRegs) : "memory");
  if (warp != 1) {
    // ---------------- TMA producers: warps 0, 2 and 3 take whole K-blocks
    // in turn (K-block j of this CTA's sequence goes to producer j % 3), each
    // issuing the A tile and the W tile of its K-blocks.  An issuing thread
    // sustains about one TMA tile per 270 ns on B200, whatever the tile's
    // size, so three issuers keep a 128 x 256 K-block's two tiles ahead of
    // the tensor pipe ----------------
    const int me = warp == 0 ? 0 : warp - 1;            // 0, 1, 2
    // the leader's stage barriers in the cluster window
    const uint32_t full_c0 = PAIR ? mapa_shared(smem_u32(&full[0]), 0) : smem_u32(&full[0]);
    int stage = 0, j = 0;
    uint32_t phase = 0;
    int issued_parity[S];
#pragma unroll
    for (int s = 0; s < S; ++s) issued_parity[s] = -1;
    int e_hint = 0;
    bool ok = true;
    for (int t = unit0; t < total && ok; t += nunits) {
      int e, mb, nb;
      decode_tile<TM>(t, tp_s, off_s, E, e_hint, e, mb, nb);
      const int a_row = off_s[e] + mb * TM + BM * (int)rank;
      const int b_row = e * (int)p.N + nb * BN + BNL * (int)rank;
      for (int kb = 0; kb < p.Kmma; ++kb, ++j) {
        if (j % kProducers == me) {
          if (!warp_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.status, 0x301u)) {
            ok = false;
            break;
          }
          if (PAIR && lane == 0) {
            // the leader's barrier counts the bytes of both CTAs' loads
            const uint32_t bar = full_c0 + 8u * (uint32_t)stage;
            if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * (L::kA + L::kB));
            tma_load_2d_pair(smem_u32(sA + stage * L::kA), &tmA, kb * BK, a_row, bar);
            // SILU: the leader stages the 128 gate rows of the h columns, the
            // peer the 128 up rows, so the MMA's N = 256 operand is gate | up
            const int w_row = SILU ? e * (int)p.N + nb * 128 + (int)rank * (int)p.seam : b_row;
            tma_load_2d_pair(smem_u32(sB + stage * L::kB), &tmB, kb * BK, w_row, bar);
          } else if (lane == 0) {
            const uint32_t bar = smem_u32(&full[stage]);
            mbar_arrive_expect_tx(bar, L::kA + L::kB);
            tma_load_2d(smem_u32(sA + stage * L::kA), &tmA, kb * BK, a_row, bar);
            if (SILU) {
              // 128 gate rows, then the 128 up rows of the same h columns:
              // the MMA's N = 256 operand is the two boxes back to back
              const int g_row = e * (int)p.N + nb * 128;
              tma_load_2d(smem_u32(sB + stage * L::kB), &tmB, kb * BK, g_row, bar);
              tma_load_2d(smem_u32(sB + stage * L::kB + 128 * BK), &tmB, kb * BK,
                          g_row + (int)p.seam, bar);
            } else {
              tma_load_2d(smem_u32(sB + stage * L::kB), &tmB, kb * BK, b_row, bar);
            }
          }
          issued_parity[stage] = (int)phase;
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (!ok && rank == 0) {
      // drain: wait (bounded) for every load this warp issued (a pair's
      // loads, the peer's too, complete on the leader's barriers)
      for (int s = 0; s < S; ++s) {
        if (issued_parity[s] < 0) continue;
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(&full[s]), (uint32_t)issued_parity[s]) &&
               globaltimer() - t0 < 100000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: lane 0 of warp 1 (of a pair's leader) ----
    // One thread, no warp-wide waits or syncs per K-block: the tensor pipe
    // queues little more than one K-block of MMAs, so any per-iteration
    // overhead in the issuing loop shows up as idle tensor cycles.
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = instr_desc<DT>(TM, BN);
      int stage = 0;
      uint32_t phase = 0, kcount = 0;
      bool ok = true, issued_any = false;
      for (int t = unit0; t < total && ok; t += nunits) {
        for (int kb = 0; kb < p.Kmma; ++kb) {
          // a TMEM buffer holds one K-block's partial, or (ONEK) a whole tile's
          const bool unit_first = !ONEK || kb == 0;
          const bool unit_last = !ONEK || kb == p.Kmma - 1;
          const uint32_t buf = kcount % kTBufs, tround = kcount / kTBufs;
          // a biased buffer's first release is the epilogue's initial fill
          const uint32_t tpar = kBias ? (tround & 1) : ((tround & 1) ^ 1);
          if ((unit_first && !mbar_wait(smem_u32(&tempty[buf]), tpar, abort_flag, p.status,
                                        0x302u)) ||
              !mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.status, 0x303u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + buf * BN;
          const uint64_t a0 = smem_desc_k128(smem_u32(sA + stage * L::kA));
          const uint64_t b0 = smem_desc_k128(smem_u32(sB + stage * L::kB));
          if constexpr (PAIR) {
#pragma unroll
            for (int j = 0; j < BK / 32; ++j)
              mma_pair<DT>(d, a0 + (uint64_t)(2 * j), b0 + (uint64_t)(2 * j), idesc,
                           (kBias || j > 0 || !unit_first) ? 1u : 0u);
            mma_commit_pair(smem_u32(&empty[stage]), (uint16_t)0x3);
            if (unit_last) mma_commit_pair(smem_u32(&tfull[buf]), (uint16_t)0x3);
          } else {
#pragma unroll
            for (int j = 0; j < BK / 32; ++j)
              mma<DT>(d, a0 + (uint64_t)(2 * j), b0 + (uint64_t)(2 * j), idesc,
                      (kBias || j > 0 || !unit_first) ? 1u : 0u);
            mma_commit(smem_u32(&empty[stage]));
            if (unit_last) mma_commit(smem_u32(&tfull[buf]));
          }
          issued_any = true;
          if (unit_last) ++kcount;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && issued_any) {
        // wait (bounded) for the issued MMAs before the teardown frees TMEM
        if constexpr (PAIR) mma_commit_pair(smem_u32(&drain[0]), (uint16_t)0x1);
        else mma_commit(smem_u32(&drain[0]));
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(&drain[0]), 0) && globaltimer() - t0 < 100000000ull) {
        }
      }
    }
    __syncwarp();
  }
  } else {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kEpiRegs) : "memory");
  {
    // ---------------- epilogue ----------------
    constexpr int CW = BN / 4;                     // columns per epilogue warp
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int rit = 32 * q + lane;                 // row inside the tile
    const uint32_t tcol = (uint32_t)(CW * half);
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    // hand a TMEM buffer back to the MMA: the leader's barrier (a pair's
    // peer arrives on it remotely)
    const uint32_t tempty_c0 = PAIR ? mapa_shared(smem_u32(&tempty[0]), 0) : 0u;
    auto release_tmem = [=](uint32_t buf) {
      if (PAIR && rank != 0) mbar_arrive_remote(tempty_c0 + 8u * buf);
      else mbar_arrive(smem_u32(&tempty[buf]));
    };
    // this warp's TMEM columns of a buffer: CW from tcol, or (SILU) the 32
    // gate and the 32 up columns of its h columns
    auto fill_bias = [=](uint32_t buf) {
      const uint32_t b0 = tmem_base + lane_base + buf * BN;
      if constexpr (SILU) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          tmem_st4_fill(b0 + 32u * (uint32_t)half + 4u * j, kMagicBits);
          tmem_st4_fill(b0 + 128u + 32u * (uint32_t)half + 4u * j, kMagicBits);
        }
      } else {
#pragma unroll
        for (int j = 0; j < CW / 4; ++j) tmem_st4_fill(b0 + tcol + 4u * j, kMagicBits);
      }
    };
    if constexpr (kBias) {
      for (int b = 0; b < kTBufs; ++b) fill_bias((uint32_t)b);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        for (int b = 0; b < kTBufs; ++b) release_tmem((uint32_t)b);
    }
    uint32_t kcount = 0, tcount = 0;
    int e_hint = 0;
    bool ok = true;
    for (int t = unit0; t < total && ok; t += nunits) {
      int e, mb, nb;
      decode_tile<TM>(t, tp_s, off_s, E, e_hint, e, mb, nb);
      const int row0 = off_s[e] + mb * TM + BM * (int)rank;
      const int64_t m = (int64_t)row0 + rit;
      const bool row_ok = rit < off_s[e + 1] - row0;
      const int64_t n0 = (int64_t)nb * BN + CW * half;
      const float* sw_e = p.sw + (int64_t)e * p.sw_expert_stride;
      const int64_t swrow = n0 < p.N ? wrow_block(n0, p.seam, p.N) * p.Kb : 0;
      // combine: this row's (token, slot) pair and routing weight, read
      // before the K loop so their latency hides behind it
      int pair = -1;
      float comb_wt = 0.f;
      if (p.comb_acc && row_ok) {
        pair = __ldg(p.comb_perm + m);
        if ((unsigned)pair < (unsigned)p.M) comb_wt = __ldg(p.comb_w + pair);
      }
      float accf[CW];
#pragma unroll
      for (int i = 0; i < CW; ++i) accf[i] = 0.f;
      if constexpr (ONEK) {
        // the tile's whole K is in one TMEM buffer: one promotion per element,
        // out = P * (sa[m] * sw[n / block_n]); the int32 sum over all of K is
        // converted with one correctly rounded int -> float
        const uint32_t buf = kcount % kTBufs, tround = kcount / kTBufs;
        const float sa_m = row_ok ? p.sa[m] : 0.f;
        if (!warp_wait(smem_u32(&tfull[buf]), tround & 1, abort_flag, p.status, 0x305u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_base + buf * BN + tcol;
        constexpr int RC = CW <= 32 ? CW : 16;
#pragma unroll
        for (int c = 0; c < CW / RC; ++c) {
          uint32_t r[RC];
          if constexpr (RC == 32) tmem_ld32(taddr, r);
          else tmem_ld16(taddr + RC * c, r);
          tmem_ld_wait();
          if (c == CW / RC - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_tmem(buf);   // TMEM free for the MMA
          }
#pragma unroll
          for (int i = 0; i < RC; ++i) {
            const int64_t col = n0 + RC * c + i;
            const float swc = col < p.N ? __ldg(sw_e + col / p.bn) : 0.f;
            const float v = DT == kInt8 ? __int2float_rn((int)r[i]) : __uint_as_float(r[i]);
            accf[RC * c + i] = v * (sa_m * swc);
          }
        }
        ++kcount;
      } else if constexpr (SILU) {
        // gate columns [32 * half, +32) and the up columns [128 + 32 * half,
        // +32) of the same h columns: h = silu(g) * u needs both in one thread
        const int64_t swg = (int64_t)nb * p.Kb;                  // gate scale row
        const int64_t swu = ((p.seam >> 7) + nb) * p.Kb;         // up scale row
        float sa_next = row_ok ? p.sa[m] : 0.f;
        float sg_next = __ldg(sw_e + swg), su_next = __ldg(sw_e + swu);
        for (int kb = 0; kb < p.Kb; ++kb) {
          const uint32_t buf = kcount % kTBufs, tround = kcount / kTBufs;
          const float fg = sa_next * sg_next, fu = sa_next * su_next;
          if (kb + 1 < p.Kb) {
            sa_next = row_ok ? p.sa[(int64_t)(kb + 1) * p.sa_rows + m] : 0.f;
            sg_next = __ldg(sw_e + swg + kb + 1);
            su_next = __ldg(sw_e + swu + kb + 1);
          }
          if (!warp_wait(smem_u32(&tfull[buf]), tround & 1, abort_flag, p.status, 0x306u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tb = tmem_base + lane_base + buf * BN + 32u * (uint32_t)half;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[16];
            tmem_ld16(tb + (c < 2 ? 16u * c : 128u + 16u * (c - 2)), r);
            tmem_ld_wait();
            if (!kBias && c == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) release_tmem(buf);   // TMEM free for the MMA
            }
            const float f = c < 2 ? fg : fu;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float x = kBias            ? __uint_as_float(r[i]) - kMagic
                              : DT == kInt8 ? __uint_as_float(r[i] + kMagicBits) - kMagic
                                            : __uint_as_float(r[i]);
              accf[16 * c + i] = fmaf(x, f, accf[16 * c + i]);
            }
          }
          if constexpr (kBias) {
            fill_bias(buf);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_tmem(buf);     // TMEM free for the MMA
          }
          ++kcount;
        }
      } else {
        float sa_next = row_ok ? p.sa[m] : 0.f;      // K-block 0
        float sw_next = n0 < p.N ? __ldg(sw_e + swrow) : 0.f;
        for (int kb = 0; kb < p.Kb; ++kb) {
          const uint32_t buf = kcount % kTBufs, tround = kcount / kTBufs;
          const float f = sa_next * sw_next;
          if (kb + 1 < p.Kb) {
            sa_next = row_ok ? p.sa[(int64_t)(kb + 1) * p.sa_rows + m] : 0.f;
            sw_next = n0 < p.N ? __ldg(sw_e + swrow + kb + 1) : 0.f;
          }
          if (!warp_wait(smem_u32(&tfull[buf]), tround & 1, abort_flag, p.status, 0x304u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = tmem_base + lane_base + buf * BN + tcol;
          // CW columns in chunks of RC: all at once for 32, 16 at a time for 64
          // (with 64 accumulators live, larger chunks do not fit the registers)
          constexpr int RC = CW <= 32 ? CW : 16;
#pragma unroll
          for (int c = 0; c < CW / RC; ++c) {
            uint32_t r[RC];
            if constexpr (RC == 32) tmem_ld32(taddr, r);
            else tmem_ld16(taddr + RC * c, r);
            tmem_ld_wait();
            if (!kBias && c == CW / RC - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) release_tmem(buf);   // TMEM free for the MMA
            }
#pragma unroll
            for (int i = 0; i < RC / 2; ++i) {
              float x0, x1;
              if constexpr (kBias) {
                x0 = __uint_as_float(r[2 * i]) - kMagic;
                x1 = __uint_as_float(r[2 * i + 1]) - kMagic;
              } else if constexpr (DT == kInt8) {
                x0 = __uint_as_float(r[2 * i] + kMagicBits) - kMagic;
                x1 = __uint_as_float(r[2 * i + 1] + kMagicBits) - kMagic;
              } else {
                x0 = __uint_as_float(r[2 * i]);
                x1 = __uint_as_float(r[2 * i + 1]);
              }
              accf[RC * c + 2 * i] = fmaf(x0, f, accf[RC * c + 2 * i]);
              accf[RC * c + 2 * i + 1] = fmaf(x1, f, accf[RC * c + 2 * i + 1]);
            }
          }
          if constexpr (kBias) {
            // refill after the last chunk is promoted (its registers are free)
            fill_bias(buf);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_tmem(buf);     // TMEM free for the MMA
          }
          ++kcount;
        }
      }
      if (!ok) break;
      if constexpr (SILU) {
        // h = bf16(silu(g) * u) from the bf16-rounded GEMM outputs (what the
        // unfused path stores and reads back), then the 1 x 128 quantisation
        // of h: the tile's 128 h columns are exactly one group of each row
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float g = bf16_bits_to_float(float_to_bf16_bits(accf[j]));
          const float u = bf16_bits_to_float(float_to_bf16_bits(accf[32 + j]));
          accf[j] = bf16_bits_to_float(silu_mul_bf16(g, u));
          amax = fmaxf(amax, fabsf(accf[j]));
        }
        // the row's group amax from the four column warps of its TMEM lane
        // quadrant (double-buffered by tile parity: the wait of the next tile
        // orders reuse)
        float* ax = amax_s + (tcount & 1u) * (4 * BM);
        ax[half * BM + rit] = amax;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&xbar[q]));
        if (!warp_wait(smem_u32(&xbar[q]), tcount & 1u, abort_flag, p.status, 0x307u)) {
          ok = false;
          break;
        }
        const float gmax = fmaxf(fmaxf(ax[rit], ax[BM + rit]), fmaxf(ax[2 * BM + rit], ax[3 * BM + rit]));
        const float sc = group_scale<DT>(gmax);
        if (row_ok) {
          uint32_t w[8];
          if constexpr (DT == kInt8) {
            // codes through the reciprocal of the scale, equal to the IEEE
            // quotient's (int8_code_recip); a zero scale gives zero codes
            const float rs = __frcp_rn(sc);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              uint32_t ww = 0;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int c = sc == 0.0f ? 0 : int8_code_recip(accf[4 * i + k], sc, rs);
                ww |= (uint32_t)(uint8_t)(int8_t)c << (8 * k);
              }
              w[i] = ww;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = pack4_codes<DT>(accf + 4 * i, sc);
          }
          uint4* qrow = reinterpret_cast<uint4*>(p.q_out + m * p.ldq + (int64_t)nb * 128 + 32 * half);
          qrow[0] = make_uint4(w[0], w[1], w[2], w[3]);
          qrow[1] = make_uint4(w[4], w[5], w[6], w[7]);
          if (half == 0) p.s_out[(int64_t)nb * p.sa_rows + m] = sc;
        }
        ++tcount;
        continue;
      }
      if (p.comb_acc) {
        // weighted top-k combine: add w[t, j] * bf16(y) to token t's fp32
        // sums, each product rounded to fp32 once.  A sum starts from zero,
        // so with top-2 (two terms) the atomic order cannot change it
        if (row_ok && n0 < p.N) {
          if ((unsigned)pair >= (unsigned)p.M) {
            record_status(p.status, kStatusBadInput, 0x309u);
          } else {
            float* arow = p.comb_acc + (int64_t)(pair / p.topk) * p.ldo + n0;
            if (n0 + CW <= p.N && ((reinterpret_cast<uintptr_t>(arow) & 15) == 0)) {
#pragma unroll
              for (int j = 0; j < CW; j += 4)
                red_add_v4(arow + j, comb_wt * bf16_round(accf[j]),
                           comb_wt * bf16_round(accf[j + 1]), comb_wt * bf16_round(accf[j + 2]),
                           comb_wt * bf16_round(accf[j + 3]));
            } else {
              for (int j = 0; j < CW; ++j)
                if (n0 + j < p.N) atomicAdd(arow + j, comb_wt * bf16_round(accf[j]));
            }
          }
        }
        continue;
      }
      if (row_ok && n0 < p.N && p.out_f32) {
        float* frow = p.out_f32 + m * p.ldo + n0;
        if (n0 + CW <= p.N && ((reinterpret_cast<uintptr_t>(frow) & 31) == 0)) {
#pragma unroll
          for (int j = 0; j < CW; j += 8) {
            uint32_t w[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) w[h] = __float_as_uint(accf[j + h]);
            st_global_v8(frow + j, w);
          }
        } else if (n0 + CW <= p.N && ((reinterpret_cast<uintptr_t>(frow) & 15) == 0)) {
#pragma unroll
          for (int j = 0; j < CW; j += 4)
            *reinterpret_cast<float4*>(frow + j) =
                make_float4(accf[j], accf[j + 1], accf[j + 2], accf[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j)
            if (n0 + j < p.N) frow[j] = accf[j];
        }
      } else if (row_ok && n0 < p.N) {
        uint16_t* orow = p.out + m * p.ldo + n0;
        const bool full_n = n0 + CW <= p.N;
        const bool vec = full_n && ((reinterpret_cast<uintptr_t>(orow) & 15) == 0);
        if (vec && (reinterpret_cast<uintptr_t>(orow) & 31) == 0) {
          // 32-byte stores: 16 outputs each, a full L2 sector per lane
#pragma unroll
          for (int j = 0; j < CW; j += 16) {
            uint32_t w[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              float v0 = accf[j + 2 * h];
              float v1 = accf[j + 2 * h + 1];
              if (p.bias) {
                v0 += bf16_bits_to_float(__ldg(p.bias + n0 + j + 2 * h));
                v1 += bf16_bits_to_float(__ldg(p.bias + n0 + j + 2 * h + 1));
              }
              w[h] = (uint32_t)float_to_bf16_bits(v0) | ((uint32_t)float_to_bf16_bits(v1) << 16);
            }
            st_global_v8(orow + j, w);
          }
        } else if (vec) {
#pragma unroll
          for (int j = 0; j < CW; j += 8) {
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
          for (int j = 0; j < CW; ++j) {
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
  }

  tc_fence_before();
  // neither CTA of a pair leaves (freeing shared memory that a pair MMA,
  // load or arrive may still address) before the other is done
  if constexpr (PAIR) cluster_sync_all();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kTBufs * BN);
    else tmem_dealloc(tmem_base, kTBufs * BN);
  }
}

// Clusters of two CTAs of a pair kernel the device holds at once.
template <typename K>
int max_active_pairs(K kern, uint32_t smem_bytes) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeClusterDimension;
  at.val.clusterDim.x = 2;
  at.val.clusterDim.y = 1;
  at.val.clusterDim.z = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  return n;
}

template <int DT, int BN, int S, bool ONEK, bool SILU, bool PAIR>
cudaError_t launch_typed(const GemmArgs& a, cudaStream_t st) {
  using L = Smem<BN, S, PAIR>;
  constexpr int TM = PAIR ? 2 * BM : BM;
  auto kern = gemm_tc_kernel<DT, BN, S, ONEK, SILU, PAIR>;
  static bool attr_set[64] = {};
  static int pairs[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::kTotal);
    if (e != cudaSuccess) return e;
    // the register split must fit what the CTA is launched with, or the
    // epilogue warps' setmaxnreg.inc would never be satisfied
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * kThreads < kSplitRegs) return cudaErrorInvalidConfiguration;
    if (PAIR) pairs[dev] = max_active_pairs(kern, L::kTotal);
    attr_set[dev] = true;
  }
  CUtensorMap tA, tB;
  if (!make_tmap(&tA, a.qa, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.lda, BM) ||
      !make_tmap(&tB, a.qw, (uint64_t)a.K, (uint64_t)(a.N * a.E), (uint64_t)a.ldw,
                 SILU ? 128u : (uint32_t)(PAIR ? BN / 2 : BN)))
    return cudaErrorInvalidValue;
  TcParams p;
  p.sa = a.sa; p.sa_rows = a.sa_rows;
  p.sw = a.sw; p.sw_expert_stride = a.sw_expert_stride;
  p.M = a.M; p.N = a.N; p.K = a.K; p.seam = a.seam;
  p.Kmma = (a.K + BK - 1) / BK;
  p.Kb = ONEK ? 1 : p.Kmma;              // K-blocks of the scale grid
  p.bn = a.bn;
  p.offsets = a.offsets; p.E = (int)a.E;
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.out = static_cast<uint16_t*>(a.out); p.ldo = a.ldo;
  p.nblk = SILU ? (int)(a.seam / 128) : (int)((a.N + BN - 1) / BN);
  p.status = a.status;
  p.q_out = static_cast<uint8_t*>(a.q_out); p.ldq = a.ldq; p.s_out = a.s_out;
  p.out_f32 = a.out_f32;
  p.comb_acc = a.comb_acc; p.comb_perm = a.comb_perm; p.comb_w = a.comb_w; p.topk = (int)a.topk;
  const int64_t mblk_bound = (a.M + TM - 1) / TM + (a.offsets ? a.E : 0);
  const int64_t tiles_bound = mblk_bound * p.nblk;
  if (!PAIR) {
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles_bound, sm_count()));
    kern<<<grid, kThreads, L::kTotal, st>>>(tA, tB, p);
    return cudaGetLastError();
  }
  const int64_t npairs = std::max<int64_t>(1, std::min<int64_t>(tiles_bound, pairs[dev]));
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

// Tile shape (tc_shape 1 forces one CTA per 128 x 256 tile, 2 a CTA pair per
// 256 x 256 tile).  By size: measured on B200, the pair is faster with one
// scale block along K (per-channel: 2020 against 1960 TOPS at 4096 x 14336 x
// 4096) and slower with per-K-block promotion (block-wise INT8 1213 against
// 1268 TOPS, FP8 1541 against 1585 TFLOPS), where the epilogue's TMEM
// hand-off, not the operand feed the pair halves, sets the pace.
bool use_pair(const GemmArgs& a) {
  if (a.tc_shape == 1) return false;
  if (a.tc_shape == 2) return true;
  return a.bk >= a.K && a.M >= 512;
}

}  // namespace

bool tc_supported(const GemmArgs& a, char* why, size_t n) {
  auto no = [&](const char* msg) {
    if (why) snprintf(why, n, "tcgen05 path: %s", msg);
    return false;
  };
  const bool onek = a.bk >= a.K;           // one scale block along K
  if (!(a.bn == 128 && a.bk == 128) && !onek)
    return no("needs block_n = block_k = 128, or block_k >= K (per-token scales)");
  if (onek && a.seam != 0 && a.seam % a.bn != 0)
    return no("with block_k >= K the gate/up seam must be a multiple of block_n");
  if (a.K < 1) return no("needs K >= 1");
  if (a.lda % 16 != 0 || a.ldw % 16 != 0) return no("row strides must be multiples of 16 bytes");
  if ((reinterpret_cast<uintptr_t>(a.qa) & 15) || (reinterpret_cast<uintptr_t>(a.qw) & 15))
    return no("operands must be 16-byte aligned");
  if (a.seam % 128 != 0) return no("the gate/up seam must be a multiple of 128");
  if (a.E > kMaxE) return no("at most 256 experts");
  if (a.M > INT32_MAX || a.N * a.E > INT32_MAX || a.K > INT32_MAX) return no("sizes exceed int32");
  if (!encode_fn()) return no("cuTensorMapEncodeTiled is unavailable");
  return true;
}

bool tc_silu_supported(const GemmArgs& a, char* why, size_t n) {
  auto no = [&](const char* msg) {
    if (why) snprintf(why, n, "fused SiLU path: %s", msg);
    return false;
  };
  if (!(a.bn == 128 && a.bk == 128)) return no("needs block_n = block_k = 128");
  if (a.seam < 128 || a.seam % 128 != 0 || a.N != 2 * a.seam)
    return no("needs a gate/up weight [2I, K] with I a multiple of 128");
  if (a.bias) return no("takes no bias");
  if (a.ldq % 16 != 0 || (reinterpret_cast<uintptr_t>(a.q_out) & 15))
    return no("the code output needs 16-byte aligned rows");
  GemmArgs b = a;
  b.q_out = nullptr;
  return tc_supported(b, why, n);
}

cudaError_t launch_gemm_tc_silu(const GemmArgs& a, cudaStream_t st) {
  if (a.M == 0 || a.seam == 0) return cudaSuccess;
  if (use_pair(a))
    return a.dtype == kInt8 ? launch_typed<kInt8, 256, 6, false, true, true>(a, st)
                            : launch_typed<kFp8, 256, 6, false, true, true>(a, st);
  if (a.dtype == kInt8) return launch_typed<kInt8, 256, 4, false, true, false>(a, st);
  return launch_typed<kFp8, 256, 4, false, true, false>(a, st);
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  // 128 x 256 tiles: a K-block's 48 KB of operands feed twice the MMA work of
  // a 128 x 128 tile (32 KB), and the L2 -> shared-memory feed is what bounds
  // this kernel on B200 (measured: FP8 +40%, INT8 +11% over 128 x 128).
  // Narrow problems keep 128-wide tiles.
  // a single scale block along K (per-token / per-channel scales): promote
  // once per tile instead of once per 128-wide K-block
  const bool onek = a.bk >= a.K;
  if (a.N > 128 && use_pair(a)) {
    if (a.dtype == kInt8)
      return onek ? launch_typed<kInt8, 256, 6, true, false, true>(a, st)
                  : launch_typed<kInt8, 256, 6, false, false, true>(a, st);
    return onek ? launch_typed<kFp8, 256, 6, true, false, true>(a, st)
                : launch_typed<kFp8, 256, 6, false, false, true>(a, st);
  }
  if (a.N > 128) {
    if (a.dtype == kInt8)
      return onek ? launch_typed<kInt8, 256, 4, true, false, false>(a, st)
                  : launch_typed<kInt8, 256, 4, false, false, false>(a, st);
    return onek ? launch_typed<kFp8, 256, 4, true, false, false>(a, st)
                : launch_typed<kFp8, 256, 4, false, false, false>(a, st);
  }
  if (a.dtype == kInt8)
    return onek ? launch_typed<kInt8, 128, 6, true, false, false>(a, st)
                : launch_typed<kInt8, 128, 6, false, false, false>(a, st);
  return onek ? launch_typed<kFp8, 128, 6, true, false, false>(a, st)
              : launch_typed<kFp8, 128, 6, false, false, false>(a, st);
}

}  // namespace bq
