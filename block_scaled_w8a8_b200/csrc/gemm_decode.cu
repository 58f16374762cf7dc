// gemm_decode.cu -- block-scaled GEMM for few tokens (decode), weight-streaming.
//
// Same contraction as the other GEMMs (block-wise INT8 page, sections 2 and 4;
// blockwise FP8 of the SGLang quantization doc), for M <= 128 tokens and
// block_n = block_k = 128.  With so few tokens the layer is bound by reading
// the weights once from HBM, so the kernel is organised around that stream
// and around what must wait for the preceding kernel:
//
//  * swap-AB: the 128 weight rows of a tile are the MMA's M dimension and the
//    tokens (padded to NT = 16/32/64/128) its N dimension, so no MMA rows are
//    wasted on padding tokens;  D[n, t] = sum_k W[n, k] * A[t, k];
//  * split-K: CTA (tile, split) streams the K-blocks [kb0, kb1) of one 128-row
//    weight tile through a TMA ring, small enough that two CTAs share an SM;
//  * before griddepcontrol.wait (programmatic dependent launch) a CTA issues
//    its first weight stages and reads its weight scales: neither depends on
//    the preceding kernel, so both overlap that kernel's tail.  The weights
//    are read exactly once and loaded with an L2 evict-first policy, so they
//    do not push the small, reused tensors of neighbouring layers out of L2.  The next
//    kernel is released once this CTA's first activation tile has arrived,
//    so its weight stream does not queue ahead of this CTA's activation reads;
//  * per-K-block promotion in the epilogue warps (one weight row per thread,
//    one token per TMEM column), each K-block drained as soon as its MMAs
//    complete: acc[t] += P * sa[kb][t] * sw[tile][kb];
//  * cluster mode (enough weight tiles to fill the GPU): the S <= 8 split
//    CTAs of a tile form a thread-block cluster.  Each pushes the partial of
//    every row to the CTA that owns the row (128/S rows each) over
//    distributed shared memory and arrives on that CTA's mbarrier; the owner
//    sums the S partials in split order (deterministic), adds the bias and
//    writes bf16.  One cluster barrier, at start-up, makes the peers'
//    mbarriers visible; no global scratch is touched;
//  * workspace mode (few tiles, so more splits than a cluster holds): split
//    partials go to a workspace; the last CTA to finish a tile sums them in
//    split order (deterministic), adds the bias, writes bf16 and resets the
//    tile's arrival counter.  The counters live in the first
//    kDecodeCounterBytes of the workspace (a fixed place, whatever the shape),
//    so a workspace whose counter region starts zeroed stays usable by any
//    sequence of calls; the partials after it need no initialisation;
//  * TMEM is released as soon as the epilogue has read it, so the CTA's exit
//    (which releases the next kernel) is not held up.
#include <cuda.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "bq_common.cuh"
#include "bq_internal.h"
#include "gemm_decode.h"
#include "sm100.cuh"

namespace bq {

namespace {

using namespace sm100;

constexpr int BN_W = 128;   // weight rows per tile (MMA M)
constexpr int BK = 128;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kMaxSplitKb = 32;  // K-blocks per split (their act scales sit in smem)

struct DecParams {
  const float* sa;       // [Kb][M]
  const float* sw;       // [Nb][Kb]
  int64_t M, N, K, Kb;
  int splits;
  int cluster;           // 1: reduce over distributed shared memory
  const uint16_t* bias;
  uint16_t* out; int64_t ldo;
  float* part;           // [splits][M][N] (splits > 1)
  unsigned* counters;    // [n_tiles]
  unsigned* status;
};

// Shared memory of one CTA.  The ring is as deep as keeps the CTA within
// ~112 KB (two CTAs per SM, so the next launch's CTAs can start streaming
// while this one finishes); NT = 128 takes one CTA per SM.
template <int NT>
struct DSmem {
  static constexpr uint32_t kW = BN_W * BK;                 // weight stage
  static constexpr uint32_t kA = NT * BK;                   // activation tile
  static constexpr uint32_t kStage = kW + kA;
  static constexpr uint32_t kSa = kMaxSplitKb * NT * 4;
  static constexpr uint32_t kSw = kMaxSplitKb * 4;
  static constexpr int kNtp = NT + 4;                        // padded token row (floats)
  static constexpr uint32_t kSlots = kNtp * BN_W * 4;        // [S][128/S][kNtp] fp32
  static constexpr uint32_t kBars = 64 * 8;
  static constexpr uint32_t kFixed = 1024 + kSa + kSw + kSlots + kBars;
  static constexpr uint32_t kBudget = NT <= 64 ? 112u * 1024u : 200u * 1024u;
  static constexpr int kStagesRaw = (int)((kBudget - kFixed) / kStage);
  static constexpr int kStages = kStagesRaw < 2 ? 2 : kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr uint32_t kRing = kStages * kStage;
  // offsets from the 1024-aligned base
  static constexpr uint32_t oSa = kRing;
  static constexpr uint32_t oSw = oSa + kSa;
  static constexpr uint32_t oSlots = oSw + kSw;
  static constexpr uint32_t oBars = oSlots + kSlots;
  static constexpr uint32_t kTotal = 1024 + oBars + kBars;
  static_assert(kRing % 1024 == 0 && kStage % 1024 == 0, "MMA operand tiles need 1 KB alignment");
  static_assert(kTotal <= 227u * 1024u, "shared memory budget");
};

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void named_bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int DT>
__device__ __forceinline__ float pval(uint32_t b) {
  if constexpr (DT == kInt8) return __int2float_rn((int)b);
  else return __uint_as_float(b);
}

// TMEM buffers of NT columns (one K-block partial each): enough that the MMA
// runs ahead of the epilogue instead of waiting for each buffer to drain.
template <int NT>
constexpr int tmem_bufs() { return NT <= 32 ? 8 : NT <= 64 ? 4 : 2; }

template <int NT>
constexpr uint32_t tmem_cols() {
  return (tmem_bufs<NT>() * NT) <= 32 ? 32 : (tmem_bufs<NT>() * NT) <= 64 ? 64
       : (tmem_bufs<NT>() * NT) <= 128 ? 128 : 256;
}

// Bounded wait on a local mbarrier whose arrivals come from other CTAs of the
// cluster (acquire at cluster scope).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag, unsigned* status,
                                                  unsigned site) {
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((i & 63u) == 63u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitTimeoutNs) {
        record_status(status, kStatusTimeout, site);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

template <int DT, int NT>
__global__ void __launch_bounds__(kThreads)
gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
                   const DecParams p) {
  using L = DSmem<NT>;
  constexpr int kStages = L::kStages;
  constexpr int kBufs = tmem_bufs<NT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sa_s = reinterpret_cast<float*>(smem + L::oSa);
  float* sw_s = reinterpret_cast<float*>(smem + L::oSw);
  float* slots = reinterpret_cast<float*>(smem + L::oSlots);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::oBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + 8;
  uint64_t* tfull = bars + 16;
  uint64_t* tempty = bars + 24;
  uint64_t* drain = bars + 32;
  uint64_t* red = bars + 33;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 34);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* epi_abort = reinterpret_cast<volatile int*>(tmem_slot + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.y;
  const int kb0 = (int)((int64_t)split * p.Kb / p.splits);
  const int kb1 = (int)((int64_t)(split + 1) * p.Kb / p.splits);
  const int nkb = kb1 - kb0;
  const int first = min(nkb, kStages);

  // this split's weight scales: constant data, requested before the weight
  // tiles so that they do not queue behind them in the memory system; the
  // epilogue warps store them to shared memory before their first use
  const int swi = (int)threadIdx.x - 64;
  const float sw_reg =
      (swi >= 0 && swi < nkb) ? __ldg(p.sw + (int64_t)tile * p.Kb + kb0 + swi) : 0.f;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 4);
    }
    mbar_init(smem_u32(&drain[0]), 1);
    mbar_init(smem_u32(&red[0]), BN_W);     // one arrival per pushed row
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();                    // barriers initialised, scale loads issued
  if (threadIdx.x == 0) {
    // The weights do not depend on the preceding kernel: the first stages are
    // requested before this CTA waits for its activations.
    tma_prefetch_desc(&tmW);
    for (int i = 0; i < first; ++i) {
      mbar_arrive_expect_tx(smem_u32(&full[i]), L::kStage);
      tma_load_2d_hint(smem_u32(smem + i * L::kStage), &tmW, (kb0 + i) * BK, tile * BN_W,
                       smem_u32(&full[i]), policy_evict_first());
    }
    tma_prefetch_desc(&tmA);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), tmem_cols<NT>());
  // start-up cluster barrier: the peers' mbarriers are initialised before
  // anyone arrives on them remotely (waited on just before the push)
  if (p.cluster) cluster_arrive();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    grid_dep_wait();                              // the activation codes are ready
    if (lane == 0) {
      for (int i = 0; i < first; ++i)
        tma_load_2d(smem_u32(smem + i * L::kStage + L::kW), &tmA, (kb0 + i) * BK, 0,
                    smem_u32(&full[i]));
    }
    bool ok = true;
    int issued_parity[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) issued_parity[s] = s < first ? 0 : -1;
    for (int i = first; i < nkb && ok; ++i) {
      const int stage = i % kStages;
      const uint32_t phase = (uint32_t)((i / kStages) & 1);
      if (!warp_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.status, 0x401u)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(smem_u32(&full[stage]), L::kStage);
        tma_load_2d_hint(smem_u32(smem + stage * L::kStage), &tmW, (kb0 + i) * BK, tile * BN_W,
                         smem_u32(&full[stage]), policy_evict_first());
        tma_load_2d(smem_u32(smem + stage * L::kStage + L::kW), &tmA, (kb0 + i) * BK, 0,
                    smem_u32(&full[stage]));
      }
      issued_parity[stage] = (int)phase;
    }
    if (!ok) {
      for (int s = 0; s < kStages; ++s) {
        if (issued_parity[s] < 0) continue;
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(&full[s]), (uint32_t)issued_parity[s]) &&
               globaltimer() - t0 < 100000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc = instr_desc<DT>(BN_W, NT);
    bool issued_any = false, ok = true;
    for (int i = 0; i < nkb; ++i) {
      const int stage = i % kStages;
      const uint32_t phase = (uint32_t)((i / kStages) & 1);
      const uint32_t buf = (uint32_t)(i % kBufs), tround = (uint32_t)(i / kBufs);
      if (!warp_wait(smem_u32(&tempty[buf]), (tround & 1) ^ 1, abort_flag, p.status, 0x402u) ||
          !warp_wait(smem_u32(&full[stage]), phase, abort_flag, p.status, 0x403u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the first activation tile has arrived: this CTA's reads of the
      // preceding kernel's output are under way, so the next kernel may be
      // scheduled (earlier, its weight stream would queue ahead of them)
      if (i == 0 && lane == 0) asm volatile("griddepcontrol.launch_dependents;");
      if (lane == 0) {
        const uint32_t d = tmem_base + buf * NT;
        const uint64_t a0 = smem_desc_k128(smem_u32(smem + stage * L::kStage));
        const uint64_t b0 = smem_desc_k128(smem_u32(smem + stage * L::kStage + L::kW));
#pragma unroll
        for (int j = 0; j < BK / 32; ++j)
          mma<DT>(d, a0 + (uint64_t)(2 * j), b0 + (uint64_t)(2 * j), idesc, j > 0 ? 1u : 0u);
        mma_commit(smem_u32(&empty[stage]));
        mma_commit(smem_u32(&tfull[buf]));
      }
      __syncwarp();
      issued_any = true;
    }
    (void)ok;
    if (issued_any) {
      // every MMA issued has completed (bounded wait) before TMEM is freed
      if (lane == 0) mma_commit(smem_u32(&drain[0]));
      __syncwarp();
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(&drain[0]), 0) && globaltimer() - t0 < 100000000ull) {
      }
    }
    // free TMEM once the epilogue warps have read their last partial
    named_bar(2, 160);
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols<NT>());
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;                       // TMEM lane quadrant of this warp
    const int et = threadIdx.x - 64;              // 0..127
    const int64_t n = (int64_t)tile * BN_W + 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    if (et < nkb) sw_s[et] = sw_reg;
    grid_dep_wait();                              // sa is written by the quantiser
    for (int idx = et; idx < nkb * NT; idx += 128) {
      const int kbl = idx / NT, t = idx % NT;
      sa_s[idx] = (t < p.M) ? p.sa[(int64_t)(kb0 + kbl) * p.M + t] : 0.f;
    }
    named_bar(1, 128);
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
    // each K-block is drained as soon as its MMAs complete (waiting for more
    // K-blocks first only delays the last ones), up to 64 columns per wait
    constexpr int kCk = NT / 16;                  // 16-column chunks per K-block
    constexpr int kCkB = kCk > 4 ? 4 : kCk;       // chunks per wait
    constexpr int kHalves = kCk / kCkB;           // waits per K-block
    constexpr int kKbPer = 1;
    bool ok = true;
    for (int i0 = 0; i0 < nkb && ok; i0 += kKbPer) {
#pragma unroll
      for (int h = 0; h < kHalves; ++h) {
        uint32_t r[kKbPer][kCkB][16];
#pragma unroll
        for (int u = 0; u < kKbPer; ++u) {
          const int i = i0 + u;
          if (i < nkb && ok) {
            const uint32_t buf = (uint32_t)(i % kBufs);
            if (h == 0) {
              if (!warp_wait(smem_u32(&tfull[buf]), (uint32_t)(i / kBufs) & 1, abort_flag,
                             p.status, 0x404u))
                ok = false;
              else
                tc_fence_after();
            }
            if (ok) {
#pragma unroll
              for (int c = 0; c < kCkB; ++c)
                tmem_ld16(tmem_base + lane_base + buf * NT + 16 * (h * kCkB + c), r[u][c]);
            }
          }
        }
        tmem_ld_wait();
        if (ok) {
#pragma unroll
          for (int u = 0; u < kKbPer; ++u) {
            const int i = i0 + u;
            if (i < nkb) {
              const float swv = sw_s[i];
#pragma unroll
              for (int c = 0; c < kCkB; ++c) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  const int t = 16 * (h * kCkB + c) + j;
                  acc[t] = fmaf(pval<DT>(r[u][c][j]), sa_s[i * NT + t] * swv, acc[t]);
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) {
        for (int u = 0; u < kKbPer && i0 + u < nkb; ++u)
          mbar_arrive(smem_u32(&tempty[(i0 + u) % kBufs]));
      }
    }
    // this warp has read TMEM for the last time: the MMA warp may free it
    tc_fence_before();
    named_bar_arrive(2, 160);
    if (p.cluster) {
      // push this thread's row partial to the CTA that reduces the row:
      // slot [source rank][token][row within the owner's share] of the
      // owner's slot array, then one arrival on the owner's mbarrier
      cluster_wait();                             // start-up barrier: peers are set up
      const int rows_per = BN_W / p.splits;
      const int r = 32 * q + lane;
      const int owner = r / rows_per, rr = r - owner * rows_per;
      const uint32_t my = cluster_rank();
      if (!*abort_flag) {
        constexpr int kNtp = L::kNtp;
        const uint32_t dst = mapa_shared(smem_u32(slots), (uint32_t)owner) +
                             4u * (uint32_t)(((int)my * rows_per + rr) * kNtp);
#pragma unroll
        for (int c = 0; c < NT / 4; ++c)
          if (4 * c < p.M)
            st_dsmem_v4(dst + 16u * (uint32_t)c, acc[4 * c], acc[4 * c + 1], acc[4 * c + 2],
                        acc[4 * c + 3]);
      }
      mbar_arrive_cluster(mapa_shared(smem_u32(&red[0]), (uint32_t)owner));
      // this CTA's rows: all S sources x rows_per rows have arrived
      const bool got = mbar_wait_cluster(smem_u32(&red[0]), 0, abort_flag, p.status, 0x405u);
      if (got && !*abort_flag) {
        // thread -> (row r2 of this CTA's share, token quads tq, tq + ng, ...)
        constexpr int kNtp = L::kNtp;
        const int r2 = et % rows_per, ng = 128 / rows_per;
        const int64_t nn = (int64_t)tile * BN_W + (int)my * rows_per + r2;
        const float b = (p.bias && nn < p.N) ? bf16_bits_to_float(p.bias[nn]) : 0.f;
        const int quads = (int)((p.M + 3) / 4);
        for (int tq = et / rows_per; tq < quads; tq += ng) {
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int src = 0; src < p.splits; ++src) {
            const float4 v =
                *reinterpret_cast<const float4*>(slots + (src * rows_per + r2) * kNtp + 4 * tq);
            sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
          }
          if (nn < p.N) {
            const float vals[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (4 * tq + j < p.M)
                p.out[(int64_t)(4 * tq + j) * p.ldo + nn] = float_to_bf16_bits(vals[j] + b);
          }
        }
      }
    } else {
      // the four epilogue warps take one decision on abort (a consistent
      // snapshot, as the named barriers below need all of them)
      named_bar(1, 128);
      if (et == 0) *epi_abort = *abort_flag;
      named_bar(1, 128);
      if (*epi_abort) return;
      const bool n_ok = n < p.N;
      if (p.splits == 1) {
        if (n_ok) {
          const float b = p.bias ? bf16_bits_to_float(p.bias[n]) : 0.f;
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < p.M) p.out[(int64_t)t * p.ldo + n] = float_to_bf16_bits(acc[t] + b);
        }
      } else {
        if (n_ok) {
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < p.M) p.part[((int64_t)split * p.M + t) * p.N + n] = acc[t];
        }
        __threadfence();
        named_bar(1, 128);
        if (et == 0) {
          const unsigned old = atomicAdd(&p.counters[tile], 1u);
          // a counter that did not start at zero (the workspace's counter
          // region was overwritten) would leave the tile unwritten: report it
          if (old >= (unsigned)p.splits) record_status(p.status, kStatusBadInput, 0x406u);
          *last_flag = (old == (unsigned)(p.splits - 1)) ? 1 : 0;
        }
        named_bar(1, 128);
        if (*last_flag) {
          __threadfence();
          if (n_ok) {
            const float b = p.bias ? bf16_bits_to_float(p.bias[n]) : 0.f;
            for (int t = 0; t < (int)p.M; ++t) {
              float sum = 0.f;
              for (int s = 0; s < p.splits; ++s)
                sum += __ldcg(p.part + ((int64_t)s * p.M + t) * p.N + n);
              p.out[(int64_t)t * p.ldo + n] = float_to_bf16_bits(sum + b);
            }
          }
          if (et == 0) p.counters[tile] = 0u;
        }
      }
    }
  }
  if (p.cluster) {
    // producer and MMA warps: their part of the start-up barrier (the
    // epilogue warps waited on it before pushing)
    if (warp < 2) cluster_wait();
    // every CTA of the cluster, aborted or not, meets here before exiting, so
    // no peer still pushes into or arrives on this CTA's shared memory after
    // it has gone (every wait before this one is bounded)
    cluster_arrive();
    cluster_wait();
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn enc() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

bool tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t ld,
          uint32_t box_rows) {
  if (!enc()) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {ld};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t es[2] = {1u, 1u};
  return enc()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Largest number of clusters of `S` CTAs of this kernel the device can hold
// at once (cached per device and S).
template <int DT, int NT>
int max_active_clusters(int S) {
  static int cache[64][4] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int si = S == 2 ? 0 : S == 4 ? 1 : 2;
  if (dev < 0 || dev >= 64) return 1;
  if (cache[dev][si] == 0) {
    using L = DSmem<NT>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, (unsigned)S, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kTotal;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 1;
    at.val.clusterDim.y = (unsigned)S;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_decode_kernel<DT, NT>, &cfg) !=
            cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = 1;
    }
    cache[dev][si] = n;
  }
  return cache[dev][si];
}

// Split count for cluster mode: keep as many CTAs resident in the first wave
// as possible (fewer waves first, then more resident CTAs, then larger S),
// with at most max_kb K-blocks per split.  0 if no split count fits.
template <int DT, int NT>
int cluster_splits(int64_t tiles, int64_t Kb, int max_kb) {
  int best = 0;
  double best_score = -1.0;
  for (int S = 8; S >= 2; S /= 2) {
    if (S > Kb || (Kb + S - 1) / S > max_kb) continue;
    const int64_t n = max_active_clusters<DT, NT>(S);
    const int64_t waves = (tiles + n - 1) / n;
    const double score = (double)std::min<int64_t>(n, tiles) * S / (double)waves;
    if (score > best_score) {
      best_score = score;
      best = S;
    }
  }
  return best;
}

template <int DT, int NT>
cudaError_t launch_nt(const GemmArgs& a, const DecodePlan& plan_in, void* ws, bool pdl,
                      cudaStream_t st) {
  using L = DSmem<NT>;
  auto kern = gemm_decode_kernel<DT, NT>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kTotal);
  if (e != cudaSuccess) return e;
  DecodePlan plan = plan_in;
  const int64_t Kb = (a.K + BK - 1) / BK;
  if (plan.cluster) {
    plan.splits = cluster_splits<DT, NT>(plan.tiles, Kb, kMaxSplitKb);
    if (plan.splits == 0) return cudaErrorInvalidValue;
  }
  CUtensorMap tW, tA;
  if (!tmap(&tW, a.qw, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.ldw, BN_W) ||
      !tmap(&tA, a.qa, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.lda, NT))
    return cudaErrorInvalidValue;
  DecParams p;
  p.sa = a.sa; p.sw = a.sw;
  p.M = a.M; p.N = a.N; p.K = a.K; p.Kb = Kb;
  p.splits = plan.splits;
  p.cluster = plan.cluster ? 1 : 0;
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.out = static_cast<uint16_t*>(a.out); p.ldo = a.ldo;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const bool use_ws = plan.splits > 1 && !plan.cluster;
  p.counters = use_ws ? reinterpret_cast<unsigned*>(w) : nullptr;
  p.part = use_ws ? reinterpret_cast<float*>(w + kDecodeCounterBytes) : nullptr;
  p.status = a.status;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)plan.tiles, (unsigned)plan.splits, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kTotal;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (plan.cluster) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = (unsigned)plan.splits;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, tW, tA, p);
}

template <int DT>
cudaError_t launch_dt(const GemmArgs& a, const DecodePlan& plan, void* ws, bool pdl,
                      cudaStream_t st) {
  switch (plan.nt) {
    case 16: return launch_nt<DT, 16>(a, plan, ws, pdl, st);
    case 32: return launch_nt<DT, 32>(a, plan, ws, pdl, st);
    case 64: return launch_nt<DT, 64>(a, plan, ws, pdl, st);
    default: return launch_nt<DT, 128>(a, plan, ws, pdl, st);
  }
}

}  // namespace
DecodePlan decode_plan(int64_t M, int64_t N, int64_t K) {
  DecodePlan d;
  d.nt = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  d.tiles = (N + BN_W - 1) / BN_W;
  const int64_t Kb = (K + BK - 1) / BK;
  // about two CTAs per SM, at most kMaxSplitKb K-blocks per split
  const int64_t want = std::max<int64_t>(1, (2 * 148 + d.tiles - 1) / d.tiles);
  d.cluster = false;
  if (d.tiles >= 16 && Kb >= 2 && (Kb + 7) / 8 <= kMaxSplitKb) {
    // cluster mode: the split count (2, 4 or 8) is chosen at launch from the
    // device's cluster occupancy; no workspace is needed
    d.splits = 0;
    d.cluster = true;
    d.part_bytes = 0;
    d.ws_bytes = 0;
    return d;
  }
  int64_t s = std::min<int64_t>(want, Kb);
  s = std::max<int64_t>(s, (Kb + kMaxSplitKb - 1) / kMaxSplitKb);
  s = std::min<int64_t>(s, 65535);
  d.splits = (int)s;
  d.part_bytes = d.splits > 1 ? (size_t)d.splits * (size_t)M * (size_t)N * 4u : 0u;
  d.part_bytes = (d.part_bytes + 255) / 256 * 256;
  d.ws_bytes = d.splits > 1 ? kDecodeCounterBytes + d.part_bytes : 0u;
  return d;
}

bool decode_supported(const GemmArgs& a, char* why, size_t n) {
  auto no = [&](const char* msg) {
    if (why) snprintf(why, n, "decode path: %s", msg);
    return false;
  };
  if (a.offsets) return no("dense problems only");
  if (a.M > 128) return no("at most 128 tokens");
  if (a.bn != 128 || a.bk != 128) return no("needs block_n = block_k = 128");
  if (a.K < 1) return no("needs K >= 1");
  if (a.lda % 16 != 0 || a.ldw % 16 != 0) return no("row strides must be multiples of 16 bytes");
  if ((reinterpret_cast<uintptr_t>(a.qa) & 15) || (reinterpret_cast<uintptr_t>(a.qw) & 15))
    return no("operands must be 16-byte aligned");
  if (a.N > INT32_MAX || a.K > INT32_MAX) return no("sizes exceed int32");
  const int64_t tiles = (a.N + BN_W - 1) / BN_W;
  if (tiles * 4 > (int64_t)kDecodeCounterBytes) return no("N too large for the counter region");
  if (!enc()) return no("cuTensorMapEncodeTiled is unavailable");
  return true;
}

// Scratch for bq_gemm_decode_noalloc: the decode kernel's arrival counters
// (first kDecodeCounterBytes) and split partials, in a fixed device array so
// that callers which cannot allocate device memory can still run the split-K
// decode GEMM.  Every GPU that loads libbq holds these 16 MiB until the
// process exits.  All calls share it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

cudaError_t noalloc_scratch(void** ptr, cudaStream_t st) {
  static std::mutex mu;
  static void* addr[kMaxScratchDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  // The symbol's name is only a host-side handle: ask the runtime for the
  // array's address on the current device.  Outside stream capture the
  // address is looked up again on every call, so a device reset (which
  // reloads the module) cannot leave a stale pointer behind; a capturing
  // stream reuses the address of the last uncaptured call on this device.
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusNone || addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_gemm_decode(const GemmArgs& a, void* ws, bool pdl, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  const DecodePlan plan = decode_plan(a.M, a.N, a.K);
  if (a.dtype == kInt8) return launch_dt<kInt8>(a, plan, ws, pdl, st);
  return launch_dt<kFp8>(a, plan, ws, pdl, st);
}

}  // namespace bq
