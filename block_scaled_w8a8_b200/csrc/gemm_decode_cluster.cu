// gemm_decode_cluster.cu -- block-scaled GEMM for few tokens (decode), with
// the split-K reduction inside thread-block clusters (no global scratch).
//
// Same contraction as the other GEMM paths (block-wise INT8 page, sections 2
// and 4: out = sum_kb P_kb * sa * sw in fp32, one bf16 rounding), organised
// for what bounds a decode layer on B200: the weights (N*K bytes) are read
// exactly once and dominate the bytes, and every synchronisation on the
// critical path costs latency (~0.1 us per mbarrier wait or tcgen05 commit,
// ~0.7 us from one kernel's end to the next kernel's dependency release).
//
//  * Work split: clusters of S CTAs per 128-row weight tile; CTA s streams
//    the weight K-blocks [s Kb / S, (s + 1) Kb / S) of its tile (swap-AB: the
//    128 weight rows are the MMA's M, the tokens, padded to NT = 16..128, its
//    N).  S is chosen so that the tiles x S CTAs cover ~80% of the SMs or
//    more, one CTA per SM.
//  * Weight stream: every CTA requests all of its weights at once, before it
//    waits for the preceding kernel (programmatic dependent launch): the
//    first two ring stages into shared memory, the rest into L2; it releases
//    the next kernel at its start, and stays under half an SM of shared
//    memory, so consecutive layers' CTAs share an SM and their weight
//    streams overlap.  Weights are loaded with an L2 evict-first policy.
//  * Ring: two stages of TWO K-blocks (weight and activation tiles of both),
//    one mbarrier per stage, so the MMA thread and the epilogue synchronise
//    once per two K-blocks.
//  * Epilogue: the partial of each K-block is promoted from tensor memory
//    with sa[kb][t] * sw[tile][kb] (packed fp32x2 arithmetic; INT8 partials
//    converted exactly by an integer add and a float subtract).
//  * Reduction: each CTA stages its 128 x NT row partials in shared memory
//    and sends the rows [o 128/S, (o + 1) 128/S) to CTA o of the cluster with
//    one bulk copy (cp.async.bulk shared::cluster) counted on that CTA's
//    mbarrier; CTA o sums the S slots in split order (deterministic), adds
//    the bias and stores bf16.
//
// Every wait is bounded (2 s): on a timeout the kernel records the site in
// the device status word, skips the remaining data work but still takes part
// in every barrier, drains its copies in flight and frees its tensor memory.
#include <cuda.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "bq_common.cuh"
#include "bq_internal.h"
#include "gemm_decode_cluster.h"
#include "sm100.cuh"

namespace bq {

namespace {

using namespace sm100;

constexpr int TW = 128;           // weight rows per tile (MMA M)
constexpr int BK = 128;           // K-block
constexpr int kEpiWarps = 4;      // warps 2..5: epilogue, one TMEM lane quadrant each
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
// named barriers: 1 = epilogue warps, 2 = MMA warp + epilogue warps (tensor
// memory free)
constexpr int kBarEpi = 1, kBarTmem = 2;

struct DecParams {
  const float* sa;                            // activation scales [Kb][M]
  const float* sw;                            // weight scales [Nb][Kb]
  int M, N, K, Kb;
  int S;                                      // CTAs (K-splits) per tile
  const uint16_t* bias;
  uint16_t* out; int64_t ldo;
  float* out_f32;                             // unrounded fp32 output (no bias) or null
  unsigned* status;
};

// Shared-memory layout for a token tile of NT columns.  Stage st of the
// two-stage ring holds TWO K-blocks: their weight tiles (16 KB each) and
// activation tiles (NT x 128 bytes each), tracked by one mbarrier.
template <int NT>
struct Lay {
  static constexpr int SW = 2;                                    // ring stages
  static constexpr int MaxKb = NT <= 32 ? 64 : 32;                // K-blocks per split
  static constexpr uint32_t kTmem = NT <= 16 ? 128u : 256u;
  static constexpr int NB = (int)(kTmem / NT) < 8 ? (int)(kTmem / NT) : 8;   // TMEM K-block buffers
  static constexpr int NP = NB / 2;                               // TMEM pair slots
  static constexpr uint32_t kW = TW * BK;
  static constexpr uint32_t kA = NT * BK;
  static constexpr uint32_t kStage = 2 * kW + 2 * kA;
  static constexpr int kNtp = NT + 4;                             // padded partial row
  static constexpr uint32_t kRed = 128u * kNtp * 4u;              // 128 rows of partials
  // The outgoing partials are staged at the start of the ring once this
  // CTA's MMAs are done.  The incoming ones get their own region, except for
  // NT = 64, where shared memory is short: there they also alias the ring
  // and a cluster barrier makes sure every CTA is done with its ring first.
  static constexpr bool kAlias = NT == 64;
  static constexpr uint32_t kRing0 = SW * kStage;
  static constexpr uint32_t oSlots = kAlias ? kRed : kRing0;
  static constexpr uint32_t kRing1 = kAlias ? (kRing0 > 2 * kRed ? kRing0 : 2 * kRed) : kRing0 + kRed;
  static constexpr uint32_t kRing = (kRing1 + 1023) / 1024 * 1024;
  static constexpr uint32_t oSa = kRing;                          // [MaxKb][NT] fp32
  static constexpr uint32_t oSw = oSa + MaxKb * NT * 4;           // [MaxKb] fp32
  static constexpr uint32_t oBar = oSw + MaxKb * 4;
  static constexpr uint32_t kBars = 16 * 8;
  static constexpr uint32_t kTotal = 1024 + oBar + kBars + 64;
  static_assert(kStage % 1024 == 0 && kA % 1024 == 0, "MMA operand tiles need 1 KB alignment");
  static_assert(NP >= 1 && NB * NT <= (int)kTmem, "tensor memory");
  static_assert(kRed <= kRing0, "staging fits in the ring");
  static_assert(NT > 64 || kTotal <= 112u * 1024u, "two CTAs per SM");
  static_assert(kTotal <= 227u * 1024u, "shared memory");
};

// Named barriers that tolerate divergent warps (non-.aligned forms).
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id, int n) {
  asm volatile("barrier.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Ask L2 to fetch a 2-D tile of the tensor map (no shared-memory copy).
__device__ __forceinline__ void tma_prefetch_l2(const CUtensorMap* m, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y)
               : "memory");
}

// Bulk copy of `bytes` (multiple of 16) from this CTA's shared memory to
// another CTA's (cluster address), completion counted on the mbarrier at
// cluster address `bar` in the destination CTA.
__device__ __forceinline__ void bulk_to_peer(uint32_t dst, uint32_t src, uint32_t bytes,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "r"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16c(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bounded wait on a local mbarrier whose arrivals may come from other CTAs
// of the cluster (acquire at cluster scope).
__device__ __forceinline__ bool wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned* status, unsigned site) {
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


// Two fp32 values of block partials.  INT8 partials (|P| < 2^22) convert
// exactly without the conversion unit: the bits of 1.5*2^23 + P, minus
// 1.5*2^23 (an integer add and a float subtract).
template <int DT>
__device__ __forceinline__ uint64_t partial2(uint32_t b0, uint32_t b1) {
  if constexpr (DT == kInt8) {
    const uint64_t biased = pack2(__int_as_float((int)b0 + 0x4B400000),
                                  __int_as_float((int)b1 + 0x4B400000));
    return add2(biased, pack2(-12582912.0f, -12582912.0f));
  } else {
    return pack2(__uint_as_float(b0), __uint_as_float(b1));
  }
}


template <int DT, int NT>
__global__ void __launch_bounds__(kThreads, NT <= 64 ? 2 : 1)
gemm_decode_cluster_kernel(const __grid_constant__ CUtensorMap tmW,
                           const __grid_constant__ CUtensorMap tmA, const DecParams p) {
  using L = Lay<NT>;
  constexpr int SW = L::SW, NP = L::NP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sa_all = reinterpret_cast<float*>(smem + L::oSa);
  float* sw_s = reinterpret_cast<float*>(smem + L::oSw);
  float* staging = reinterpret_cast<float*>(smem);            // after this CTA's MMAs
  float* slots = reinterpret_cast<float*>(smem + L::oSlots);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::oBar);
  uint64_t* full = bars;            // [SW] weight + activation tiles of a stage arrived
  uint64_t* empty = bars + 2;       // [SW] the MMAs reading a stage completed
  uint64_t* tfull = bars + 4;       // [NP] a pair of K-block partials is in tensor memory
  uint64_t* tempty = bars + 8;      // [NP] the epilogue has read it
  uint64_t* red = bars + 12;        // the split partials of this CTA's rows arrived
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // K-block h (0, 1) of stage st
  auto wtile = [&](int st, int h) { return smem + st * L::kStage + h * L::kW; };
  auto atile = [&](int st, int h) { return smem + st * L::kStage + 2 * L::kW + h * L::kA; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S;
  const int s = (int)cluster_rank();
  const int tile = (int)blockIdx.x / S;
  const int kb0 = (int)((int64_t)s * p.Kb / S), kb1 = (int)((int64_t)(s + 1) * p.Kb / S);
  const int nkb = kb1 - kb0;
  const int npair = (nkb + 1) / 2;
  auto nbk = [&](int pr) { return min(2, nkb - 2 * pr); };     // K-blocks in pair pr
  const int M = p.M;
  const int R = TW / S;                          // rows of the tile this CTA reduces

  if (threadIdx.x == 0) {
    for (int i = 0; i < SW; ++i) {
      mbar_init(smem_u32(&full[i]), 2);          // weight arm + activation arm
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int b = 0; b < NP; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), kEpiWarps);
    }
    mbar_init(smem_u32(&red[0]), 1);
    mbar_init(smem_u32(&drain[0]), 1);
    *abort_flag = 0;
    fence_mbar_init();
    // the S splits of this tile each send R rows of NT + 4 floats here
    mbar_arrive_expect_tx(smem_u32(&red[0]), L::kRed);
  } else if (warp >= 2) {
    // the weight scales of this split do not depend on the preceding kernel
    for (int j = (int)threadIdx.x - 64; j < nkb; j += kEpiThreads)
      sw_s[j] = __ldg(p.sw + (int64_t)tile * p.Kb + kb0 + j);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("griddepcontrol.launch_dependents;");
    // every weight byte of this CTA is requested now, before the wait for the
    // preceding kernel: the first two stages into the ring, the rest into L2
    const uint64_t pol = policy_evict_first();
    for (int pr = 0; pr < min(SW, npair); ++pr) {
      mbar_arrive_expect_tx(smem_u32(&full[pr]), (uint32_t)nbk(pr) * L::kW);
      for (int h = 0; h < nbk(pr); ++h)
        tma_load_2d_hint(smem_u32(wtile(pr, h)), &tmW, (kb0 + 2 * pr + h) * BK, tile * TW,
                         smem_u32(&full[pr]), pol);
    }
    for (int i = 2 * SW; i < nkb; ++i) tma_prefetch_l2(&tmW, (kb0 + i) * BK, tile * TW);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), L::kTmem);
  // cluster barrier, phase 1: every CTA's mbarriers are initialised before any
  // CTA copies into its shared memory (waited on later)
  cluster_arrive();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the remaining cluster phases of the warps that take no part in the reduction
  auto finish_phases = [&]() {
    cluster_wait();                      // phase 1
    if (L::kAlias) {
      cluster_arrive();                  // phase 2: rings free
      cluster_wait();
    }
    cluster_arrive();                    // last phase: every copy has landed
    cluster_wait();
  };

  if (warp == 0) {
    // ------------------------- TMA producer -------------------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      grid_dep_wait();                           // codes are the predecessor's output
      for (int pr = 0; pr < min(SW, npair); ++pr) {
        mbar_arrive_expect_tx(smem_u32(&full[pr]), (uint32_t)nbk(pr) * L::kA);
        for (int h = 0; h < nbk(pr); ++h)
          tma_load_2d(smem_u32(atile(pr, h)), &tmA, (kb0 + 2 * pr + h) * BK, 0,
                      smem_u32(&full[pr]));
      }
      int issued = min(SW, npair);
      for (int pr = SW; pr < npair; ++pr) {
        const int st = pr % SW;
        if (!mbar_wait(smem_u32(&empty[st]), (uint32_t)(((pr / SW) & 1) ^ 1), abort_flag,
                       p.status, 0x501u))
          break;
        mbar_arrive_expect_tx(smem_u32(&full[st]), (uint32_t)nbk(pr) * (L::kW + L::kA));
        for (int h = 0; h < nbk(pr); ++h) {
          tma_load_2d_hint(smem_u32(wtile(st, h)), &tmW, (kb0 + 2 * pr + h) * BK, tile * TW,
                           smem_u32(&full[st]), pol);
          tma_load_2d(smem_u32(atile(st, h)), &tmA, (kb0 + 2 * pr + h) * BK, 0,
                      smem_u32(&full[st]));
        }
        mbar_arrive(smem_u32(&full[st]));       // the stage's second arrival
        issued = pr + 1;
      }
      if (*abort_flag) {
        // wait (bounded) for the copies that may still be landing in the ring
        for (int pr = max(0, issued - SW); pr < issued; ++pr) {
          const uint64_t t1 = globaltimer();
          while (!mbar_try_wait(smem_u32(&full[pr % SW]), (uint32_t)((pr / SW) & 1)) &&
                 globaltimer() - t1 < 100000000ull) {
          }
        }
      }
    }
    __syncwarp();
    finish_phases();
    return;
  }

  if (warp == 1) {
    // --------------------------- MMA issuer ---------------------------
    constexpr uint32_t idesc = instr_desc<DT>(TW, NT);
    if (lane == 0) {
      bool issued_any = false;
      for (int pr = 0; pr < npair; ++pr) {
        const int pp = pr % NP, st = pr % SW;
        // a tensor-memory pair slot used before must have been read (first
        // uses need no wait)
        if (pr >= NP && !mbar_wait(smem_u32(&tempty[pp]), (uint32_t)(((pr / NP) & 1) ^ 1),
                                   abort_flag, p.status, 0x503u))
          break;
        if (!mbar_wait(smem_u32(&full[st]), (uint32_t)((pr / SW) & 1), abort_flag, p.status,
                       0x504u))
          break;
        tc_fence_after();
        for (int h = 0; h < nbk(pr); ++h) {
          const uint32_t d = tmem_base + (uint32_t)((2 * pp + h) * NT);
          const uint64_t a0 = smem_desc_k128(smem_u32(wtile(st, h)));
          const uint64_t b0 = smem_desc_k128(smem_u32(atile(st, h)));
#pragma unroll
          for (int j = 0; j < BK / 32; ++j)
            mma<DT>(d, a0 + (uint64_t)(2 * j), b0 + (uint64_t)(2 * j), idesc, j > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&empty[st]));
        mma_commit(smem_u32(&tfull[pp]));
        issued_any = true;
      }
      if (issued_any) {
        // every MMA issued has completed (bounded) before tensor memory is freed
        mma_commit(smem_u32(&drain[0]));
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(&drain[0]), 0) && globaltimer() - t0 < 100000000ull) {
        }
      }
    }
    __syncwarp();
    named_bar(kBarTmem, 32 + kEpiThreads);   // the epilogue has read tensor memory for the last time
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmem);
    __syncwarp();
    finish_phases();
    return;
  }

  // ------------------------- epilogue (warps 2..5) -------------------------
  const int et = (int)threadIdx.x - 64;          // 0..127
  grid_dep_wait();                               // scales and output of the predecessor
  for (int idx = et; idx < nkb * M; idx += kEpiThreads) {
    const int j = idx / M, t = idx - j * M;
    sa_all[j * NT + t] = p.sa[(int64_t)(kb0 + j) * M + t];
  }
  named_bar(kBarEpi, kEpiThreads);
  cluster_wait();                                // phase 1
  const int q = warp & 3;                        // TMEM lane quadrant of this warp
  const int r = 32 * q + lane;                   // weight row within the tile
  const uint32_t lane_base = (uint32_t)(32 * q) << 16;
  uint64_t acc[NT / 2];                          // fp32 pairs (tokens 2c, 2c + 1)
#pragma unroll
  for (int c = 0; c < NT / 2; ++c) acc[c] = 0ull;
  for (int pr = 0; pr < npair; ++pr) {
    const int pp = pr % NP;
    const bool got = warp_wait(smem_u32(&tfull[pp]), (uint32_t)((pr / NP) & 1), abort_flag,
                               p.status, 0x507u);
    if (!got) continue;
    tc_fence_after();
    for (int h = 0; h < nbk(pr); ++h) {
      const int i = 2 * pr + h;
      const uint64_t swp = pack2(sw_s[i], sw_s[i]);
      const float* sai = sa_all + i * NT;
      // 16 columns at a time (token columns >= M are skipped)
#pragma unroll
      for (int c = 0; c < NT / 16; ++c) {
        if (16 * c < M) {
          uint32_t rr[16];
          tmem_ld16c(tmem_base + lane_base + (uint32_t)((2 * pp + h) * NT + 16 * c), rr);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint64_t scl =
                fma2(*reinterpret_cast<const uint64_t*>(sai + 16 * c + 2 * e), swp, 0ull);
            acc[8 * c + e] = fma2(partial2<DT>(rr[2 * e], rr[2 * e + 1]), scl, acc[8 * c + e]);
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&tempty[pp]));
  }
  // tensor memory is no longer read by this warp: the MMA warp may free it
  tc_fence_before();
  named_bar_arrive(kBarTmem, 32 + kEpiThreads);

  if (L::kAlias) {
    // phase 2: every CTA is done with its ring, whose second part receives
    // the peers' partials
    cluster_arrive();
    cluster_wait();
  }
  {
    // this CTA's row partials, then one bulk copy per owner: rows
    // [o R, (o + 1) R) go to the CTA that reduces them, into its slot s
    float* row = staging + r * L::kNtp;
#pragma unroll
    for (int c = 0; c < NT / 4; ++c)
      if (4 * c < M)
        *reinterpret_cast<uint4*>(row + 4 * c) =
            make_uint4((uint32_t)acc[2 * c], (uint32_t)(acc[2 * c] >> 32),
                       (uint32_t)acc[2 * c + 1], (uint32_t)(acc[2 * c + 1] >> 32));
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    named_bar(kBarEpi, kEpiThreads);
    if (et == 0 && !*abort_flag) {
      for (int o = 0; o < S; ++o) {
        bulk_to_peer(mapa_shared(smem_u32(slots + s * R * L::kNtp), (uint32_t)o),
                     smem_u32(staging + o * R * L::kNtp), (uint32_t)(R * L::kNtp * 4),
                     mapa_shared(smem_u32(&red[0]), (uint32_t)o));
      }
    }
  }
  const bool all_in = wait_cluster(smem_u32(&red[0]), 0, abort_flag, p.status, 0x508u);
  if (all_in && !*abort_flag) {
    const int quads = (M + 3) / 4;
    for (int idx = et; idx < R * quads; idx += kEpiThreads) {
      const int rr = idx % R, tq = idx / R;
      const int64_t n = (int64_t)tile * TW + s * R + rr;
      if (n >= p.N) continue;
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int src = 0; src < S; ++src) {
        const float4 v =
            *reinterpret_cast<const float4*>(slots + (src * R + rr) * L::kNtp + 4 * tq);
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      const float vals[4] = {sum.x, sum.y, sum.z, sum.w};
      if (p.out_f32) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * tq + e < M) p.out_f32[(int64_t)(4 * tq + e) * p.ldo + n] = vals[e];
        continue;
      }
      const float bv = p.bias ? bf16_bits_to_float(p.bias[n]) : 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (4 * tq + e < M)
          p.out[(int64_t)(4 * tq + e) * p.ldo + n] = float_to_bf16_bits(vals[e] + bv);
    }
  }
  // last phase: once every CTA has its rows, every bulk copy (which reads the
  // sender's shared memory) has completed and the CTAs may exit
  cluster_arrive();
  cluster_wait();
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
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

bool tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t ld,
             uint32_t box_rows) {
  if (!encoder()) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {ld};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t es[2] = {1u, 1u};
  return encoder()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int nt_for(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

int max_kb_for(int nt) { return nt <= 32 ? Lay<16>::MaxKb : Lay<64>::MaxKb; }


template <int DT, int NT>
cudaError_t launch_one(const DecClusterArgs& a, const DecClusterPlan& plan, cudaStream_t st) {
  using L = Lay<NT>;
  auto kern = gemm_decode_cluster_kernel<DT, NT>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kTotal);
  if (e != cudaSuccess) return e;
  CUtensorMap tW, tA;
  if (!tmap_u8(&tW, a.qw, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.ldw, TW) ||
      !tmap_u8(&tA, a.qa, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.lda, NT))
    return cudaErrorInvalidValue;
  DecParams p;
  p.sa = a.sa; p.sw = a.sw;
  p.M = (int)a.M; p.N = (int)a.N; p.K = (int)a.K; p.Kb = (int)((a.K + BK - 1) / BK);
  p.S = plan.S;
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.out = static_cast<uint16_t*>(a.out); p.ldo = a.ldo;
  p.out_f32 = a.out_f32;
  p.status = a.status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(plan.tiles * p.S), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kTotal;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tW, tA, p);
}

template <int DT>
cudaError_t launch_dt(const DecClusterArgs& a, const DecClusterPlan& plan, cudaStream_t st) {
  switch (plan.nt) {
    case 16: return launch_one<DT, 16>(a, plan, st);
    case 32: return launch_one<DT, 32>(a, plan, st);
    case 64: return launch_one<DT, 64>(a, plan, st);
    default: return launch_one<DT, 128>(a, plan, st);
  }
}

int sm_count() {
  static int n[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1)
      v = 148;
    n[dev] = v;
  }
  return n[dev];
}

}  // namespace

DecClusterPlan gemm_decode_cluster_plan(int64_t M, int64_t N, int64_t K) {
  DecClusterPlan d;
  d.nt = nt_for(M);
  d.tiles = (N + TW - 1) / TW;
  const int64_t Kb = (K + BK - 1) / BK;
  // CTAs: at least ~80% of the SMs where the tiles allow it (one CTA per SM
  // and up to 8 K-splits, the portable cluster size)
  const int64_t target = (sm_count() * 4) / 5;
  int S = 1;
  while (S < 8 && d.tiles * S < target && 2 * S <= Kb) S *= 2;
  while (S < 8 && 2 * S <= Kb && (Kb + S - 1) / S > max_kb_for(d.nt)) S *= 2;
  d.S = S;
  d.ok = (Kb + S - 1) / S <= max_kb_for(d.nt) && d.tiles * S <= INT32_MAX;
  return d;
}

bool gemm_decode_cluster_supported(const DecClusterArgs& a, char* why, size_t n) {
  auto no = [&](const char* msg) {
    if (why) snprintf(why, n, "cluster decode path: %s", msg);
    return false;
  };
  if (a.M < 1 || a.M > 128) return no("needs 1 <= M <= 128");
  if (a.bn != 128 || a.bk != 128) return no("needs block_n = block_k = 128");
  if (a.K < 1) return no("needs K >= 1");
  if (a.N > INT32_MAX || a.K > INT32_MAX) return no("sizes exceed int32");
  if (a.ldw % 16 != 0 || (reinterpret_cast<uintptr_t>(a.qw) & 15))
    return no("weight rows must be 16-byte aligned");
  if (a.lda % 16 != 0 || (reinterpret_cast<uintptr_t>(a.qa) & 15))
    return no("activation code rows must be 16-byte aligned");
  if (!gemm_decode_cluster_plan(a.M, a.N, a.K).ok) return no("too many K-blocks per split");
  if (!encoder()) return no("cuTensorMapEncodeTiled is unavailable");
  return true;
}

cudaError_t launch_gemm_decode_cluster(const DecClusterArgs& a, cudaStream_t st) {
  const DecClusterPlan plan = gemm_decode_cluster_plan(a.M, a.N, a.K);
  if (!plan.ok) return cudaErrorInvalidValue;
  if (a.dtype == kInt8) return launch_dt<kInt8>(a, plan, st);
  return launch_dt<kFp8>(a, plan, st);
}

}  // namespace bq
