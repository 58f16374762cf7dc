// moe.cu -- MoE token permutation and weighted combine; bounded-wait self-test.
//
// Permutation (block-wise INT8 page, sections 5-6: experts own their weights,
// routed tokens run per expert): the T*topk (token, slot) pairs are grouped
// by expert in a stable order (by expert, then flat index t*topk + j).  One
// CTA of 1024 threads: pass 1 counts pairs per expert (shared-memory
// atomics), an exclusive scan gives expert_offsets, pass 2 walks the pairs in
// chunks of 1024 and ranks each pair among equal experts with a warp
// match + per-warp counts scanned across warps, so the order is stable
// without any global sort.  Everything stays on the device.
//
// Combine: out[t, n] = bf16( sum_j w[t, j] * y[inv_perm[t*topk+j], n] ),
// fp32 accumulation, one rounding; 8 bf16 per thread with 16-byte vectors.
//
// Routing (the topk_ids / topk_weights the MoE runner of sections 5-6
// receives): one warp per token picks its top-k experts from the fp32 router
// logits -- the softmax is monotonic, so the k largest logits are the k
// largest probabilities, ties to the lower expert index -- and weights them
// exp(l_j - l_max) / sum over the k of exp(l_i - l_max): the softmax
// probabilities renormalised over the chosen k (the full softmax denominator
// cancels).
#include <algorithm>

#include "bq_common.cuh"
#include "bq_internal.h"

namespace bq {

namespace {

constexpr int kPermThreads = 1024;
constexpr int kMaxExperts = 256;

__global__ void __launch_bounds__(kPermThreads)
moe_permute_kernel(const int32_t* __restrict__ ids, int64_t R, int E,
                   int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                   int32_t* __restrict__ inv_perm, unsigned* status) {
  __shared__ int cnt[kMaxExperts];
  __shared__ int base[kMaxExperts];
  __shared__ int wcnt[kPermThreads / 32][kMaxExperts + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int64_t i = tid; i < R; i += kPermThreads) {
    int e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else bad = true;
  }
  if (bad) record_status(status, kStatusBadInput, 0x101u);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      base[e] = run;
      offsets[e] = run;
      run += cnt[e];
    }
    offsets[E] = run;
  }
  __syncthreads();
  for (int64_t c0 = 0; c0 < R; c0 += kPermThreads) {
    const int64_t i = c0 + tid;
    int e = (i < R) ? ids[i] : -1;
    if (e < 0 || e >= E) e = -1;
    // zero the per-warp counters
    for (int x = lane; x < E; x += 32) wcnt[warp][x] = 0;
    __syncwarp();
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_in_warp = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    if (e >= 0 && lane == leader) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    // exclusive scan over warps for each expert (one thread per expert)
    for (int x = tid; x < E; x += kPermThreads) {
      int run = base[x];
      for (int w = 0; w < kPermThreads / 32; ++w) {
        int v = wcnt[w][x];
        wcnt[w][x] = run;
        run += v;
      }
      base[x] = run;
    }
    __syncthreads();
    if (e >= 0) {
      const int r = wcnt[warp][e] + rank_in_warp;
      perm[r] = (int32_t)i;
      inv_perm[i] = (int32_t)r;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256)
moe_combine_kernel(const uint16_t* __restrict__ y, int64_t ldy,
                   const int32_t* __restrict__ inv_perm, const float* __restrict__ w,
                   int64_t T, int topk, int64_t H, uint16_t* __restrict__ out, int64_t ldo,
                   bool vec) {
  const int64_t chunks = (H + 7) / 8;
  const int64_t total = T * chunks;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = idx / chunks, c = idx - t * chunks;
    const int64_t n0 = c * 8;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = 0; j < topk; ++j) {
      const float wt = w[t * topk + j];
      const uint16_t* row = y + (int64_t)inv_perm[t * topk + j] * ldy + n0;
      if (vec && n0 + 8 <= H) {
        uint4 u = *reinterpret_cast<const uint4*>(row);
        const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(wt, bf16_bits_to_float((uint16_t)(p[i] & 0xFFFFu)), acc[2 * i]);
          acc[2 * i + 1] = fmaf(wt, bf16_bits_to_float((uint16_t)(p[i] >> 16)), acc[2 * i + 1]);
        }
      } else {
        for (int i = 0; i < 8; ++i)
          if (n0 + i < H) acc[i] = fmaf(wt, bf16_bits_to_float(row[i]), acc[i]);
      }
    }
    uint16_t* orow = out + t * ldo + n0;
    if (vec && n0 + 8 <= H) {
      uint4 u;
      u.x = (uint32_t)float_to_bf16_bits(acc[0]) | ((uint32_t)float_to_bf16_bits(acc[1]) << 16);
      u.y = (uint32_t)float_to_bf16_bits(acc[2]) | ((uint32_t)float_to_bf16_bits(acc[3]) << 16);
      u.z = (uint32_t)float_to_bf16_bits(acc[4]) | ((uint32_t)float_to_bf16_bits(acc[5]) << 16);
      u.w = (uint32_t)float_to_bf16_bits(acc[6]) | ((uint32_t)float_to_bf16_bits(acc[7]) << 16);
      *reinterpret_cast<uint4*>(orow) = u;
    } else {
      for (int i = 0; i < 8; ++i)
        if (n0 + i < H) orow[i] = float_to_bf16_bits(acc[i]);
    }
  }
}

// Top-k routing of one token per warp: the k largest logits in k rounds of a
// warp arg-max (ties to the lower expert index; softmax is increasing, so
// this is the top-k of the probabilities), then their softmax weights
// renormalised over the k: exp(l_j - l_max) / sum.
constexpr int kRouteMaxE = 256, kRouteMaxK = 8;

__global__ void __launch_bounds__(256)
moe_route_kernel(const float* __restrict__ logits, int64_t ld, int64_t T, int E, int topk,
                 int32_t* __restrict__ ids, float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = kRouteMaxE / 32;
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + t * ld;
  // lane holds experts lane, lane + 32, ...
  float v[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? row[e] : -INFINITY;
  }
  unsigned taken = 0;                           // bit i: expert lane + 32 i chosen
  int sel[kRouteMaxK];
  float lsel[kRouteMaxK];
  for (int j = 0; j < topk; ++j) {
    // this lane's best unchosen (largest logit, then lowest expert index)
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken & (1u << i)) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    sel[j] = be;
    lsel[j] = bv;
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
  }
  if (lane == 0) {
    float ex[kRouteMaxK], sum = 0.0f;
    for (int j = 0; j < topk; ++j) {
      ex[j] = expf(lsel[j] - lsel[0]);
      sum += ex[j];
    }
    for (int j = 0; j < topk; ++j) {
      ids[t * topk + j] = sel[j];
      w[t * topk + j] = ex[j] / sum;
    }
  }
}

// Waits for a flag that nothing sets, at most spin_limit polls, then records
// a timeout in the status word and returns.
__global__ void selftest_wait_kernel(int64_t spin_limit, unsigned* status) {
  __shared__ volatile int flag;
  if (threadIdx.x == 0) flag = 0;
  __syncthreads();
  if (threadIdx.x != 0) return;
  int64_t it = 0;
  while (flag == 0) {
    if (++it >= spin_limit) {
      record_status(status, kStatusTimeout, 0xFF0u);
      return;
    }
    __nanosleep(32);
  }
}

}  // namespace

cudaError_t launch_moe_permute(const int32_t* ids, int64_t T, int64_t topk, int64_t E,
                               int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                               unsigned* status, cudaStream_t st) {
  if (E > kMaxExperts) return cudaErrorInvalidValue;
  const int64_t R = T * topk;
  moe_permute_kernel<<<1, kPermThreads, 0, st>>>(ids, R, (int)E, offsets, perm, inv_perm,
                                                 status);
  return cudaGetLastError();
}

cudaError_t launch_moe_combine(const void* y, int64_t ldy, const int32_t* inv_perm,
                               const float* w, int64_t T, int64_t topk, int64_t H, void* out,
                               int64_t ldo, cudaStream_t st) {
  if (T == 0 || H == 0) return cudaSuccess;
  const bool vec = ((uintptr_t)y % 16 == 0) && ((uintptr_t)out % 16 == 0) && ldy % 8 == 0 &&
                   ldo % 8 == 0;
  const int64_t total = T * ((H + 7) / 8);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, 148 * 8));
  moe_combine_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(y), ldy, inv_perm, w, T,
                                           (int)topk, H, static_cast<uint16_t*>(out), ldo,
                                           vec);
  return cudaGetLastError();
}

// out[t, n] = bf16(acc[t, n]) and acc[t, n] = 0: the single rounding of
// the combine sums the w2 epilogue accumulated, leaving the sums ready for
// the next layer call.  Four columns per chunk; a thread first loads its
// kFinUnroll chunks, then stores them: a store of zeros right behind the
// load of the same address holds the thread's next load until the first
// returns (measured on B200: 6.5x slower at 64 MB of sums).
constexpr int kFinUnroll = 8;

__global__ void __launch_bounds__(256)
moe_combine_finish_kernel(float* __restrict__ acc, int64_t T, int64_t N, int64_t ld_acc,
                          uint16_t* __restrict__ out, int64_t ldo, bool vec) {
  const int64_t chunks = (N + 3) / 4;
  const int64_t total = T * chunks;
  const int64_t tile = (int64_t)blockDim.x * kFinUnroll;
  for (int64_t base = (int64_t)blockIdx.x * tile; base < total; base += (int64_t)gridDim.x * tile) {
    float4 v[kFinUnroll];
#pragma unroll
    for (int k = 0; k < kFinUnroll; ++k) {
      const int64_t idx = base + (int64_t)k * blockDim.x + threadIdx.x;
      if (idx >= total) break;
      const int64_t t = idx / chunks, n0 = (idx - t * chunks) * 4;
      if (vec && n0 + 4 <= N) v[k] = *reinterpret_cast<const float4*>(acc + t * ld_acc + n0);
    }
#pragma unroll
    for (int k = 0; k < kFinUnroll; ++k) {
      const int64_t idx = base + (int64_t)k * blockDim.x + threadIdx.x;
      if (idx >= total) break;
      const int64_t t = idx / chunks, n0 = (idx - t * chunks) * 4;
      float* a = acc + t * ld_acc + n0;
      uint16_t* o = out + t * ldo + n0;
      if (vec && n0 + 4 <= N) {
        *reinterpret_cast<float4*>(a) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<uint2*>(o) = make_uint2(
            (uint32_t)float_to_bf16_bits(v[k].x) | ((uint32_t)float_to_bf16_bits(v[k].y) << 16),
            (uint32_t)float_to_bf16_bits(v[k].z) | ((uint32_t)float_to_bf16_bits(v[k].w) << 16));
      } else {
        for (int i = 0; i < 4 && n0 + i < N; ++i) {
          o[i] = float_to_bf16_bits(a[i]);
          a[i] = 0.f;
        }
      }
    }
  }
}

cudaError_t launch_moe_combine_finish(float* acc, int64_t T, int64_t N, int64_t ld_acc, void* out,
                                      int64_t ldo, cudaStream_t st) {
  if (T == 0 || N == 0) return cudaSuccess;
  const bool vec = ((uintptr_t)acc % 16 == 0) && ((uintptr_t)out % 8 == 0) && ld_acc % 4 == 0 &&
                   ldo % 4 == 0;
  const int64_t total = T * ((N + 3) / 4);
  const int64_t tiles = (total + 256 * kFinUnroll - 1) / (256 * kFinUnroll);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, 148 * 8));
  moe_combine_finish_kernel<<<grid, 256, 0, st>>>(acc, T, N, ld_acc, static_cast<uint16_t*>(out),
                                                  ldo, vec);
  return cudaGetLastError();
}

cudaError_t launch_moe_route(const float* logits, int64_t ld, int64_t T, int64_t E,
                             int64_t topk, int32_t* ids, float* w, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (E < 1 || E > kRouteMaxE || topk < 1 || topk > kRouteMaxK || topk > E)
    return cudaErrorInvalidValue;
  const int64_t blocks = (T + 7) / 8;
  if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
  moe_route_kernel<<<(unsigned)blocks, 256, 0, st>>>(logits, ld, T, (int)E, (int)topk, ids, w);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(int64_t spin_limit, unsigned* status, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(spin_limit, status);
  return cudaGetLastError();
}

}  // namespace bq
