// gemm_tc_common.cuh -- pieces shared by the tensor-core GEMM kernels: the
// kernel parameter block, the weight-scale row of an output column, the tile
// scheduler, and the host-side TMA descriptor and device queries.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "bq_common.cuh"

namespace bq {
namespace tc {

constexpr int kMaxE = 256;                      // experts a grouped launch may hold
constexpr int BK = 128;                         // K-block (= block_k)
constexpr uint32_t kMagicBits = 0x4B400000u;    // float 1.5 * 2^23
constexpr float kMagic = 12582912.0f;

struct TcParams {
  const float* sa; int64_t sa_rows;             // activation scales [Kb][sa_rows]
  const float* sw; int64_t sw_expert_stride;    // weight scales [E][Nbs][Kb]
  int64_t M, N, K, Kb, seam;
  int64_t Kmma;                                 // 128-wide K-blocks the MMAs walk
  int64_t bn;                                   // weight-scale rows cover bn output columns
  const int32_t* offsets; int E;                // grouped: expert row ranges (device)
  const uint16_t* bias;
  uint16_t* out; int64_t ldo;
  int nblk;                                     // tile columns
  unsigned* status;
  // fused SiLU * up + requantisation (gate/up weight, seam = I): codes of h
  // [rows, I] (row stride ldq) and scales [I / 128][sa_rows] instead of out
  uint8_t* q_out; int64_t ldq; float* s_out;
  float* out_f32;                               // unrounded fp32 output (no bias) or null
  // weighted top-k combine into fp32 token rows (w2 of the MoE layer) or null
  float* comb_acc; const int32_t* comb_perm; const float* comb_w; int topk;
};

// Four fp32 atomic adds to consecutive, 16-byte aligned global addresses in
// one vector reduction.
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// x rounded to bf16 (nearest even) and back.
__device__ __forceinline__ float bf16_round(float x) {
  return bf16_bits_to_float(float_to_bf16_bits(x));
}

// Weight-scale row of output column n (block_n = 128).  A fused gate+up
// weight blocks its halves separately: rows past the seam restart at
// ceil(seam / 128).
__device__ __forceinline__ int64_t wrow_block(int64_t n, int64_t seam, int64_t N) {
  if (seam <= 0 || seam >= N || n < seam) return n >> 7;
  return ((seam + 127) >> 7) + ((n - seam) >> 7);
}

// Expert row ranges into shared memory (clamped to [0, M], nondecreasing;
// anything else is recorded as bad input) and the prefix of tile counts per
// expert, for tiles of TM rows and `nblk` tile columns.  One thread.
template <int TM>
__device__ inline void load_expert_ranges(const TcParams& p, int* off_s, int* tp_s) {
  int prev = 0;
  bool bad = false;
  for (int e = 0; e <= p.E; ++e) {
    int v = p.offsets ? p.offsets[e] : (e == 0 ? 0 : (int)p.M);
    if (e == 0 && v != 0) bad = true;
    int c = min(max(v, prev), (int)p.M);
    if (c != v) bad = true;
    off_s[e] = (e == 0) ? 0 : c;
    prev = off_s[e];
  }
  if (bad) record_status(p.status, kStatusBadInput, 0x201u);
  tp_s[0] = 0;
  for (int e = 0; e < p.E; ++e)
    tp_s[e + 1] = tp_s[e] + ((off_s[e + 1] - off_s[e] + TM - 1) / TM) * p.nblk;
}

// Tile t -> (expert, m-block, n-block) for tiles of TM rows; m-blocks vary
// fastest so concurrent CTAs share weight tiles and an expert's activations
// stay in L2.
template <int TM>
__device__ __forceinline__ void decode_tile(int t, const int* tp, const int* off, int E,
                                            int& e_hint, int& e, int& mb, int& nb) {
  int ee = e_hint;
  while (ee + 1 < E && t >= tp[ee + 1]) ++ee;
  e_hint = ee;
  e = ee;
  const int local = t - tp[ee];
  const int mblocks = (off[ee + 1] - off[ee] + TM - 1) / TM;
  mb = local % mblocks;
  nb = local / mblocks;
}

// ---- host side ------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (libbq does
// not link libcuda).
inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Row-major [rows, inner] uint8 tensor with row stride ld_bytes; boxes of
// box_rows x 128 bytes, 128-byte swizzle, zero fill out of bounds.
inline bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                      uint64_t ld_bytes, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {ld_bytes};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

inline int sm_count() {
  static int n[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (n[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n[dev] = v > 0 ? v : 148;
  }
  return n[dev];
}

}  // namespace tc
}  // namespace bq
