// bq_internal.h -- host-side launcher declarations shared by the libbq
// translation units.  Launchers only enqueue; argument checking is done by the
// C ABI layer (api.cu) before any launcher is called.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace bq {

// Activation quantisation, 1 x group_k groups, optional row gather:
// output row r reads source row (perm ? perm[r] / topk : r).
cudaError_t launch_quant_act(const void* x, int64_t M_out, int64_t K, int64_t ldx,
                             const int32_t* perm, int64_t topk, int64_t group_k, int dtype,
                             void* q, int64_t ldq, float* s, cudaStream_t st);

// Offline [bn, bk] block quantisation of fp32 weights.
cudaError_t launch_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw,
                                int64_t bn, int64_t bk, int dtype, void* q, int64_t ldq,
                                float* s, cudaStream_t st);

// h = bf16(silu(gate) * up) then 1 x group_k quantisation of h.
cudaError_t launch_silu_mul_quant(const void* y, int64_t ldy, int64_t R, int64_t I,
                                  int64_t group_k, int dtype, void* q, int64_t ldq, float* s,
                                  void* h_out, cudaStream_t st);

// Problem description shared by the GEMM kernels.  Grouped problems set
// offsets (device, E+1 entries) and per-expert strides; dense ones set E = 1
// and offsets = nullptr (rows [0, M)).
struct GemmArgs {
  const void* qa; int64_t lda; const float* sa; int64_t sa_rows;  // sa is [Kb][sa_rows]
  const void* qw; int64_t ldw; const float* sw;
  int64_t M, N, K, bn, bk, seam;
  int64_t Nbs;            // weight-scale rows per expert
  int dtype;
  const void* bias;       // bf16 [N] or nullptr
  void* out; int64_t ldo;
  const int32_t* offsets; int64_t E;   // grouped: expert row ranges
  int64_t w_expert_stride;   // bytes between experts' codes (N*K)
  int64_t sw_expert_stride;  // floats between experts' scales (Nbs*Kb)
  unsigned* status;
  // fused SiLU * up + requantisation output (tcgen05 path only): when q_out
  // is set, out is unused and the kernel writes codes [M, seam] (row stride
  // ldq) and scales [seam / 128][sa_rows]
  void* q_out; int64_t ldq; float* s_out;
  // fp32 partial output (bq_gemm_partial): when set, out and bias are unused
  // and the kernel stores sum_kb P_kb * sa * sw unrounded to out_f32 [M, ldo]
  float* out_f32;
  // weighted top-k combine (tcgen05 path only): when comb_acc is set, out
  // and bias are unused and row m adds comb_w[comb_perm[m]] * bf16(row m) to
  // fp32 row comb_perm[m] / topk of comb_acc (row stride ldo) atomically
  float* comb_acc; const int32_t* comb_perm; const float* comb_w; int64_t topk;
  // tcgen05 tile shape: 0 chosen by size, 1 one CTA per tile, 2 CTA pairs
  int tc_shape;
};

cudaError_t launch_gemm_simt(const GemmArgs& a, cudaStream_t st);

// MoE permutation (single CTA) and weighted combine.
cudaError_t launch_moe_permute(const int32_t* ids, int64_t T, int64_t topk, int64_t E,
                               int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                               unsigned* status, cudaStream_t st);
// fp32 combine sums -> bf16 out, and the sums reset to zero.
cudaError_t launch_moe_combine_finish(float* acc, int64_t T, int64_t N, int64_t ld_acc, void* out,
                                      int64_t ldo, cudaStream_t st);
cudaError_t launch_moe_combine(const void* y, int64_t ldy, const int32_t* inv_perm,
                               const float* w, int64_t T, int64_t topk, int64_t H, void* out,
                               int64_t ldo, cudaStream_t st);

// out = bf16(part + bias): the single rounding after a K-sharded sum.
cudaError_t launch_finish_bf16(const float* part, int64_t ldp, int64_t M, int64_t N,
                               const void* bias, void* out, int64_t ldo, cudaStream_t st);

// Top-k routing from fp32 router logits [T, E] (row stride ld).
cudaError_t launch_moe_route(const float* logits, int64_t ld, int64_t T, int64_t E,
                             int64_t topk, int32_t* ids, float* w, cudaStream_t st);

// Bounded-wait self-test.
cudaError_t launch_selftest_wait(int64_t spin_limit, unsigned* status, cudaStream_t st);

}  // namespace bq
