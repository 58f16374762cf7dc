/*
 * bq.h -- C ABI of libbq: block-scaled W8A8 (INT8 / FP8-e4m3) linear layers
 * and their MoE grouped-GEMM variant, for NVIDIA B200 (sm_100a).
 *
 * What is computed (sources are web pages, cited by title and section):
 *
 *  - "[SGLang] Block-wise INT8: 블록 단위 정수 양자화" (the block-wise INT8 page):
 *      structure diagram + section 2: weight W [N, K] int8 (row n = output
 *        channel, K contiguous) with fp32 block scales [ceil(N/bn), ceil(K/bk)],
 *        one per [block_n, block_k] block; the stored scale multiplies the
 *        code back to the weight (W ~= q * s);
 *      section 1: block size has two dimensions, activations are quantised
 *        dynamically only, the checkpoint is already int8-serialised;
 *      section 4: the activation scale is computed at run time (input_scale
 *        = None), per token, inside the kernel;
 *      section 5/6: MoE experts hold their own weights and scales; w13 is the
 *        gate and up projections fused, [E, 2I, H], scales
 *        [E, 2*ceil(I/bn), ceil(H/bk)].
 *  - SGLang "양자화 (Quantization)" doc, "FP4/FP8 양자화용 GEMM 백엔드":
 *      blockwise FP8 GEMM, the same contraction on e4m3 codes; the MXFP8
 *      dense linear (format read as the microscaling one: see bq_mx_*).
 *  - "LLM 양자화 완전 정리 — FP8, AWQ, GPTQ, GGUF 차이와 선택법", FP8 section:
 *      e4m3 = 1 sign, 4 exponent, 3 mantissa bits.
 *
 * The arithmetic, with the readings taken where the pages are silent:
 *   activation group = 1 x group_k elements of one row (per token, per K-block);
 *   s = amax / Q in IEEE fp32 division, Q = 127 (INT8) or 448 (FP8 e4m3);
 *   q = clamp(round_half_even(x / s), -128, 127)           (INT8)
 *     = e4m3(x / s), round-to-nearest-even, saturating at +-448  (FP8)
 *     with x / s one IEEE fp32 division; an all-zero group has s = 0, q = 0;
 *   out[m, n] = bf16( sum_kb P_kb[m,n] * sa[kb][m] * sw[nb(n)][kb] + bias[n] )
 *     with P_kb the exact int32 (INT8) / fp32-accumulated (FP8) dot product
 *     of the codes inside K-block kb, the sum over blocks in fp32, and one
 *     round-to-nearest-even conversion to bf16 at the end.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller, except where
 *    stated.  The library never allocates or frees device memory; kernels that
 *    need scratch take a caller-provided workspace, sized by the matching
 *    *_workspace_size query.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call only enqueues work on it and never synchronises, except
 *    bq_check_device_status.
 *  - Sizes are int64_t element counts; leading dimensions ("ld") are in
 *    elements of the array's type.  bf16 arrays are passed as void* holding
 *    16-bit bfloat16 values.  Quantised codes are passed as void* holding one
 *    byte per element (int8 two's complement, or e4m3 bits).
 *  - Every call returns a bq_status.  Argument errors are detected on the host
 *    before anything is enqueued; bq_last_error_message() then describes the
 *    problem (thread-local).  M == 0 (or N == 0, R == 0, T == 0) is a no-op.
 *  - Activation scales use the K-block-major layout [Kb][M] (Kb =
 *    ceil(K/group_k)), dense: the scale of row m in K-block g is s[g*M + m].
 *    (The pages do not fix this layout; K-block-major lets a GEMM tile read
 *    the scales of its rows for one K-block as one contiguous run.)
 *  - Weight scales are [Nb][Kb] row-major as on the block-wise INT8 page.
 *  - The MXFP8 calls (bq_mx_*) keep their E8M0 scales in the tensor-core
 *    atom layout described before bq_mx_scale_bytes.
 */
#ifndef BQ_H_
#define BQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bq_status {
    BQ_OK = 0,
    BQ_ERR_INVALID_ARG = 1,     /* bad pointer, size, stride or dtype */
    BQ_ERR_UNSUPPORTED = 2,     /* valid request no kernel implements */
    BQ_ERR_ALIGNMENT = 3,       /* a forced kernel path needs aligned data */
    BQ_ERR_WORKSPACE = 4,       /* workspace missing or too small */
    BQ_ERR_CUDA = 5,            /* a CUDA runtime call failed */
    BQ_ERR_DEVICE_TIMEOUT = 6   /* a bounded device-side wait gave up */
} bq_status;

typedef enum bq_dtype {
    BQ_INT8 = 0,      /* int8 codes, Q = 127, int32 block partials */
    BQ_FP8_E4M3 = 1   /* e4m3 codes, Q = 448, fp32 block partials */
} bq_dtype;

/* GEMM kernel families (for bq_set_path). */
typedef enum bq_path {
    BQ_PATH_AUTO = 0,     /* choose by shape and alignment */
    BQ_PATH_SIMT = 1,     /* generic CUDA-core kernel: any shape/stride */
    BQ_PATH_TCGEN05 = 2,  /* TMA + tcgen05 tensor-core kernel (large M; tile shape by size) */
    BQ_PATH_DECODE = 3,   /* split-K weight-streaming kernel (small M) */
    BQ_PATH_TCGEN05_1CTA = 4,  /* force the single-CTA tcgen05 kernel (128x256 tiles) */
    BQ_PATH_TCGEN05_PAIR = 5   /* force the CTA-pair tcgen05 kernel (256x256 tiles, cta_group::2) */
} bq_path;

/* ---- library information and errors ---------------------------------- */

/* Library version, major*10000 + minor*100 + patch. */
int bq_version(void);

/* Static description of a status code (never NULL). */
const char* bq_status_string(int status);

/* Description of the last error raised on the calling host thread ("" if
 * none).  The pointer stays valid until the next bq_* call on this thread. */
const char* bq_last_error_message(void);

/* Force the GEMM kernel family used by bq_gemm / bq_linear /
 * bq_grouped_gemm on the calling host thread (BQ_PATH_AUTO restores the
 * automatic choice).  A forced path that cannot run the given shape returns
 * BQ_ERR_UNSUPPORTED or BQ_ERR_ALIGNMENT instead of falling back. */
bq_status bq_set_path(int path);
int bq_get_path(void);

/* Read and clear the current device's status word, which kernels set when a
 * bounded wait gives up (BQ_ERR_DEVICE_TIMEOUT, with the wait site in the
 * message) or when they meet invalid device-side input such as an expert id
 * out of range (BQ_ERR_INVALID_ARG).  Synchronises `stream`. */
bq_status bq_check_device_status(void* stream);

/* Self-test of the device status word: launches one tiny kernel that waits
 * for a flag nothing sets, with an iteration limit of `spin_limit`; the wait
 * runs out and records a timeout.  A following bq_check_device_status
 * returns BQ_ERR_DEVICE_TIMEOUT.  Faults nothing and leaves the context
 * usable. */
bq_status bq_selftest_bounded_wait(int64_t spin_limit, void* stream);

/* ---- configuration checks (host only) --------------------------------- */

/* The three rejections of the block-wise INT8 config (page section 1):
 * a block size requires an int8-serialised checkpoint
 * (checkpoint_int8_serialized != 0), the block size has exactly two
 * dimensions (n_block_dims == 2), and the activation scheme is dynamic
 * (dynamic_activation != 0).  has_block_size == 0 accepts everything.
 * Returns BQ_OK or BQ_ERR_INVALID_ARG with the reason in the message. */
bq_status bq_check_block_config(int has_block_size, int checkpoint_int8_serialized,
                                int64_t n_block_dims, int dynamic_activation);

/* Tensor-parallel alignment of the block-wise INT8 page, section 3.
 * Row-parallel (tp_size > 1 and input_size / input_size_per_partition ==
 * tp_size): input_size_per_partition must be a multiple of block_k.
 * Column-parallel: every output_partition_sizes[i] (host array of n_parts)
 * must be a multiple of block_n.  Returns BQ_OK or BQ_ERR_INVALID_ARG. */
bq_status bq_check_tp_partition(int64_t tp_size, int64_t input_size,
                                int64_t input_size_per_partition,
                                const int64_t* output_partition_sizes, int64_t n_parts,
                                int64_t block_n, int64_t block_k);

/* ---- dynamic activation quantisation ------------------------------ */

/* x: bf16 [M, K], row stride ldx >= K.  Writes q [M, K] codes (row stride
 * ldq >= K) and s: fp32 [ceil(K/group_k)][M] (K-block-major, dense).
 * group_k >= 1; the last group of a row may be partial (ceil division) and
 * takes its amax over its valid elements only.  dtype: bq_dtype.
 * Block-wise INT8 page section 4 (dynamic, per token); groups of 1 x
 * block_k so that each K-block has its own activation scale. */
bq_status bq_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, int64_t group_k,
                       int dtype, void* q, int64_t ldq, float* s, void* stream);

/* ---- offline weight block quantisation ---------------------------- */

/* w: fp32 [N, K] (row stride ldw >= K).  Writes q [N, K] (row stride
 * ldq >= K) and s: fp32 [ceil(N/block_n)][ceil(K/block_k)] row-major, one
 * scale per [block_n, block_k] block (amax over the block's valid elements
 * / Q).  Block-wise INT8 page, structure diagram and section 2.  Not on the
 * inference path: checkpoints arrive quantised. */
bq_status bq_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw,
                          int64_t block_n, int64_t block_k, int dtype, void* q,
                          int64_t ldq, float* s, void* stream);

/* ---- block-scaled GEMM ----------------------------------------- */

/* Bytes of workspace bq_gemm needs for this problem (0 is possible). */
bq_status bq_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int64_t block_n,
                                 int64_t block_k, int dtype, size_t* bytes);

/* out[m, n] = bf16( sum_kb P_kb[m,n] * sa[kb*M + m] * sw[(n/block_n)*Kb + kb]
 *                   + bias[n] )
 * qa: codes [M, K] (row stride lda >= K); sa: fp32 [Kb][M] activation scales
 *   from bq_quant_act with group_k == block_k;
 * qw: codes [N, K] (row stride ldw >= K), sw: fp32 [ceil(N/block_n)][Kb];
 * bias: bf16 [N] or NULL; out: bf16 [M, N] (row stride ldo >= N).
 * block_k <= 65536 keeps INT8 block partials exact in int32.
 * Kernels (BQ_PATH_AUTO): block_n = block_k = 128 with M <= 128 runs the
 *   split-K decode kernel (its K-splits reduced inside thread-block clusters;
 *   split K ranges too long for its shared memory -- K above 65536, or above
 *   32768 for M > 32 -- run the split-K kernel that reduces through the
 *   workspace instead); M > 128 runs the tcgen05 kernel, which promotes
 *   each 128-wide K-block.  block_k >= K (one scale per token and per
 *   block_n rows of W: per-token / per-channel W8A8 with block_n = 1) also
 *   runs the tcgen05 kernel for M > 128, which then accumulates all of K in
 *   tensor memory and promotes once (the int32 sum is rounded once to fp32).
 *   The tensor-core kernels need 16-byte aligned operands with row strides
 *   that are multiples of 16 bytes; everything else runs the CUDA-core
 *   kernel.
 * Stream overlap: the decode kernel starts as a programmatic dependent of
 *   the kernel before it on the stream and requests its weight codes and
 *   scales BEFORE waiting for that kernel to finish (activations, bias and
 *   output are touched only after the wait).  The weights must therefore not
 *   be written by the kernel immediately preceding this call on the stream
 *   (libbq's own bq_quant_weight makes its writes visible before it exits).
 * workspace: device memory of at least bq_gemm_workspace_size bytes (may be
 *   NULL when that size is 0).  Its first 64 KiB hold arrival counters: they
 *   must be zero before the workspace is first used, and every completed
 *   call leaves them zero again, whatever the shape, so one workspace can
 *   serve any sequence of calls.  The rest needs no initialisation.  Every
 *   libbq call that takes a workspace (bq_linear and bq_mx_linear included)
 *   leaves these 64 KiB untouched, so one buffer can be shared by all of
 *   them.  A counter found non-zero at a split's arrival is reported by
 *   bq_check_device_status as invalid device-side input (site 0x406).  Calls
 *   sharing one workspace must not overlap on the GPU; after a call that
 *   reported a device error, zero the counter region again.
 * Block-wise INT8 page sections 2 and 4 (apply_w8a8_block_int8_linear with
 * input_scale=None, after the activation quantisation); blockwise FP8 of the
 * SGLang quantization doc. */
bq_status bq_gemm(const void* qa, int64_t lda, const float* sa, const void* qw, int64_t ldw,
                  const float* sw, int64_t M, int64_t N, int64_t K, int64_t block_n,
                  int64_t block_k, int dtype, const void* bias, void* out, int64_t ldo,
                  void* workspace, size_t workspace_bytes, void* stream);

/* The same contraction as bq_gemm without the last step: out (fp32 [M, N],
 * row stride ldo >= N) = sum_kb P_kb[m,n] * sa[kb*M + m] * sw[(n/block_n)*Kb + kb],
 * unrounded and without bias.  This is the per-GPU part of a linear layer
 * whose K dimension is split over GPUs (row-parallel tensor parallelism,
 * block-wise INT8 page, section 3: each GPU's input_size_per_partition is a
 * multiple of block_k, so its activation groups and weight blocks are whole):
 * the partials of all shards are summed in fp32 (an all-reduce or a
 * reduce-scatter), then bq_finish_bf16 adds the bias and rounds once, as the
 * unsharded layer does.  Arguments and kernels as bq_gemm; the decode path
 * needs the cluster kernel (the fallback is the CUDA-core kernel).  K = 0
 * writes zeros. */
bq_status bq_gemm_partial(const void* qa, int64_t lda, const float* sa, const void* qw,
                          int64_t ldw, const float* sw, int64_t M, int64_t N, int64_t K,
                          int64_t block_n, int64_t block_k, int dtype, float* out, int64_t ldo,
                          void* workspace, size_t workspace_bytes, void* stream);

/* out[m, n] = bf16(part[m, n] + bias[n]) (one round-to-nearest-even; bias
 * bf16 [N] or NULL): the single rounding that ends a K-sharded linear layer
 * after its fp32 partials were summed (see bq_gemm_partial).  part: fp32
 * [M, N] (row stride ldp >= N); out: bf16 [M, N] (row stride ldo >= N). */
bq_status bq_finish_bf16(const float* part, int64_t ldp, int64_t M, int64_t N, const void* bias,
                         void* out, int64_t ldo, void* stream);

/* bq_gemm restricted to the split-K decode kernel, with NO workspace argument
 * and no device allocation: for callers that cannot allocate device memory
 * where they call this -- a plugin inside another engine that owns every
 * device byte, or a serving loop that plans all memory up front and forbids
 * allocation (cudaMalloc can synchronise the device) once it is running.
 * The kernel's scratch (64 KiB of arrival counters plus the split partials)
 * is a fixed 16 MiB device array inside libbq, which every GPU that loads the
 * library holds until the process exits.  Arguments and results are those of
 * bq_gemm; the caller still provides inputs and output.  Limits: M <= 128,
 * block_n = block_k = 128, 16-byte aligned operands and row strides, and a
 * split-K plan whose scratch fits in 16 MiB (e.g. M = 64 with N = K = 4096
 * fits; larger problems return BQ_ERR_UNSUPPORTED with the bytes needed).
 * Each call made outside stream capture looks up the array's device address
 * (so a device reset cannot leave a stale address); a call made while its
 * stream is capturing reuses the last address looked up on that device, so
 * make the first call on each device before any stream capture.  Each call clears the counters
 * it uses.  All calls share the one array, so calls that overlap on the GPU
 * (different streams, or concurrent host threads) race and corrupt each
 * other's results: serialise them.  The pages have no counterpart to this
 * entry point; it exists for callers without an allocator. */
bq_status bq_gemm_decode_noalloc(const void* qa, int64_t lda, const float* sa, const void* qw,
                                 int64_t ldw, const float* sw, int64_t M, int64_t N, int64_t K,
                                 int64_t block_n, int64_t block_k, int dtype, const void* bias,
                                 void* out, int64_t ldo, void* stream);

/* Workspace for bq_linear: bq_gemm's workspace (at offset 0, so the counter
 * rule above applies) followed by the activation codes and scales. */
bq_status bq_linear_workspace_size(int64_t M, int64_t N, int64_t K, int64_t block_n,
                                   int64_t block_k, int dtype, size_t* bytes);

/* The whole linear layer: bq_quant_act(x, group_k = block_k) then bq_gemm,
 * i.e. apply_w8a8_block_int8_linear(input, weight, block_size, weight_scale,
 * input_scale=None, bias) of the block-wise INT8 page, section 4.
 * x: bf16 [M, K] (row stride ldx >= K); other arguments as bq_gemm.  The
 * workspace (bq_linear_workspace_size bytes) follows bq_gemm's rules.  The
 * GEMM starts as a programmatic dependent of the quantiser, so its weight
 * stream overlaps the quantisation (bq_gemm's stream-overlap rule applies). */
bq_status bq_linear(const void* x, int64_t ldx, int64_t M, int64_t K, const void* qw,
                    int64_t ldw, const float* sw, int64_t N, int64_t block_n, int64_t block_k,
                    int dtype, const void* bias, void* out, int64_t ldo, void* workspace,
                    size_t workspace_bytes, void* stream);

/* ---- MoE (block-wise INT8 page, sections 5 and 6) ---------------- */

/* Top-k routing of T tokens over E experts from fp32 router logits [T, E]
 * (row stride ld >= E): topk_ids int32 [T, topk] are the experts of the topk
 * largest logits of each row, in descending order, ties to the lower expert
 * index (the softmax is monotonic, so these are the topk most probable
 * experts); topk_weights fp32 [T, topk] are their softmax probabilities
 * renormalised over the chosen topk, computed as exp(l_j - l_max) divided by
 * the sum over the topk (fp32 expf: within a few ulp of the exact values).
 * These are the topk_ids / topk_weights the MoE runner of the block-wise INT8
 * page (sections 5-6) receives; the pages leave the tie order and the
 * renormalisation open, and this is the reading taken.  E <= 256, topk <= 8. */
bq_status bq_moe_route(const float* logits, int64_t ld, int64_t T, int64_t E, int64_t topk,
                       int32_t* topk_ids, float* topk_weights, void* stream);

/* Bytes of workspace bq_moe_permute needs. */
bq_status bq_moe_permute_workspace_size(int64_t T, int64_t topk, int64_t E, size_t* bytes);

/* Group the T*topk (token, slot) pairs by expert, stably (by expert, then by
 * flat index t*topk + j).  topk_ids: int32 [T, topk], each in [0, E).
 * Writes expert_offsets: int32 [E+1] (exclusive prefix of per-expert counts,
 * expert_offsets[E] = T*topk), perm: int32 [T*topk] (flat pair index at
 * each permuted row) and inv_perm: int32 [T*topk] (permuted row of each
 * pair).  An id outside [0, E) is placed nowhere (expert_offsets[E] then
 * falls short of T*topk) and is recorded in the device status word, which
 * bq_check_device_status reports as BQ_ERR_INVALID_ARG.  Group sizes stay
 * on the device (no host read-back). */
bq_status bq_moe_permute(const int32_t* topk_ids, int64_t T, int64_t topk, int64_t E,
                         int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Activation quantisation of the routed rows: permuted row r holds token
 * perm[r] / topk.  x: bf16 [T, H] (row stride ldx >= H).  Writes q
 * [T*topk, H] (row stride ldq >= H) and s fp32 [ceil(H/group_k)][T*topk].
 * Codes are identical to bq_quant_act of x followed by a row gather. */
bq_status bq_moe_quant_gather(const void* x, int64_t T, int64_t H, int64_t ldx,
                              const int32_t* perm, int64_t topk, int64_t group_k, int dtype,
                              void* q, int64_t ldq, float* s, void* stream);

/* Bytes of workspace bq_grouped_gemm needs. */
bq_status bq_grouped_gemm_workspace_size(int64_t R, int64_t N, int64_t K, int64_t E,
                                         int64_t block_n, int64_t block_k, int dtype,
                                         size_t* bytes);

/* Per expert e, rows [expert_offsets[e], expert_offsets[e+1]) of qa run the
 * block-scaled GEMM against expert e's weight:
 * qa: codes [R, K] (row stride lda), sa: fp32 [Kb][R];
 * expert_offsets: DEVICE int32 [E+1], nondecreasing, offsets[0] = 0,
 *   offsets[E] <= R (rows past offsets[E] are left untouched);
 * qw: codes [E, N, K] (dense), sw: fp32 [E][Nbs][Kb] with Nbs weight-scale
 *   rows per expert;
 * n_seam: 0 for a plain weight (Nbs = ceil(N/block_n)); for a fused gate+up
 *   weight the gate/up boundary I (= N/2): rows [0, I) use scale row n/bn and
 *   rows [I, N) use ceil(I/bn) + (n-I)/bn, so Nbs = 2*ceil(I/bn)
 *   (block-wise INT8 page, section 5);
 * out: bf16 [R, N] (row stride ldo >= N). */
bq_status bq_grouped_gemm(const void* qa, int64_t lda, const float* sa, int64_t R,
                          const int32_t* expert_offsets, int64_t E, const void* qw,
                          const float* sw, int64_t N, int64_t K, int64_t block_n,
                          int64_t block_k, int64_t n_seam, int dtype, void* out, int64_t ldo,
                          void* workspace, size_t workspace_bytes, void* stream);

/* The w13 grouped GEMM fused with the SiLU * up requantisation (block-wise
 * INT8 page, section 5: the gate+up weight, then the activation quantisation
 * of the down projection's input).  For each expert e and each row r in
 * [expert_offsets[e], expert_offsets[e+1]):
 *   y[r, :] = bf16(block-scaled GEMM of qa[r] against qw13[e])  (as bq_grouped_gemm
 *             with n_seam = I: gate rows [0, I), up rows [I, 2I));
 *   h[r, i] = bf16(silu(y[r, i]) * y[r, I + i])                  (as bq_moe_silu_mul_quant);
 *   q[r, :], s[:, r] = the 1 x 128 quantisation of h[r, :]        (as bq_quant_act).
 * y and h are never stored: the tensor-core epilogue holds a tile's gate and
 * up columns in registers.  The codes and scales are bit-identical to
 * bq_grouped_gemm followed by bq_moe_silu_mul_quant with group_k = 128.
 * qa: codes [R, K] (row stride lda), sa: fp32 [ceil(K/128)][R];
 * qw13: codes [E, 2I, K] (dense), sw13: fp32 [E][2I/128][ceil(K/128)];
 * q: codes [R, I] (row stride ldq, a multiple of 16; q 16-byte aligned),
 * s: fp32 [I/128][R].  Rows past expert_offsets[E] are left untouched.
 * Needs block_n = block_k = 128, I a multiple of 128, and the tensor-core
 * path (BQ_PATH_AUTO or one of the BQ_PATH_TCGEN05 paths); otherwise
 * BQ_ERR_UNSUPPORTED, and the caller runs the two unfused calls.  Needs no
 * workspace. */
bq_status bq_grouped_gemm_silu_quant(const void* qa, int64_t lda, const float* sa, int64_t R,
                                     const int32_t* expert_offsets, int64_t E, const void* qw13,
                                     const float* sw13, int64_t I, int64_t K, int64_t block_n,
                                     int64_t block_k, int dtype, void* q, int64_t ldq, float* s,
                                     void* stream);

/* The w2 grouped GEMM fused with the weighted top-k combine (block-wise INT8
 * page, sections 5-6: the down projection, then each token's top-k expert
 * outputs summed with their routing weights).  For each expert e and each
 * row r in [expert_offsets[e], expert_offsets[e+1]), with p = perm[r] the
 * row's (token, slot) pair t * topk + j:
 *   y[r, :] = bf16(block-scaled GEMM of qa[r] against qw[e])  (as bq_grouped_gemm);
 *   acc[t, :] += fp32(topk_w[p] * y[r, :])                      (fp32 atomic add).
 * y is never stored.  acc: fp32 [T, N], T = R / topk (row stride ld_acc >= N;
 * 16-byte aligned rows take vector atomics), must hold zeros on entry;
 * bq_moe_combine_finish then rounds it once to bf16 and zeroes it again.
 * Every sum starts from zero, so with topk <= 2 the atomic order cannot
 * change it: out = bf16(fp32(w0*y0) + fp32(w1*y1)), deterministic.  With
 * topk > 2 the fp32 sum's association follows the atomic order (each result
 * is within the fp32 rounding of the sum, not bit-reproducible).
 * qa: codes [R, K] (row stride lda), sa: fp32 [ceil(K/128)][R]; qw: codes
 * [E, N, K] (dense), sw: fp32 [E][ceil(N/128)][ceil(K/128)]; perm: int32 [R]
 * as bq_moe_permute writes it (an entry outside [0, R) is skipped and
 * recorded in the device status word as BQ_ERR_INVALID_ARG); topk_w: fp32
 * [T, topk].  Rows past expert_offsets[E] add nothing.  Needs R a multiple
 * of topk, block_n = block_k = 128 (or block_k >= K) and the tensor-core
 * path (BQ_PATH_AUTO or one of the BQ_PATH_TCGEN05 paths); otherwise
 * BQ_ERR_UNSUPPORTED.  Needs no workspace. */
bq_status bq_grouped_gemm_combine(const void* qa, int64_t lda, const float* sa, int64_t R,
                                  const int32_t* expert_offsets, int64_t E, const void* qw,
                                  const float* sw, int64_t N, int64_t K, int64_t block_n,
                                  int64_t block_k, int dtype, const int32_t* perm,
                                  const float* topk_w, int64_t topk, float* acc, int64_t ld_acc,
                                  void* stream);

/* out[t, n] = bf16(acc[t, n]) (round to nearest even), then acc[t, n] = 0,
 * for the fp32 sums bq_grouped_gemm_combine accumulated.  acc: fp32 [T, N]
 * (row stride ld_acc >= N), out: bf16 [T, N] (row stride ldo >= N). */
bq_status bq_moe_combine_finish(float* acc, int64_t T, int64_t N, int64_t ld_acc, void* out,
                                int64_t ldo, void* stream);

/* ---------------- MXFP8 dense linear ----------------
 * The SGLang quantization doc ("GEMM backends for FP4/FP8") lists an MXFP8
 * dense linear beside the blockwise FP8 GEMM but does not define the format;
 * the reading here is the microscaling format the name refers to.  Groups of
 * 32 consecutive elements along K share a scale 2^(E - 127), E an 8-bit
 * exponent (E8M0); elements are e4m3 codes.  Quantisation of a group:
 * se = clamp(floor(log2 amax) - 8, -127, 127), E = se + 127, code =
 * e4m3_rne_satfinite(x * 2^-se); an all-zero group has E = 0 and zero codes.
 * Scale arrays use the tensor-core layout: rows in blocks of 128 and K in
 * blocks of 128 (4 groups); each (row block, K block) is one 512-byte atom,
 * atoms row-block major; row r, group g sits at byte
 * 16*(r%32) + 4*((r%128)/32) + g%4 of its atom.  Bytes of rows past the last
 * row are never written nor used.  K must be a multiple of 128. */

/* Bytes of the scale array of R rows: ceil(R/128) * (K/128) * 512.
 * BQ_ERR_UNSUPPORTED if K is not a multiple of 128. */
bq_status bq_mx_scale_bytes(int64_t R, int64_t K, size_t* bytes);

/* MX quantisation of bf16 activations x [M, K] (row stride ldx) into e4m3
 * codes q [M, K] (row stride ldq, 4-byte aligned rows) and the scale array
 * sf (bq_mx_scale_bytes(M, K) bytes). */
bq_status bq_mx_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, void* q,
                          int64_t ldq, void* sf, void* stream);

/* The same rule for fp32 weights w [N, K] (offline; row stride ldw). */
bq_status bq_mx_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw, void* q,
                             int64_t ldq, void* sf, void* stream);

/* out[m, n] = bf16( sum_g 2^(Ea[m,g]-127) * 2^(Ew[n,g]-127) * sum_{k in g} a[m,k]*w[n,k]
 *                   + bias[n] ), fp32 accumulation on the block-scaled tensor
 * cores (tcgen05.mma kind::mxf8f6f4.block_scale; the scales are applied
 * inside the MMA).  qa e4m3 [M, K] (row stride lda), sfa its scale array;
 * qw e4m3 [N, K] (row stride ldw), sfw its scale array; bias bf16 [N] or
 * NULL; out bf16 [M, N] (row stride ldo).  Needs K a positive multiple of
 * 128, lda and ldw multiples of 16, and 16-byte aligned qa, qw, sfa, sfw
 * (else BQ_ERR_UNSUPPORTED / BQ_ERR_ALIGNMENT), and the tensor-core path
 * (BQ_PATH_AUTO or one of the BQ_PATH_TCGEN05 paths).  No workspace. */
bq_status bq_mx_gemm(const void* qa, int64_t lda, const void* sfa, const void* qw, int64_t ldw,
                     const void* sfw, int64_t M, int64_t N, int64_t K, const void* bias,
                     void* out, int64_t ldo, void* stream);

/* Workspace for bq_mx_linear: the activation codes (rows padded to 16 bytes)
 * and their scale atoms. */
bq_status bq_mx_linear_workspace_size(int64_t M, int64_t K, size_t* bytes);

/* The MXFP8 dense linear layer: bq_mx_quant_act of x (bf16 [M, K], row stride
 * ldx) into the workspace, then bq_mx_gemm against qw / sfw (from
 * bq_mx_quant_weight).  Same requirements as those two calls; workspace:
 * bq_mx_linear_workspace_size bytes, 16-byte aligned, no initialisation.
 * The codes start 64 KiB into the workspace: its first 64 KiB are left
 * untouched, so the same buffer can also serve bq_gemm / bq_linear. */
bq_status bq_mx_linear(const void* x, int64_t ldx, int64_t M, int64_t K, const void* qw,
                       int64_t ldw, const void* sfw, int64_t N, const void* bias, void* out,
                       int64_t ldo, void* workspace, size_t workspace_bytes, void* stream);

/* h = bf16(silu(y[r, i]) * y[r, I + i]) (gate then up, block-wise INT8
 * page section 5 "gate + up fused"; SiLU is the reading for a gate/up pair),
 * then the activation quantisation of h with 1 x group_k groups.
 * y: bf16 [R, 2I] (row stride ldy >= 2I).  Writes q [R, I] (row stride
 * ldq >= I), s fp32 [ceil(I/group_k)][R] and, if h_out is not NULL, h as
 * bf16 [R, I] (dense). */
bq_status bq_moe_silu_mul_quant(const void* y, int64_t ldy, int64_t R, int64_t I,
                                int64_t group_k, int dtype, void* q, int64_t ldq, float* s,
                                void* h_out, void* stream);

/* out[t, n] = bf16( sum_j topk_w[t*topk + j] * y[inv_perm[t*topk + j], n] ),
 * fp32 accumulation, one rounding.  y: bf16 [T*topk, H] (row stride ldy),
 * topk_w: fp32 [T, topk], out: bf16 [T, H] (row stride ldo). */
bq_status bq_moe_combine(const void* y, int64_t ldy, const int32_t* inv_perm,
                         const float* topk_w, int64_t T, int64_t topk, int64_t H, void* out,
                         int64_t ldo, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H_ */
