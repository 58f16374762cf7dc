// api.cu -- the extern "C" boundary of libbq (declared in include/bq.h).
//
// Every entry point validates its arguments on the host before enqueueing any
// work, mirroring the block-wise INT8 page's ValueErrors (section 1: two-
// dimensional block size, dynamic activations, int8-serialised checkpoint;
// section 3: tensor-parallel block alignment), then chooses a kernel family.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "bq.h"
#include "bq_common.cuh"
#include "bq_internal.h"
#include "gemm_decode.h"
#include "gemm_mx.h"
#include "gemm_paths.h"
#include "gemm_tc.h"

namespace {

thread_local char g_msg[512] = "";
thread_local int g_path = BQ_PATH_AUTO;

bq_status fail(bq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

bq_status ok() {
  g_msg[0] = '\0';
  return BQ_OK;
}

bq_status cuda_fail(cudaError_t e, const char* where) {
  return fail(BQ_ERR_CUDA, "%s: CUDA error %d (%s)", where, (int)e, cudaGetErrorString(e));
}

#define BQ_CHECK_ARG(cond, ...) \
  do {                          \
    if (!(cond)) return fail(BQ_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define BQ_CHECK_CUDA(expr, where)             \
  do {                                         \
    cudaError_t e_ = (expr);                   \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device status word: one per device, its address fetched once per device.
__device__ unsigned g_bq_status_word;
constexpr int kMaxDevices = 64;
unsigned* g_status_ptr[kMaxDevices] = {};

std::mutex g_status_mu;

bq_status status_word(unsigned** out) {
  int dev = 0;
  BQ_CHECK_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BQ_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    BQ_CHECK_CUDA(cudaGetSymbolAddress(&p, g_bq_status_word), "cudaGetSymbolAddress");
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_status_ptr[dev];
  return BQ_OK;
}

bool valid_dtype(int d) { return d == BQ_INT8 || d == BQ_FP8_E4M3; }

}  // namespace

extern "C" {

int bq_version(void) { return 100; }

const char* bq_status_string(int s) {
  switch (s) {
    case BQ_OK: return "ok";
    case BQ_ERR_INVALID_ARG: return "invalid argument";
    case BQ_ERR_UNSUPPORTED: return "unsupported";
    case BQ_ERR_ALIGNMENT: return "alignment";
    case BQ_ERR_WORKSPACE: return "workspace";
    case BQ_ERR_CUDA: return "cuda error";
    case BQ_ERR_DEVICE_TIMEOUT: return "device timeout";
    default: return "unknown status";
  }
}

const char* bq_last_error_message(void) { return g_msg; }

// Paths that run the tensor-core kernels; the tile shape a forced path picks.
static bool tc_path(int path) {
  return path == BQ_PATH_AUTO || path == BQ_PATH_TCGEN05 || path == BQ_PATH_TCGEN05_1CTA ||
         path == BQ_PATH_TCGEN05_PAIR;
}

static int tc_shape(int path) {
  return path == BQ_PATH_TCGEN05_1CTA ? 1 : path == BQ_PATH_TCGEN05_PAIR ? 2 : 0;
}

bq_status bq_set_path(int path) {
  BQ_CHECK_ARG(path >= BQ_PATH_AUTO && path <= BQ_PATH_TCGEN05_PAIR, "unknown path %d", path);
  g_path = path;
  return ok();
}

int bq_get_path(void) { return g_path; }

bq_status bq_check_device_status(void* stream) {
  unsigned* w = nullptr;
  bq_status st = status_word(&w);
  if (st != BQ_OK) return st;
  unsigned h = 0;
  BQ_CHECK_CUDA(cudaStreamSynchronize(as_stream(stream)), "cudaStreamSynchronize");
  BQ_CHECK_CUDA(cudaMemcpy(&h, w, sizeof(h), cudaMemcpyDeviceToHost), "status read");
  if (h == 0) return ok();
  const unsigned zero = 0;
  BQ_CHECK_CUDA(cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice), "status clear");
  const unsigned kind = h & 0xFFu, site = h >> 8;
  if (kind == bq::kStatusTimeout)
    return fail(BQ_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up (site 0x%x)", site);
  return fail(BQ_ERR_INVALID_ARG, "invalid device-side input (site 0x%x)", site);
}

bq_status bq_selftest_bounded_wait(int64_t spin_limit, void* stream) {
  BQ_CHECK_ARG(spin_limit >= 1 && spin_limit <= (int64_t)1 << 26,
               "spin_limit must be in [1, 2^26], got %lld", (long long)spin_limit);
  unsigned* w = nullptr;
  bq_status st = status_word(&w);
  if (st != BQ_OK) return st;
  BQ_CHECK_CUDA(bq::launch_selftest_wait(spin_limit, w, as_stream(stream)), "selftest launch");
  return ok();
}

bq_status bq_check_block_config(int has_block_size, int checkpoint_int8_serialized,
                                int64_t n_block_dims, int dynamic_activation) {
  if (!has_block_size) return ok();
  BQ_CHECK_ARG(checkpoint_int8_serialized,
               "block-wise quantisation only supports an int8-serialised checkpoint");
  BQ_CHECK_ARG(n_block_dims == 2, "the weight block size must have 2 dimensions, got %lld",
               (long long)n_block_dims);
  BQ_CHECK_ARG(dynamic_activation, "block-wise quantisation only supports dynamic activations");
  return ok();
}

bq_status bq_check_tp_partition(int64_t tp_size, int64_t input_size,
                                int64_t input_size_per_partition,
                                const int64_t* output_partition_sizes, int64_t n_parts,
                                int64_t block_n, int64_t block_k) {
  BQ_CHECK_ARG(tp_size >= 1 && block_n >= 1 && block_k >= 1 && n_parts >= 0,
               "tp_size, block_n and block_k must be >= 1");
  BQ_CHECK_ARG(input_size_per_partition >= 1, "input_size_per_partition must be >= 1");
  BQ_CHECK_ARG(n_parts == 0 || output_partition_sizes != nullptr,
               "output_partition_sizes is NULL");
  if (tp_size > 1 && input_size / input_size_per_partition == tp_size) {
    BQ_CHECK_ARG(input_size_per_partition % block_k == 0,
                 "weight input_size_per_partition = %lld is not divisible by weight "
                 "quantization block_k = %lld",
                 (long long)input_size_per_partition, (long long)block_k);
  }
  for (int64_t i = 0; i < n_parts; ++i) {
    BQ_CHECK_ARG(output_partition_sizes[i] % block_n == 0,
                 "weight output_partition_size = %lld is not divisible by weight "
                 "quantization block_n = %lld",
                 (long long)output_partition_sizes[i], (long long)block_n);
  }
  return ok();
}

bq_status bq_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, int64_t group_k,
                       int dtype, void* q, int64_t ldq, float* s, void* stream) {
  BQ_CHECK_ARG(valid_dtype(dtype), "unknown dtype %d", dtype);
  BQ_CHECK_ARG(M >= 0 && K >= 0, "M and K must be >= 0");
  BQ_CHECK_ARG(group_k >= 1, "group_k must be >= 1, got %lld", (long long)group_k);
  BQ_CHECK_ARG(ldx >= K && ldq >= K, "leading dimensions must be >= K");
  if (M == 0 || K == 0) return ok();
  BQ_CHECK_ARG(x && q && s, "x, q and s must not be NULL");
  BQ_CHECK_CUDA(bq::launch_quant_act(x, M, K, ldx, nullptr, 1, group_k, dtype, q, ldq, s,
                                     as_stream(stream)),
                "quant_act launch");
  return ok();
}

bq_status bq_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw, int64_t block_n,
                          int64_t block_k, int dtype, void* q, int64_t ldq, float* s,
                          void* stream) {
  BQ_CHECK_ARG(valid_dtype(dtype), "unknown dtype %d", dtype);
  BQ_CHECK_ARG(N >= 0 && K >= 0, "N and K must be >= 0");
  BQ_CHECK_ARG(block_n >= 1 && block_k >= 1, "block sizes must be >= 1");
  BQ_CHECK_ARG(ldw >= K && ldq >= K, "leading dimensions must be >= K");
  if (N == 0 || K == 0) return ok();
  BQ_CHECK_ARG(w && q && s, "w, q and s must not be NULL");
  BQ_CHECK_ARG(cdiv(N, block_n) <= 65535, "too many weight block rows");
  BQ_CHECK_CUDA(bq::launch_quant_weight(w, N, K, ldw, block_n, block_k, dtype, q, ldq, s,
                                        as_stream(stream)),
                "quant_weight launch");
  return ok();
}

static bq_status check_gemm_shape(int64_t M, int64_t N, int64_t K, int64_t block_n,
                                  int64_t block_k, int dtype) {
  BQ_CHECK_ARG(valid_dtype(dtype), "unknown dtype %d", dtype);
  BQ_CHECK_ARG(M >= 0 && N >= 0 && K >= 0, "M, N and K must be >= 0");
  BQ_CHECK_ARG(block_n >= 1 && block_k >= 1, "block_n and block_k must be >= 1");
  if (block_k > 65536)
    return fail(BQ_ERR_UNSUPPORTED, "block_k = %lld > 65536 would overflow int32 partials",
                (long long)block_k);
  return BQ_OK;
}

bq_status bq_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int64_t block_n,
                                 int64_t block_k, int dtype, size_t* bytes) {
  bq_status st = check_gemm_shape(M, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(bytes, "bytes must not be NULL");
  *bytes = bq::gemm_workspace_bytes(M, N, K, block_n, block_k, dtype);
  return ok();
}

static bq_status gemm_impl(const void* qa, int64_t lda, const float* sa, const void* qw,
                           int64_t ldw, const float* sw, int64_t M, int64_t N, int64_t K,
                           int64_t block_n, int64_t block_k, int dtype, const void* bias,
                           void* out, int64_t ldo, void* workspace, size_t workspace_bytes,
                           void* stream, bool after_quant) {
  bq_status st = check_gemm_shape(M, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(lda >= K && ldw >= K && ldo >= N, "leading dimensions too small");
  if (M == 0 || N == 0) return ok();
  BQ_CHECK_ARG(out, "out must not be NULL");
  BQ_CHECK_ARG(K == 0 || (qa && sa && qw && sw), "qa, sa, qw and sw must not be NULL");
  const size_t need = bq::gemm_workspace_bytes(M, N, K, block_n, block_k, dtype);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(BQ_ERR_WORKSPACE, "bq_gemm needs %zu workspace bytes, got %zu", need,
                workspace ? workspace_bytes : (size_t)0);
  unsigned* w = nullptr;
  st = status_word(&w);
  if (st != BQ_OK) return st;
  bq::GemmArgs a{};
  a.qa = qa; a.lda = lda; a.sa = sa; a.sa_rows = M;
  a.qw = qw; a.ldw = ldw; a.sw = sw;
  a.M = M; a.N = N; a.K = K; a.bn = block_n; a.bk = block_k; a.seam = 0;
  a.Nbs = cdiv(N, block_n);
  a.dtype = dtype; a.bias = bias; a.out = out; a.ldo = ldo;
  a.offsets = nullptr; a.E = 1; a.w_expert_stride = 0; a.sw_expert_stride = 0;
  a.status = w;
  char why[256] = "";
  const int rc = after_quant ? bq::run_gemm_after_quant(a, g_path, workspace, workspace_bytes,
                                                        as_stream(stream), why, sizeof(why))
                             : bq::run_gemm(a, g_path, workspace, workspace_bytes,
                                            as_stream(stream), why, sizeof(why));
  if (rc == bq::kRunOk) return ok();
  if (rc == bq::kRunUnsupported) return fail(BQ_ERR_UNSUPPORTED, "%s", why);
  if (rc == bq::kRunAlignment) return fail(BQ_ERR_ALIGNMENT, "%s", why);
  return fail(BQ_ERR_CUDA, "%s", why);
}

bq_status bq_gemm_partial(const void* qa, int64_t lda, const float* sa, const void* qw,
                          int64_t ldw, const float* sw, int64_t M, int64_t N, int64_t K,
                          int64_t block_n, int64_t block_k, int dtype, float* out, int64_t ldo,
                          void* workspace, size_t workspace_bytes, void* stream) {
  bq_status st = check_gemm_shape(M, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(lda >= K && ldw >= K && ldo >= N, "leading dimensions too small");
  if (M == 0 || N == 0) return ok();
  BQ_CHECK_ARG(out, "out must not be NULL");
  if (K == 0) {
    for (int64_t m = 0; m < M; ++m)
      BQ_CHECK_CUDA(cudaMemsetAsync(out + m * ldo, 0, (size_t)N * sizeof(float), as_stream(stream)),
                    "zero partial");
    return ok();
  }
  BQ_CHECK_ARG(qa && sa && qw && sw, "qa, sa, qw and sw must not be NULL");
  unsigned* w = nullptr;
  st = status_word(&w);
  if (st != BQ_OK) return st;
  bq::GemmArgs a{};
  a.qa = qa; a.lda = lda; a.sa = sa; a.sa_rows = M;
  a.qw = qw; a.ldw = ldw; a.sw = sw;
  a.M = M; a.N = N; a.K = K; a.bn = block_n; a.bk = block_k; a.seam = 0;
  a.Nbs = cdiv(N, block_n);
  a.dtype = dtype; a.bias = nullptr; a.out = nullptr; a.ldo = ldo;
  a.offsets = nullptr; a.E = 1; a.w_expert_stride = 0; a.sw_expert_stride = 0;
  a.status = w;
  a.out_f32 = out;
  char why[256] = "";
  const int rc = bq::run_gemm(a, g_path, workspace, workspace_bytes, as_stream(stream), why,
                              sizeof(why));
  if (rc == bq::kRunOk) return ok();
  if (rc == bq::kRunUnsupported) return fail(BQ_ERR_UNSUPPORTED, "%s", why);
  if (rc == bq::kRunAlignment) return fail(BQ_ERR_ALIGNMENT, "%s", why);
  return fail(BQ_ERR_CUDA, "%s", why);
}

bq_status bq_finish_bf16(const float* part, int64_t ldp, int64_t M, int64_t N, const void* bias,
                         void* out, int64_t ldo, void* stream) {
  BQ_CHECK_ARG(M >= 0 && N >= 0, "M and N must be >= 0");
  BQ_CHECK_ARG(ldp >= N && ldo >= N, "leading dimensions too small");
  if (M == 0 || N == 0) return ok();
  BQ_CHECK_ARG(part && out, "part and out must not be NULL");
  BQ_CHECK_CUDA(bq::launch_finish_bf16(part, ldp, M, N, bias, out, ldo, as_stream(stream)),
                "finish_bf16 launch");
  return ok();
}

bq_status bq_gemm(const void* qa, int64_t lda, const float* sa, const void* qw, int64_t ldw,
                  const float* sw, int64_t M, int64_t N, int64_t K, int64_t block_n,
                  int64_t block_k, int dtype, const void* bias, void* out, int64_t ldo,
                  void* workspace, size_t workspace_bytes, void* stream) {
  return gemm_impl(qa, lda, sa, qw, ldw, sw, M, N, K, block_n, block_k, dtype, bias, out, ldo,
                   workspace, workspace_bytes, stream, false);
}

// bq_linear workspace: [GEMM workspace, at least the 64 KiB counter region]
// [activation codes M x ldq] [activation scales Kb x M].
static void linear_layout(int64_t M, int64_t N, int64_t K, int64_t block_n, int64_t block_k,
                          int dtype, size_t* gemm_bytes, size_t* q_off, size_t* s_off,
                          size_t* total, int64_t* ldq) {
  *ldq = (int64_t)round_up((size_t)K, 16);
  // the GEMM region always spans at least the counter region, so activation
  // codes never land where a later decode call expects zeroed counters
  *gemm_bytes = round_up(std::max(bq::gemm_workspace_bytes(M, N, K, block_n, block_k, dtype),
                                  bq::kDecodeCounterBytes),
                         256);
  *q_off = *gemm_bytes;
  *s_off = *q_off + round_up((size_t)(M * *ldq), 256);
  *total = *s_off + round_up((size_t)(cdiv(K, block_k) * M) * sizeof(float), 256);
}

bq_status bq_gemm_decode_noalloc(const void* qa, int64_t lda, const float* sa, const void* qw,
                                 int64_t ldw, const float* sw, int64_t M, int64_t N, int64_t K,
                                 int64_t block_n, int64_t block_k, int dtype, const void* bias,
                                 void* out, int64_t ldo, void* stream) {
  bq_status st = check_gemm_shape(M, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(lda >= K && ldw >= K && ldo >= N, "leading dimensions too small");
  if (M == 0 || N == 0) return ok();
  BQ_CHECK_ARG(out && qa && sa && qw && sw, "qa, sa, qw, sw and out must not be NULL");
  unsigned* w = nullptr;
  st = status_word(&w);
  if (st != BQ_OK) return st;
  bq::GemmArgs a{};
  a.qa = qa; a.lda = lda; a.sa = sa; a.sa_rows = M;
  a.qw = qw; a.ldw = ldw; a.sw = sw;
  a.M = M; a.N = N; a.K = K; a.bn = block_n; a.bk = block_k; a.seam = 0;
  a.Nbs = cdiv(N, block_n);
  a.dtype = dtype; a.bias = bias; a.out = out; a.ldo = ldo;
  a.offsets = nullptr; a.E = 1; a.w_expert_stride = 0; a.sw_expert_stride = 0;
  a.status = w;
  char why[256] = "";
  if (!bq::decode_supported(a, why, sizeof(why))) return fail(BQ_ERR_UNSUPPORTED, "%s", why);
  const bq::DecodePlan plan = bq::decode_plan(M, N, K);
  if (plan.ws_bytes > bq::kNoAllocScratchBytes)
    return fail(BQ_ERR_UNSUPPORTED,
                "this problem needs %zu bytes of scratch; the fixed scratch of "
                "bq_gemm_decode_noalloc holds %zu (use bq_gemm with a workspace)",
                plan.ws_bytes, bq::kNoAllocScratchBytes);
  void* scratch = nullptr;
  BQ_CHECK_CUDA(bq::noalloc_scratch(&scratch, as_stream(stream)), "static scratch address");
  if (plan.ws_bytes > 0) {
    // arrival counters must start at zero; the partials need no clearing
    BQ_CHECK_CUDA(cudaMemsetAsync(scratch, 0, (size_t)plan.tiles * sizeof(unsigned),
                                  as_stream(stream)),
                  "scratch counter clear");
  }
  BQ_CHECK_CUDA(bq::launch_gemm_decode(a, scratch, false, as_stream(stream)),
                "decode GEMM launch");
  return ok();
}

bq_status bq_linear_workspace_size(int64_t M, int64_t N, int64_t K, int64_t block_n,
                                   int64_t block_k, int dtype, size_t* bytes) {
  bq_status st = check_gemm_shape(M, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(bytes, "bytes must not be NULL");
  size_t g, qo, so, tot;
  int64_t ldq;
  linear_layout(M, N, K, block_n, block_k, dtype, &g, &qo, &so, &tot, &ldq);
  *bytes = tot;
  return ok();
}

bq_status bq_linear(const void* x, int64_t ldx, int64_t M, int64_t K, const void* qw,
                    int64_t ldw, const float* sw, int64_t N, int64_t block_n, int64_t block_k,
                    int dtype, const void* bias, void* out, int64_t ldo, void* workspace,
                    size_t workspace_bytes, void* stream) {
  bq_status st = check_gemm_shape(M, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(ldx >= K && ldw >= K && ldo >= N, "leading dimensions too small");
  if (M == 0 || N == 0) return ok();
  BQ_CHECK_ARG(out, "out must not be NULL");
  BQ_CHECK_ARG(K == 0 || (x && qw && sw), "x, qw and sw must not be NULL");
  size_t g, qo, so, need;
  int64_t ldq;
  linear_layout(M, N, K, block_n, block_k, dtype, &g, &qo, &so, &need, &ldq);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(BQ_ERR_WORKSPACE, "bq_linear needs %zu workspace bytes, got %zu", need,
                workspace ? workspace_bytes : (size_t)0);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  void* q = base + qo;
  float* s = reinterpret_cast<float*>(base + so);
  if (K > 0) {
    BQ_CHECK_CUDA(bq::launch_quant_act(x, M, K, ldx, nullptr, 1, block_k, dtype, q, ldq, s,
                                       as_stream(stream)),
                  "quant_act launch");
  }
  return gemm_impl(q, ldq, s, qw, ldw, sw, M, N, K, block_n, block_k, dtype, bias, out, ldo,
                   base, g, stream, true);
}

bq_status bq_moe_route(const float* logits, int64_t ld, int64_t T, int64_t E, int64_t topk,
                       int32_t* topk_ids, float* topk_weights, void* stream) {
  BQ_CHECK_ARG(T >= 0 && E >= 1 && topk >= 1, "need T >= 0, E >= 1, topk >= 1");
  BQ_CHECK_ARG(topk <= E, "topk (%lld) exceeds E (%lld)", (long long)topk, (long long)E);
  BQ_CHECK_ARG(ld >= E, "ld must be >= E");
  if (E > 256 || topk > 8)
    return fail(BQ_ERR_UNSUPPORTED, "routing supports E <= 256 and topk <= 8");
  if (T == 0) return ok();
  BQ_CHECK_ARG(logits && topk_ids && topk_weights, "logits, ids and weights must not be NULL");
  BQ_CHECK_CUDA(bq::launch_moe_route(logits, ld, T, E, topk, topk_ids, topk_weights,
                                     as_stream(stream)),
                "moe_route launch");
  return ok();
}

bq_status bq_moe_permute_workspace_size(int64_t T, int64_t topk, int64_t E, size_t* bytes) {
  BQ_CHECK_ARG(T >= 0 && topk >= 1 && E >= 1, "need T >= 0, topk >= 1, E >= 1");
  BQ_CHECK_ARG(bytes, "bytes must not be NULL");
  *bytes = 0;
  return ok();
}

bq_status bq_moe_permute(const int32_t* topk_ids, int64_t T, int64_t topk, int64_t E,
                         int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                         void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  BQ_CHECK_ARG(T >= 0 && topk >= 1 && E >= 1, "need T >= 0, topk >= 1, E >= 1");
  if (E > 256) return fail(BQ_ERR_UNSUPPORTED, "at most 256 experts, got %lld", (long long)E);
  BQ_CHECK_ARG(T * topk <= INT32_MAX, "T*topk must fit in int32");
  BQ_CHECK_ARG(expert_offsets, "expert_offsets must not be NULL");
  BQ_CHECK_ARG(T == 0 || (topk_ids && perm && inv_perm), "ids/perm/inv_perm must not be NULL");
  unsigned* w = nullptr;
  bq_status st = status_word(&w);
  if (st != BQ_OK) return st;
  BQ_CHECK_CUDA(bq::launch_moe_permute(topk_ids, T, topk, E, expert_offsets, perm, inv_perm, w,
                                       as_stream(stream)),
                "moe_permute launch");
  return ok();
}

bq_status bq_moe_quant_gather(const void* x, int64_t T, int64_t H, int64_t ldx,
                              const int32_t* perm, int64_t topk, int64_t group_k, int dtype,
                              void* q, int64_t ldq, float* s, void* stream) {
  BQ_CHECK_ARG(valid_dtype(dtype), "unknown dtype %d", dtype);
  BQ_CHECK_ARG(T >= 0 && H >= 0 && topk >= 1, "need T >= 0, H >= 0, topk >= 1");
  BQ_CHECK_ARG(group_k >= 1, "group_k must be >= 1");
  BQ_CHECK_ARG(ldx >= H && ldq >= H, "leading dimensions must be >= H");
  if (T == 0 || H == 0) return ok();
  BQ_CHECK_ARG(x && perm && q && s, "x, perm, q and s must not be NULL");
  BQ_CHECK_CUDA(bq::launch_quant_act(x, T * topk, H, ldx, perm, topk, group_k, dtype, q, ldq,
                                     s, as_stream(stream)),
                "moe_quant_gather launch");
  return ok();
}

bq_status bq_grouped_gemm_workspace_size(int64_t R, int64_t N, int64_t K, int64_t E,
                                         int64_t block_n, int64_t block_k, int dtype,
                                         size_t* bytes) {
  bq_status st = check_gemm_shape(R, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(E >= 1, "E must be >= 1");
  BQ_CHECK_ARG(bytes, "bytes must not be NULL");
  *bytes = bq::grouped_workspace_bytes(R, N, K, E, block_n, block_k, dtype);
  return ok();
}

bq_status bq_grouped_gemm(const void* qa, int64_t lda, const float* sa, int64_t R,
                          const int32_t* expert_offsets, int64_t E, const void* qw,
                          const float* sw, int64_t N, int64_t K, int64_t block_n,
                          int64_t block_k, int64_t n_seam, int dtype, void* out, int64_t ldo,
                          void* workspace, size_t workspace_bytes, void* stream) {
  bq_status st = check_gemm_shape(R, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(E >= 1 && E <= 65535, "E must be in [1, 65535]");
  BQ_CHECK_ARG(lda >= K && ldo >= N, "leading dimensions too small");
  BQ_CHECK_ARG(n_seam >= 0 && n_seam <= N, "n_seam must be in [0, N]");
  if (R == 0 || N == 0) return ok();
  BQ_CHECK_ARG(out && expert_offsets, "out and expert_offsets must not be NULL");
  BQ_CHECK_ARG(K == 0 || (qa && sa && qw && sw), "qa, sa, qw and sw must not be NULL");
  const size_t need = bq::grouped_workspace_bytes(R, N, K, E, block_n, block_k, dtype);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(BQ_ERR_WORKSPACE, "bq_grouped_gemm needs %zu workspace bytes, got %zu", need,
                workspace ? workspace_bytes : (size_t)0);
  unsigned* w = nullptr;
  st = status_word(&w);
  if (st != BQ_OK) return st;
  const bool seam = n_seam > 0 && n_seam < N;
  const int64_t Kb = cdiv(K, block_k);
  bq::GemmArgs a{};
  a.qa = qa; a.lda = lda; a.sa = sa; a.sa_rows = R;
  a.qw = qw; a.ldw = K; a.sw = sw;
  a.M = R; a.N = N; a.K = K; a.bn = block_n; a.bk = block_k; a.seam = seam ? n_seam : 0;
  a.Nbs = seam ? cdiv(n_seam, block_n) + cdiv(N - n_seam, block_n) : cdiv(N, block_n);
  a.dtype = dtype; a.bias = nullptr; a.out = out; a.ldo = ldo;
  a.offsets = expert_offsets; a.E = E;
  a.w_expert_stride = N * K; a.sw_expert_stride = a.Nbs * Kb;
  a.status = w;
  char why[256] = "";
  const int rc = bq::run_grouped_gemm(a, g_path, workspace, workspace_bytes, as_stream(stream),
                                      why, sizeof(why));
  if (rc == bq::kRunOk) return ok();
  if (rc == bq::kRunUnsupported) return fail(BQ_ERR_UNSUPPORTED, "%s", why);
  if (rc == bq::kRunAlignment) return fail(BQ_ERR_ALIGNMENT, "%s", why);
  return fail(BQ_ERR_CUDA, "%s", why);
}

bq_status bq_grouped_gemm_silu_quant(const void* qa, int64_t lda, const float* sa, int64_t R,
                                     const int32_t* expert_offsets, int64_t E, const void* qw13,
                                     const float* sw13, int64_t I, int64_t K, int64_t block_n,
                                     int64_t block_k, int dtype, void* q, int64_t ldq, float* s,
                                     void* stream) {
  BQ_CHECK_ARG(I >= 0, "I must be >= 0");
  bq_status st = check_gemm_shape(R, 2 * I, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(E >= 1 && E <= 65535, "E must be in [1, 65535]");
  BQ_CHECK_ARG(lda >= K && ldq >= I, "leading dimensions too small");
  if (R == 0 || I == 0) return ok();
  BQ_CHECK_ARG(q && s && expert_offsets, "q, s and expert_offsets must not be NULL");
  BQ_CHECK_ARG(K == 0 || (qa && sa && qw13 && sw13), "qa, sa, qw13 and sw13 must not be NULL");
  if (!tc_path(g_path))
    return fail(BQ_ERR_UNSUPPORTED, "the fused SiLU GEMM runs on the tensor-core path only");
  const int64_t Kb = cdiv(K, block_k);
  bq::GemmArgs a{};
  a.qa = qa; a.lda = lda; a.sa = sa; a.sa_rows = R;
  a.qw = qw13; a.ldw = K; a.sw = sw13;
  a.M = R; a.N = 2 * I; a.K = K; a.bn = block_n; a.bk = block_k; a.seam = I;
  a.Nbs = 2 * cdiv(I, block_n);
  a.dtype = dtype; a.bias = nullptr; a.out = nullptr; a.ldo = 0;
  a.offsets = expert_offsets; a.E = E;
  a.w_expert_stride = 2 * I * K; a.sw_expert_stride = a.Nbs * Kb;
  a.q_out = q; a.ldq = ldq; a.s_out = s;
  a.tc_shape = tc_shape(g_path);
  char why[256] = "";
  if (!bq::tc_silu_supported(a, why, sizeof(why))) return fail(BQ_ERR_UNSUPPORTED, "%s", why);
  unsigned* w = nullptr;
  st = status_word(&w);
  if (st != BQ_OK) return st;
  a.status = w;
  BQ_CHECK_CUDA(bq::launch_gemm_tc_silu(a, as_stream(stream)), "fused SiLU GEMM launch");
  return ok();
}

bq_status bq_grouped_gemm_combine(const void* qa, int64_t lda, const float* sa, int64_t R,
                                  const int32_t* expert_offsets, int64_t E, const void* qw,
                                  const float* sw, int64_t N, int64_t K, int64_t block_n,
                                  int64_t block_k, int dtype, const int32_t* perm,
                                  const float* topk_w, int64_t topk, float* acc, int64_t ld_acc,
                                  void* stream) {
  bq_status st = check_gemm_shape(R, N, K, block_n, block_k, dtype);
  if (st != BQ_OK) return st;
  BQ_CHECK_ARG(E >= 1 && E <= 65535, "E must be in [1, 65535]");
  BQ_CHECK_ARG(topk >= 1 && topk <= 65535, "topk must be in [1, 65535]");
  BQ_CHECK_ARG(R % topk == 0, "R must be T * topk");
  BQ_CHECK_ARG(lda >= K && ld_acc >= N, "leading dimensions too small");
  if (R == 0 || N == 0) return ok();
  BQ_CHECK_ARG(acc && perm && topk_w && expert_offsets,
               "acc, perm, topk_w and expert_offsets must not be NULL");
  BQ_CHECK_ARG(K == 0 || (qa && sa && qw && sw), "qa, sa, qw and sw must not be NULL");
  if (!tc_path(g_path))
    return fail(BQ_ERR_UNSUPPORTED, "the combining GEMM runs on the tensor-core path only");
  const int64_t Kb = cdiv(K, block_k);
  bq::GemmArgs a{};
  a.qa = qa; a.lda = lda; a.sa = sa; a.sa_rows = R;
  a.qw = qw; a.ldw = K; a.sw = sw;
  a.M = R; a.N = N; a.K = K; a.bn = block_n; a.bk = block_k; a.seam = 0;
  a.Nbs = cdiv(N, block_n);
  a.dtype = dtype; a.bias = nullptr; a.out = nullptr; a.ldo = ld_acc;
  a.offsets = expert_offsets; a.E = E;
  a.w_expert_stride = N * K; a.sw_expert_stride = a.Nbs * Kb;
  a.comb_acc = acc; a.comb_perm = perm; a.comb_w = topk_w; a.topk = topk;
  a.tc_shape = tc_shape(g_path);
  char why[256] = "";
  if (!bq::tc_supported(a, why, sizeof(why))) return fail(BQ_ERR_UNSUPPORTED, "%s", why);
  unsigned* w = nullptr;
  st = status_word(&w);
  if (st != BQ_OK) return st;
  a.status = w;
  BQ_CHECK_CUDA(bq::launch_gemm_tc(a, as_stream(stream)), "combining grouped GEMM launch");
  return ok();
}

bq_status bq_moe_combine_finish(float* acc, int64_t T, int64_t N, int64_t ld_acc, void* out,
                                int64_t ldo, void* stream) {
  BQ_CHECK_ARG(T >= 0 && N >= 0, "need T >= 0 and N >= 0");
  BQ_CHECK_ARG(ld_acc >= N && ldo >= N, "leading dimensions must be >= N");
  if (T == 0 || N == 0) return ok();
  BQ_CHECK_ARG(acc && out, "acc and out must not be NULL");
  BQ_CHECK_CUDA(bq::launch_moe_combine_finish(acc, T, N, ld_acc, out, ldo, as_stream(stream)),
                "moe_combine_finish launch");
  return ok();
}

// ---------------- MXFP8 ----------------

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bq_status bq_mx_scale_bytes(int64_t R, int64_t K, size_t* bytes) {
  BQ_CHECK_ARG(bytes, "bytes must not be NULL");
  BQ_CHECK_ARG(R >= 0 && K >= 0, "R and K must be >= 0");
  if (K % 128 != 0) return fail(BQ_ERR_UNSUPPORTED, "MXFP8 needs K a multiple of 128");
  *bytes = bq::mx_scale_bytes(R, K);
  return ok();
}

static bq_status mx_quant_check(const void* x, int64_t R, int64_t K, int64_t ldx, void* q,
                                int64_t ldq, void* sf) {
  BQ_CHECK_ARG(R >= 0 && K >= 0, "rows and K must be >= 0");
  BQ_CHECK_ARG(ldx >= K && ldq >= K, "leading dimensions too small");
  if (K % 128 != 0) return fail(BQ_ERR_UNSUPPORTED, "MXFP8 needs K a multiple of 128");
  if (R == 0 || K == 0) return BQ_OK;
  BQ_CHECK_ARG(x && q && sf, "x, q and sf must not be NULL");
  if (ldq % 4 != 0 || (reinterpret_cast<uintptr_t>(q) & 3))
    return fail(BQ_ERR_ALIGNMENT, "MXFP8 codes need 4-byte aligned rows");
  return BQ_OK;
}

bq_status bq_mx_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, void* q,
                          int64_t ldq, void* sf, void* stream) {
  bq_status st = mx_quant_check(x, M, K, ldx, q, ldq, sf);
  if (st != BQ_OK || M == 0 || K == 0) return st == BQ_OK ? ok() : st;
  BQ_CHECK_CUDA(bq::launch_mx_quant_act(x, M, K, ldx, q, ldq, sf, as_stream(stream)),
                "mx_quant_act launch");
  return ok();
}

bq_status bq_mx_quant_weight(const float* w, int64_t N, int64_t K, int64_t ldw, void* q,
                             int64_t ldq, void* sf, void* stream) {
  bq_status st = mx_quant_check(w, N, K, ldw, q, ldq, sf);
  if (st != BQ_OK || N == 0 || K == 0) return st == BQ_OK ? ok() : st;
  BQ_CHECK_CUDA(bq::launch_mx_quant_weight(w, N, K, ldw, q, ldq, sf, as_stream(stream)),
                "mx_quant_weight launch");
  return ok();
}

bq_status bq_mx_gemm(const void* qa, int64_t lda, const void* sfa, const void* qw, int64_t ldw,
                     const void* sfw, int64_t M, int64_t N, int64_t K, const void* bias,
                     void* out, int64_t ldo, void* stream) {
  BQ_CHECK_ARG(M >= 0 && N >= 0 && K >= 0, "M, N and K must be >= 0");
  BQ_CHECK_ARG(lda >= K && ldw >= K && ldo >= N, "leading dimensions too small");
  if (K % 128 != 0 || K == 0)
    return fail(BQ_ERR_UNSUPPORTED, "MXFP8 GEMM needs K a positive multiple of 128");
  if (M == 0 || N == 0) return ok();
  BQ_CHECK_ARG(qa && sfa && qw && sfw && out, "qa, sfa, qw, sfw and out must not be NULL");
  if (!tc_path(g_path))
    return fail(BQ_ERR_UNSUPPORTED, "the MXFP8 GEMM runs on the tensor-core path only");
  if (lda % 16 != 0 || ldw % 16 != 0 || !aligned16(qa) || !aligned16(qw) || !aligned16(sfa) ||
      !aligned16(sfw))
    return fail(BQ_ERR_ALIGNMENT,
                "MXFP8 GEMM: code rows and bases, and the scale arrays, must be 16-byte aligned");
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
    return fail(BQ_ERR_UNSUPPORTED, "sizes exceed int32");
  unsigned* w = nullptr;
  bq_status st = status_word(&w);
  if (st != BQ_OK) return st;
  bq::MxArgs a{};
  a.qa = qa; a.lda = lda; a.sfa = sfa;
  a.qw = qw; a.ldw = ldw; a.sfw = sfw;
  a.M = M; a.N = N; a.K = K; a.bias = bias; a.out = out; a.ldo = ldo; a.status = w;
  BQ_CHECK_CUDA(bq::launch_gemm_mx(a, as_stream(stream)), "MXFP8 GEMM launch");
  return ok();
}

// bq_mx_linear workspace: [64 KiB left untouched] [codes M x ldq] [scale atoms].
// The first kDecodeCounterBytes are skipped, as in bq_linear, so that one
// workspace can serve both calls: the decode GEMM keeps its arrival counters
// there and needs them to stay zero.
static void mx_linear_layout(int64_t M, int64_t K, int64_t* ldq, size_t* q_off, size_t* sf_off,
                             size_t* total) {
  *ldq = (int64_t)round_up((size_t)K, 16);
  *q_off = bq::kDecodeCounterBytes;
  *sf_off = *q_off + round_up((size_t)(M * *ldq), 256);
  *total = *sf_off + round_up(bq::mx_scale_bytes(M, K), 256);
}

bq_status bq_mx_linear_workspace_size(int64_t M, int64_t K, size_t* bytes) {
  BQ_CHECK_ARG(bytes, "bytes must not be NULL");
  BQ_CHECK_ARG(M >= 0 && K >= 0, "M and K must be >= 0");
  if (K % 128 != 0) return fail(BQ_ERR_UNSUPPORTED, "MXFP8 needs K a multiple of 128");
  int64_t ldq;
  size_t qo, so;
  mx_linear_layout(M, K, &ldq, &qo, &so, bytes);
  return ok();
}

bq_status bq_mx_linear(const void* x, int64_t ldx, int64_t M, int64_t K, const void* qw,
                       int64_t ldw, const void* sfw, int64_t N, const void* bias, void* out,
                       int64_t ldo, void* workspace, size_t workspace_bytes, void* stream) {
  BQ_CHECK_ARG(M >= 0 && N >= 0 && K >= 0, "M, N and K must be >= 0");
  BQ_CHECK_ARG(ldx >= K && ldw >= K && ldo >= N, "leading dimensions too small");
  if (K % 128 != 0 || K == 0)
    return fail(BQ_ERR_UNSUPPORTED, "MXFP8 linear needs K a positive multiple of 128");
  if (M == 0 || N == 0) return ok();
  BQ_CHECK_ARG(x && qw && sfw && out, "x, qw, sfw and out must not be NULL");
  int64_t ldq;
  size_t qo, so, need;
  mx_linear_layout(M, K, &ldq, &qo, &so, &need);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(BQ_ERR_WORKSPACE, "bq_mx_linear needs %zu workspace bytes, got %zu", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(BQ_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  uint8_t* base = static_cast<uint8_t*>(workspace);
  bq_status st = bq_mx_quant_act(x, M, K, ldx, base + qo, ldq, base + so, stream);
  if (st != BQ_OK) return st;
  return bq_mx_gemm(base + qo, ldq, base + so, qw, ldw, sfw, M, N, K, bias, out, ldo, stream);
}

bq_status bq_moe_silu_mul_quant(const void* y, int64_t ldy, int64_t R, int64_t I,
                                int64_t group_k, int dtype, void* q, int64_t ldq, float* s,
                                void* h_out, void* stream) {
  BQ_CHECK_ARG(valid_dtype(dtype), "unknown dtype %d", dtype);
  BQ_CHECK_ARG(R >= 0 && I >= 0, "R and I must be >= 0");
  BQ_CHECK_ARG(group_k >= 1, "group_k must be >= 1");
  BQ_CHECK_ARG(ldy >= 2 * I && ldq >= I, "leading dimensions too small");
  if (R == 0 || I == 0) return ok();
  BQ_CHECK_ARG(y && q && s, "y, q and s must not be NULL");
  BQ_CHECK_CUDA(bq::launch_silu_mul_quant(y, ldy, R, I, group_k, dtype, q, ldq, s, h_out,
                                          as_stream(stream)),
                "silu_mul_quant launch");
  return ok();
}

bq_status bq_moe_combine(const void* y, int64_t ldy, const int32_t* inv_perm,
                         const float* topk_w, int64_t T, int64_t topk, int64_t H, void* out,
                         int64_t ldo, void* stream) {
  BQ_CHECK_ARG(T >= 0 && H >= 0 && topk >= 1, "need T >= 0, H >= 0, topk >= 1");
  BQ_CHECK_ARG(ldy >= H && ldo >= H, "leading dimensions must be >= H");
  if (T == 0 || H == 0) return ok();
  BQ_CHECK_ARG(y && inv_perm && topk_w && out, "y, inv_perm, topk_w and out must not be NULL");
  BQ_CHECK_CUDA(bq::launch_moe_combine(y, ldy, inv_perm, topk_w, T, topk, H, out, ldo,
                                       as_stream(stream)),
                "moe_combine launch");
  return ok();
}

}  // extern "C"
