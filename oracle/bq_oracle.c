/*
 * bq_oracle.c -- plain, slow, obviously-correct CPU oracle for the block-scaled
 * W8A8 linear layer and its MoE variant.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file:
 * only the test-suite, the smoke check and the benchmark's CPU-baseline leg use
 * it.  It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (web pages; cited by title and section):
 *   [BWI8]  "[SGLang] Block-wise INT8: 블록 단위 정수 양자화" (block-wise INT8 page)
 *           - structure diagram: W [N,K] int8, scale [N/bn, K/bk] fp32
 *           - §2 "가중치 생성과 블록 스케일": scale grid is
 *             ceil(N/block_n) x ceil(K/block_k); [4096,4096] with [128,128] -> [32,32]
 *           - §4 "추론 적용": input_scale=None, activation scale computed at
 *             run time per token inside the kernel (dynamic activation)
 *           - §5 "MoE 전용 BlockInt8": w13 = gate+up fused, [E, 2I, H],
 *             scales [E, 2*ceil(I/bn), ceil(H/bk)]
 *           - "설계 근거" item 3: int8 range -128..127, fp32 scales
 *   [QDOC]  SGLang "양자화 (Quantization)" doc, "FP4/FP8 양자화용 GEMM 백엔드":
 *           blockwise FP8 GEMM is the FP8 form of the same contraction.
 *   [LLMQ]  "LLM 양자화 완전 정리 — FP8, AWQ, GPTQ, GGUF 차이와 선택법",
 *           "FP8 — 신세대 GPU를 위한 양자화 / 개념": e4m3 = 1 sign, 4 exponent,
 *           3 mantissa bits.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - activation groups are 1 x group_k (per token, per K-block);
 *   - scale = amax / 127 (INT8) or amax / 448 (FP8 e4m3), computed as one IEEE
 *     fp32 division; codes = fp32 division x / scale, then round-half-even and
 *     clamp to [-128,127] (INT8) or one round-to-nearest-even conversion to
 *     e4m3 with saturation to +-448 (FP8);
 *   - an all-zero group gets scale 0 and all-zero codes;
 *   - partial blocks (ceil division) take amax over their valid elements only;
 *   - the stored weight scale is the dequantisation multiplier: W ~= q * s.
 *
 * Floating point: compile WITHOUT -ffast-math / -Ofast; no FTZ/DAZ.  The
 * divisions below are float/float in C, i.e. IEEE single-precision division
 * rounded to nearest even (FLT_EVAL_METHOD 0 on x86-64 SSE).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define BQ_REF_INT8 0
#define BQ_REF_FP8 1

/* ------------------------------------------------------------------------ */
/* bf16 <-> double                                                          */
/* ------------------------------------------------------------------------ */

/* A bf16 value is the upper 16 bits of an IEEE binary32. */
double bq_ref_bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits, binary32 exponent
 * range), ties to even, in ONE rounding step.  Overflow gives +-inf. */
uint16_t bq_ref_bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    int neg = v < 0.0;
    double a = neg ? -v : v;
    int e;
    frexp(a, &e);               /* a = m * 2^e, 0.5 <= m < 1 */
    int q = e - 8;              /* quantum exponent for 8 significant bits */
    if (q < -133) q = -133;     /* bf16 subnormal quantum 2^-133 */
    double t = ldexp(a, -q);    /* exact: scaling by a power of two */
    double f = floor(t);
    double d = t - f;           /* exact */
    double r;
    if (d > 0.5) r = f + 1.0;
    else if (d < 0.5) r = f;
    else r = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
    double res = ldexp(r, q);
    if (res > 3.3895313892515355e38) { /* beyond max finite bf16 */
        return neg ? 0xFF80 : 0x7F80;
    }
    float rf = (float)res;      /* exact: res has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, 4);
    uint16_t h = (uint16_t)(u >> 16);
    return neg ? (uint16_t)(h | 0x8000) : h;
}

/* ------------------------------------------------------------------------ */
/* FP8 e4m3 ("fn" variant: no infinities, S.1111.111 is NaN, max 448)       */
/* ------------------------------------------------------------------------ */

/* Value of a code: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits
 * ([LLMQ] "개념").  Exponent field 0 encodes subnormals m * 2^-9. */
double bq_ref_e4m3_decode(uint8_t c) {
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Encode a binary32 value: round to nearest, ties to the code with an even
 * mantissa (= even code), saturate magnitudes above 448 to 448, keep the sign
 * of zero.  Done by searching the ordered table of non-negative codes. */
uint8_t bq_ref_e4m3_encode(float x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* non-negative finite codes 0x00..0x7E are increasing in value */
    int c = 0;
    while (c < 0x7E && bq_ref_e4m3_decode((uint8_t)(c + 1)) <= a) c++;
    /* now value(c) <= a < value(c+1) (c < 0x7E because a < 448) */
    double lo = bq_ref_e4m3_decode((uint8_t)c);
    double hi = bq_ref_e4m3_decode((uint8_t)(c + 1));
    double mid = 0.5 * (lo + hi);     /* exact in double */
    int pick;
    if (a < mid) pick = c;
    else if (a > mid) pick = c + 1;
    else pick = (c % 2 == 0) ? c : c + 1;
    return (uint8_t)(sign | (uint8_t)pick);
}

/* ------------------------------------------------------------------------ */
/* Scalar quantisation of one group                                         */
/* ------------------------------------------------------------------------ */

/* Round half to even of a float, returned as double (exact). */
static double round_half_even(float c) {
    double v = (double)c;
    double f = floor(v);
    double d = v - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Quantise the L values x[0..L) (already binary32) as one group.
 * INT8: s = fl32(amax / 127); q_i = clamp(rhe(fl32(x_i / s)), -128, 127).
 * FP8 : s = fl32(amax / 448); q_i = e4m3_rne_satfinite(fl32(x_i / s)).
 * amax == 0: s = 0 and every code is 0 (+0 for FP8).
 * Codes are written as raw bytes (int8 two's complement, or e4m3 bits). */
static float quant_group(const float* x, long L, int dtype, uint8_t* q) {
    float amax = 0.0f;
    for (long i = 0; i < L; i++) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    const float qmax = (dtype == BQ_REF_INT8) ? 127.0f : 448.0f;
    float s = amax / qmax;                 /* one IEEE fp32 division */
    for (long i = 0; i < L; i++) {
        if (s == 0.0f) { q[i] = 0; continue; }
        float c = x[i] / s;                /* one IEEE fp32 division */
        if (dtype == BQ_REF_INT8) {
            double r = round_half_even(c);
            if (r > 127.0) r = 127.0;
            if (r < -128.0) r = -128.0;
            q[i] = (uint8_t)(int8_t)(int)r;
        } else {
            q[i] = bq_ref_e4m3_encode(c);
        }
    }
    return s;
}

/* Decode one stored code to its exact value. */
static double code_value(uint8_t c, int dtype) {
    if (dtype == BQ_REF_INT8) return (double)(int8_t)c;
    return bq_ref_e4m3_decode(c);
}

/* ------------------------------------------------------------------------ */
/* dynamic activation quantisation, groups 1 x group_k ([BWI8] §4)       */
/* ------------------------------------------------------------------------ */

/* x: bf16 [M, K] (row stride ldx); q: [M, K] bytes (row stride ldq);
 * s: fp32 [M, Kb] row-major, Kb = ceil(K / group_k).  The last group of a
 * row holds K - (Kb-1)*group_k valid elements. */
void bq_ref_quant_act(const uint16_t* x, long M, long K, long ldx, long group_k,
                      int dtype, uint8_t* q, long ldq, float* s) {
    long Kb = (K + group_k - 1) / group_k;
    /* rows are independent: the OpenMP build (baseline timing only) splits
     * them over threads; without -fopenmp the pragmas are ignored */
#pragma omp parallel
    {
        float* buf = (float*)malloc(sizeof(float) * (size_t)(group_k > 0 ? group_k : 1));
#pragma omp for schedule(static)
        for (long m = 0; m < M; m++) {
            for (long g = 0; g < Kb; g++) {
                long k0 = g * group_k;
                long L = (k0 + group_k <= K) ? group_k : K - k0;
                for (long i = 0; i < L; i++)
                    buf[i] = (float)bq_ref_bf16_to_double(x[m * ldx + k0 + i]);
                s[m * Kb + g] = quant_group(buf, L, dtype, q + m * ldq + k0);
            }
        }
        free(buf);
    }
}

/* ------------------------------------------------------------------------ */
/* offline weight block quantisation ([BWI8] §2, structure diagram)     */
/* ------------------------------------------------------------------------ */

/* w: fp32 [N, K] row-major (stride ldw); q: [N, K] bytes (stride ldq);
 * s: fp32 [Nb, Kb] row-major with Nb = ceil(N/bn), Kb = ceil(K/bk).
 * One scale per [bn, bk] block; partial edge blocks use their valid part. */
void bq_ref_quant_weight(const float* w, long N, long K, long ldw, long bn, long bk,
                         int dtype, uint8_t* q, long ldq, float* s) {
    long Nb = (N + bn - 1) / bn, Kb = (K + bk - 1) / bk;
    for (long i = 0; i < Nb; i++) {
        for (long j = 0; j < Kb; j++) {
            long n0 = i * bn, k0 = j * bk;
            long Ln = (n0 + bn <= N) ? bn : N - n0;
            long Lk = (k0 + bk <= K) ? bk : K - k0;
            float* buf = (float*)malloc(sizeof(float) * (size_t)(Ln * Lk));
            uint8_t* qb = (uint8_t*)malloc((size_t)(Ln * Lk));
            for (long r = 0; r < Ln; r++)
                for (long c = 0; c < Lk; c++) buf[r * Lk + c] = w[(n0 + r) * ldw + k0 + c];
            s[i * Kb + j] = quant_group(buf, Ln * Lk, dtype, qb);
            for (long r = 0; r < Ln; r++)
                for (long c = 0; c < Lk; c++) q[(n0 + r) * ldq + k0 + c] = qb[r * Lk + c];
            free(buf);
            free(qb);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* block-scaled GEMM ([BWI8] §2, §4; [QDOC] blockwise FP8)            */
/* ------------------------------------------------------------------------ */

/* Weight-scale row of output column n.  With seam == 0 (or >= N) this is
 * n / bn.  A fused gate+up weight ([BWI8] §5) blocks its two halves
 * separately: rows [0, seam) use n / bn, rows [seam, N) use
 * ceil(seam / bn) + (n - seam) / bn. */
static long wrow_block(long n, long bn, long seam, long N) {
    if (seam <= 0 || seam >= N || n < seam) return n / bn;
    return (seam + bn - 1) / bn + (n - seam) / bn;
}

/* One output element, exactly as the method defines it:
 *   out[m,n] = sum_kb  P_kb[m,n] * sa[m,kb] * sw[nb(n),kb]  (+ bias[n])
 *   P_kb[m,n] = sum_{k in block kb} qa[m,k] * qw[n,k]
 * P is exact (int64 for INT8; for FP8 every product of two e4m3 values and
 * every partial sum of <= 2^16 of them fits in a double's 53 bits).  The
 * rescale and the sum over blocks are done in fp64. */
double bq_ref_gemm_entry(const uint8_t* qa, long lda, const float* sa, const uint8_t* qw,
                         long ldw, const float* sw, long N, long K, long bn, long bk,
                         long seam, int dtype, const uint16_t* bias, long m, long n) {
    long Kb = (K + bk - 1) / bk;
    long nb = wrow_block(n, bn, seam, N);
    double acc = 0.0;
    for (long kb = 0; kb < Kb; kb++) {
        long k0 = kb * bk, k1 = (k0 + bk <= K) ? k0 + bk : K;
        double P;
        if (dtype == BQ_REF_INT8) {
            int64_t Pi = 0;
            for (long k = k0; k < k1; k++)
                Pi += (int64_t)(int8_t)qa[m * lda + k] * (int64_t)(int8_t)qw[n * ldw + k];
            P = (double)Pi;
        } else {
            P = 0.0;
            for (long k = k0; k < k1; k++)
                P += bq_ref_e4m3_decode(qa[m * lda + k]) * bq_ref_e4m3_decode(qw[n * ldw + k]);
        }
        acc += P * (double)sa[m * Kb + kb] * (double)sw[nb * Kb + kb];
    }
    if (bias) acc += bq_ref_bf16_to_double(bias[n]);
    return acc;
}

/* Full output, out64 [M, N] row-major.  sa is [M, Kb] row-major; sw is
 * [rows, Kb] row-major. */
void bq_ref_gemm(const uint8_t* qa, long lda, const float* sa, const uint8_t* qw,
                 long ldw, const float* sw, long M, long N, long K, long bn, long bk,
                 long seam, int dtype, const uint16_t* bias, double* out) {
#pragma omp parallel for schedule(static)
    for (long m = 0; m < M; m++)
        for (long n = 0; n < N; n++)
            out[m * N + n] = bq_ref_gemm_entry(qa, lda, sa, qw, ldw, sw, N, K, bn, bk, seam,
                                               dtype, bias, m, n);
}

/* Dequantised reference: sum_k (qa*sa)(qw*sw), one term at a time, in fp64.
 * Mathematically equal to bq_ref_gemm_entry; used to pin it by brute force. */
double bq_ref_dequant_dot(const uint8_t* qa, long lda, const float* sa, const uint8_t* qw,
                          long ldw, const float* sw, long N, long K, long bn, long bk,
                          long seam, int dtype, long m, long n) {
    long Kb = (K + bk - 1) / bk;
    long nb = wrow_block(n, bn, seam, N);
    double acc = 0.0;
    for (long k = 0; k < K; k++) {
        long kb = k / bk;
        double a = code_value(qa[m * lda + k], dtype) * (double)sa[m * Kb + kb];
        double b = code_value(qw[n * ldw + k], dtype) * (double)sw[nb * Kb + kb];
        acc += a * b;
    }
    return acc;
}

/* ------------------------------------------------------------------------ */
/* MoE routing: topk_ids and topk_weights, the inputs the block-wise INT8  */
/* page's MoE runner (§5-§6) receives; the workload routes each token to   */
/* its top-2 experts by the softmax of its router logits.  The pages do    */
/* not fix the tie order or whether the top-k weights are renormalised;    */
/* the reading: softmax in fp64, experts by descending probability, ties   */
/* to the lower expert index, the k probabilities divided by their sum.    */
/* ------------------------------------------------------------------------ */

/* logits: fp32 [T, E] (row stride ld); ids: int32 [T, topk]; w: fp32 [T, topk]. */
void bq_ref_moe_route(const float* logits, long ld, long T, long E, long topk, int32_t* ids,
                      float* w) {
    double* p = (double*)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1));
    unsigned char* taken = (unsigned char*)malloc((size_t)(E > 0 ? E : 1));
    for (long t = 0; t < T; t++) {
        const float* l = logits + t * ld;
        double mx = (double)l[0];
        for (long e = 1; e < E; e++)
            if ((double)l[e] > mx) mx = (double)l[e];
        double sum = 0.0;
        for (long e = 0; e < E; e++) {
            p[e] = exp((double)l[e] - mx);
            sum += p[e];
        }
        for (long e = 0; e < E; e++) {
            p[e] /= sum;
            taken[e] = 0;
        }
        double topsum = 0.0;
        for (long j = 0; j < topk; j++) {
            long best = -1;
            for (long e = 0; e < E; e++)
                if (!taken[e] && (best < 0 || p[e] > p[best])) best = e;
            taken[best] = 1;
            ids[t * topk + j] = (int32_t)best;
            topsum += p[best];
        }
        for (long j = 0; j < topk; j++)
            w[t * topk + j] = (float)(p[ids[t * topk + j]] / topsum);
    }
    free(p);
    free(taken);
}

/* ------------------------------------------------------------------------ */
/* MoE token permutation ([BWI8] §5-§6: per-expert weights, routed      */
/* tokens).  Stable order: by expert, then by flat slot index t*topk + j.   */
/* ------------------------------------------------------------------------ */

/* ids: [T, topk] expert of each (token, slot); offsets: [E+1] exclusive
 * prefix of per-expert counts; perm[r] = flat slot index placed at permuted
 * row r; inv_perm[t*topk + j] = its permuted row.  Returns 0, or -1 if an
 * id is outside [0, E). */
int bq_ref_moe_permute(const int32_t* ids, long T, long topk, long E, int32_t* offsets,
                       int32_t* perm, int32_t* inv_perm) {
    long R = T * topk;
    for (long i = 0; i < R; i++)
        if (ids[i] < 0 || ids[i] >= E) return -1;
    long r = 0;
    for (long e = 0; e < E; e++) {
        offsets[e] = (int32_t)r;
        for (long i = 0; i < R; i++) {
            if (ids[i] == e) {
                perm[r] = (int32_t)i;
                inv_perm[i] = (int32_t)r;
                r++;
            }
        }
    }
    offsets[E] = (int32_t)r;
    return 0;
}

/* h = silu(g) * u rounded once to bf16, g = y[r, i], u = y[r, I + i]
 * ("gate + up fused", [BWI8] §5; SiLU is the reading for a gate/up pair).
 * silu(g) = g / (1 + exp(-g)), in fp64. */
void bq_ref_silu_mul(const uint16_t* y, long R, long I, long ldy, uint16_t* h) {
#pragma omp parallel for schedule(static)
    for (long r = 0; r < R; r++) {
        for (long i = 0; i < I; i++) {
            double g = bq_ref_bf16_to_double(y[r * ldy + i]);
            double u = bq_ref_bf16_to_double(y[r * ldy + I + i]);
            double v = g / (1.0 + exp(-g)) * u;
            h[r * I + i] = bq_ref_bf16_from_double(v);
        }
    }
}

/* out[t, n] = bf16( sum_j w[t, j] * y[inv_perm[t*topk + j], n] ), fp64. */
void bq_ref_moe_combine(const uint16_t* y, long ldy, const int32_t* inv_perm,
                        const float* w, long T, long topk, long H, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (long t = 0; t < T; t++) {
        for (long n = 0; n < H; n++) {
            double acc = 0.0;
            for (long j = 0; j < topk; j++) {
                long r = inv_perm[t * topk + j];
                acc += (double)w[t * topk + j] * bq_ref_bf16_to_double(y[r * ldy + n]);
            }
            out[t * H + n] = bq_ref_bf16_from_double(acc);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP8 ([QDOC] "FP4/FP8 양자화용 GEMM 백엔드": MXFP8 dense linear)        */
/* ------------------------------------------------------------------------ */
/* The pages name the MXFP8 dense linear but do not define the format.
 * Reading: the microscaling (MX) format the name refers to -- groups of 32
 * consecutive elements along K share one scale 2^(E - 127) stored as an
 * 8-bit exponent E (E8M0; 255 would be NaN and is never produced), elements
 * are e4m3 codes.  The group's scale exponent is floor(log2(amax)) minus the
 * largest exponent of an e4m3 normal (8), clamped to [-127, 127]; each
 * element is x / 2^se (exact: a power-of-two scaling) converted to e4m3 by
 * one round-to-nearest-even with saturation to +-448.  An all-zero group
 * gets E = 0 and zero codes. */

#define BQ_REF_MX_GROUP 32

/* floor(log2(a)) for a finite a > 0, exactly (frexp: a = f * 2^e, f in [0.5, 1)). */
static int floor_log2(double a) {
    int e;
    (void)frexp(a, &e);
    return e - 1;
}

/* One group of L <= 32 values: returns the E8M0 byte, writes L codes. */
static uint8_t mx_group(const double* x, long L, uint8_t* q) {
    double amax = 0.0;
    for (long i = 0; i < L; i++) {
        double a = fabs(x[i]);
        if (a > amax) amax = a;
    }
    int se = -127;
    if (amax > 0.0) {
        se = floor_log2(amax) - 8;
        if (se < -127) se = -127;
        if (se > 127) se = 127;
    }
    double inv = ldexp(1.0, -se);
    for (long i = 0; i < L; i++) q[i] = bq_ref_e4m3_encode((float)(x[i] * inv));
    return (uint8_t)(se + 127);
}

/* x: [R, K] doubles (exact copies of the bf16 or fp32 inputs), row stride ldx;
 * q: [R, K] e4m3 codes (row stride ldq); s: [R, ceil(K/32)] E8M0 bytes
 * row-major.  The last group of a row holds the remaining K mod 32 values. */
void bq_ref_mx_quant(const double* x, long R, long K, long ldx, uint8_t* q, long ldq,
                     uint8_t* s) {
    long G = (K + BQ_REF_MX_GROUP - 1) / BQ_REF_MX_GROUP;
    for (long r = 0; r < R; r++)
        for (long g = 0; g < G; g++) {
            long k0 = g * BQ_REF_MX_GROUP;
            long L = (k0 + BQ_REF_MX_GROUP <= K) ? BQ_REF_MX_GROUP : K - k0;
            s[r * G + g] = mx_group(x + r * ldx + k0, L, q + r * ldq + k0);
        }
}

/* out[m, n] = sum_g 2^(sa[m,g]-127) * 2^(sw[n,g]-127) * sum_{k in g} qa[m,k] qw[n,k]
 * (+ bias[n]) in fp64; out64 [M, N] row-major.  sa [M, G], sw [N, G] E8M0. */
void bq_ref_mx_gemm(const uint8_t* qa, long lda, const uint8_t* sa, const uint8_t* qw,
                    long ldw, const uint8_t* sw, long M, long N, long K,
                    const uint16_t* bias, double* out) {
    long G = (K + BQ_REF_MX_GROUP - 1) / BQ_REF_MX_GROUP;
#pragma omp parallel for schedule(static)
    for (long m = 0; m < M; m++)
        for (long n = 0; n < N; n++) {
            double acc = 0.0;
            for (long g = 0; g < G; g++) {
                long k0 = g * BQ_REF_MX_GROUP;
                long k1 = (k0 + BQ_REF_MX_GROUP <= K) ? k0 + BQ_REF_MX_GROUP : K;
                double P = 0.0;
                for (long k = k0; k < k1; k++)
                    P += bq_ref_e4m3_decode(qa[m * lda + k]) * bq_ref_e4m3_decode(qw[n * ldw + k]);
                acc += P * ldexp(1.0, (int)sa[m * G + g] - 127) *
                       ldexp(1.0, (int)sw[n * G + g] - 127);
            }
            if (bias != NULL) acc += bq_ref_bf16_to_double(bias[n]);
            out[m * N + n] = acc;
        }
}

/* Threads used by the row loops above: the OpenMP build (compiled with
 * -fopenmp, for the CPU baseline timing) sets and reports them; the plain
 * build always runs one thread. */
#ifdef _OPENMP
#include <omp.h>
int bq_ref_threads(int n) {
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
}
#else
int bq_ref_threads(int n) {
    (void)n;
    return 1;
}
#endif
