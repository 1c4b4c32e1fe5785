/*
 * bitnet_oracle.c -- plain, slow, obviously-correct CPU oracle of the
 * BitNet b1.58 BitLinear forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file.  It exists so that the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg can compare the CUDA kernels against an
 * independent restatement of the method.  It shares no code, header, table or
 * constant with the CUDA sources.
 *
 * Sources (web pages; cited by title and section):
 *   [FT158] "LLM を 1.58 ビットにファインチューニング：BitNet による極端な量子化"
 *           (agentlenshq digest of Hugging Face's 1.58-bit fine-tuning post).
 *           Sections used: 量子化の仕組み (how quantization works),
 *           主な発見 (key findings: weights packed into int8 tensors),
 *           計算パラダイム (integer additions replace FP16 multiply-adds).
 *   [ERA1B] "[論文レビュー] The Era of 1-bit LLMs: All Large Language Models are
 *           in 1.58 Bits" (nubint review).  Section 提案手法 (method):
 *           absmean weight quantization to {-1,0,1}; RMSNorm in a LLaMA-like
 *           block.
 *   [BNCPP] "Microsoftの推論フレームワークにより、1ビットの大規模言語モデルが
 *           ローカルデバイスで実行可能になる" (unite.ai).  Section 数学的基礎,
 *           items 2 (activation quantization, Q_b and the infinity norm) and
 *           3 (BitLinear output rescale); partly garbled in the text.
 *
 * What each function computes, and the readings taken where the pages are
 * silent, are stated beside the function.  Arithmetic is IEEE-754 with
 * round-to-nearest-even; this file must be built with -ffp-contract=off and
 * without -ffast-math so that every a*b and a+b below is one rounded
 * operation (fmaf is the single fused step the sum of squares asks for).
 *
 * Pins (what checks this file against something other than itself) live in
 * tests/test_oracle_pins.py: a hand-worked 4x4 case, brute-force integer
 * matmul, closed forms for the scale statistics, invariants.  The two
 * reduction orders below (sum of squares, sum of |W|) are definitional
 * choices: the pages fix the formula, not the order, so the order itself is
 * "parity unpinned"; only the value is pinned, within its rounding bound.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_OVERFLOW 2

/* Number of partial sums used by both canonical reductions. */
#define NPART 256

/* ---------------------------------------------------------------- helpers */

static float bf16_bits_to_float(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16; /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
static uint16_t float_to_bf16_bits_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static float load_x(const void *x, int x_is_bf16, int64_t idx) {
    if (x_is_bf16) return bf16_bits_to_float(((const uint16_t *)x)[idx]);
    return ((const float *)x)[idx];
}

/* Pairwise tree over NPART partials: for s = NPART/2, ..., 1 the partial i
 * (i < s) absorbs partial i+s.  The result is partial 0. */
static float tree_f32(float *p) {
    for (int s = NPART / 2; s >= 1; s /= 2)
        for (int i = 0; i < s; ++i) p[i] = p[i] + p[i + s];
    return p[0];
}

static double tree_f64(double *p) {
    for (int s = NPART / 2; s >= 1; s /= 2)
        for (int i = 0; i < s; ++i) p[i] = p[i] + p[i + s];
    return p[0];
}

/* ------------------------------------------------- activations: RMSNorm */

/*
 * Inverse RMS of one token row, r = 1 / sqrt(mean(x^2) + eps).
 *
 * Norm type: [ERA1B] 提案手法 names RMSNorm for the LLaMA-like block, while
 * [FT158] 量子化の仕組み says a layer norm precedes activation quantization to
 * keep the output variance; the reading taken is RMSNorm with a per-channel
 * gain gamma.
 *
 * Reduction order (pages silent; definitional): element k feeds partial
 * (k/8) mod 256, each partial is updated in increasing k as p = fma(x, x, p)
 * starting from +0, and the 256 partials are combined by tree_f32.
 * mean = ss / K, then r = 1 / sqrt(mean + eps) with correctly rounded
 * division and square root.
 * Returns 0 and sets *r when mean + eps > 0; returns 1 (r undefined) when
 * mean + eps == 0 (an all-zero row with eps = 0), which callers treat as
 * "normalised row is all zeros".
 */
static int rms_inverse(const void *x, int x_is_bf16, int64_t row, int64_t K,
                       float eps, float *r) {
    float p[NPART];
    for (int i = 0; i < NPART; ++i) p[i] = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float v = load_x(x, x_is_bf16, row * K + k);
        int idx = (int)((k / 8) % NPART);
        p[idx] = fmaf(v, v, p[idx]);
    }
    float ss = tree_f32(p);
    float ms = ss / (float)K;
    float d = ms + eps;
    if (d == 0.0f) return 1;
    *r = 1.0f / sqrtf(d);
    return 0;
}

/*
 * RMSNorm followed by per-token absmax int8 quantization.
 *
 * [FT158] 量子化の仕組み: activations go to 8 bits per token with an absmax
 * scale that maps them into [-128, 127], after a normalisation.
 * [BNCPP] 数学的基礎 item 2: the quantization range Q_b and the infinity norm of
 * the token; its epsilon against overflow has no value on the page.
 *
 *   x_n[k] = (x[k] * r) * gamma[k]            (two rounded fp32 products;
 *                                               gamma == NULL means 1)
 *   amax   = max(max_k |x_n[k]|, 1e-5)        (floor is the epsilon reading)
 *   s_x    = 127 / amax
 *   x_q[k] = clamp(rint(x_n[k] * s_x), -128, 127)   (rint: ties to even)
 *
 * A row whose mean square plus eps is zero gives x_n = 0 and so x_q = 0.
 * Optional outputs: x_n (fp32 [M,K]) and rowsum (sum of x_q per row) may be
 * NULL.
 */
int oracle_rmsnorm_quant_act(const void *x, int x_is_bf16, const float *gamma,
                             float eps, int64_t M, int64_t K, int8_t *x_q,
                             float *s_x, float *x_n_out, int32_t *rowsum) {
    if (!x || !x_q || !s_x || M < 0 || K <= 0 || eps < 0.0f) return ORACLE_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        float r = 0.0f;
        int zero_row = rms_inverse(x, x_is_bf16, m, K, eps, &r);
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float xn = 0.0f;
            if (!zero_row) {
                float g = gamma ? gamma[k] : 1.0f;
                xn = (load_x(x, x_is_bf16, m * K + k) * r) * g;
            }
            if (x_n_out) x_n_out[m * K + k] = xn;
            float a = fabsf(xn);
            if (a > amax) amax = a;
        }
        if (amax < 1e-5f) amax = 1e-5f;
        float sx = 127.0f / amax;
        s_x[m] = sx;
        int32_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            float xn = 0.0f;
            if (!zero_row) {
                float g = gamma ? gamma[k] : 1.0f;
                xn = (load_x(x, x_is_bf16, m * K + k) * r) * g;
            }
            float q = rintf(xn * sx);
            if (q > 127.0f) q = 127.0f;
            if (q < -128.0f) q = -128.0f;
            x_q[m * K + k] = (int8_t)q;
            sum += (int32_t)q;
        }
        if (rowsum) rowsum[m] = sum;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------ weights: absmean scale */

/*
 * Per-tensor absmean scale, s_w = 1 / mean|W|.
 *
 * [FT158] 量子化の仕組み: symmetric per-tensor weight quantization whose scale
 * is the reciprocal of the mean absolute weight.  [ERA1B] 提案手法: the
 * absmean scheme, gamma = mean |W|.
 *
 * Reduction (pages silent; definitional): in fp64.  Row n: element k feeds
 * partial (k/4) mod 256 in increasing k, partials combined by tree_f64 into
 * R_n.  Then R_n feeds partial n mod 256 in increasing n, combined by
 * tree_f64 into S.  mean = (float)(S / (N*K)), floored at 1e-5 (epsilon
 * reading), s_w = 1 / mean in fp32.
 * Optional: S_out receives S.
 */
int oracle_weight_scale(const float *W, int64_t N, int64_t K, float *s_w,
                        double *S_out) {
    if (!W || !s_w || N <= 0 || K <= 0) return ORACLE_ERR_ARG;
    double q[NPART];
    for (int i = 0; i < NPART; ++i) q[i] = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double p[NPART];
        for (int i = 0; i < NPART; ++i) p[i] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            int idx = (int)((k / 4) % NPART);
            p[idx] = p[idx] + fabs((double)W[n * K + k]);
        }
        double Rn = tree_f64(p);
        int j = (int)(n % NPART);
        q[j] = q[j] + Rn;
    }
    double S = tree_f64(q);
    if (S_out) *S_out = S;
    float mean = (float)(S / (double)(N * K));
    if (mean < 1e-5f) mean = 1e-5f;
    *s_w = 1.0f / mean;
    return ORACLE_OK;
}

/*
 * Ternary value of one weight: clamp(rint(w * s_w), -1, 1).
 * [FT158] 量子化の仕組み: scale, round, clamp to [-1, 1].  [ERA1B] 提案手法 and
 * [BNCPP] 3値重みシステム: the three values -1, 0, 1.  Rounding reading: ties
 * to even (0.5 -> 0, 1.5 -> 2 -> clamped to 1).
 */
static int ternary_of(float w, float s_w) {
    float v = rintf(w * s_w);
    if (v > 1.0f) v = 1.0f;
    if (v < -1.0f) v = -1.0f;
    return (int)v;
}

/*
 * Quantize and pack: code = t + 1 in {0,1,2} (3 never produced), four codes
 * per byte, weight k of row n in bits [2*(k%4), 2*(k%4)+1] of byte
 * W_p[n*(K/4) + k/4] (low bits first), rows back to back.
 * [FT158] 主な発見: ternary weights stored packed into int8 tensors; the
 * pages give no bit layout, so the layout is this reading.
 * Requires K % 4 == 0.  Optional T_out receives the int8 ternary values.
 */
int oracle_quantize_pack(const float *W, int64_t N, int64_t K, float s_w,
                         uint8_t *W_p, int8_t *T_out) {
    if (!W || !W_p || N <= 0 || K <= 0 || (K % 4) != 0) return ORACLE_ERR_ARG;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < K / 4; ++b) {
            unsigned byte = 0;
            for (int j = 0; j < 4; ++j) {
                int64_t k = 4 * b + j;
                int t = ternary_of(W[n * K + k], s_w);
                if (T_out) T_out[n * K + k] = (int8_t)t;
                byte |= (unsigned)(t + 1) << (2 * j);
            }
            W_p[n * (K / 4) + b] = (uint8_t)byte;
        }
    }
    return ORACLE_OK;
}

/* Ternary value of weight (n, k) read back from the packed bytes. */
static int unpack_one(const uint8_t *W_p, int64_t K, int64_t n, int64_t k) {
    unsigned byte = W_p[n * (K / 4) + k / 4];
    unsigned code = (byte >> (2 * (k % 4))) & 3u;
    return (int)code - 1;
}

/* Inverse of the packing: T[n,k] in {-1,0,1}; returns ORACLE_ERR_ARG if a
 * code 3 (never written by the packer) is met. */
int oracle_unpack(const uint8_t *W_p, int64_t N, int64_t K, int8_t *T) {
    if (!W_p || !T || N <= 0 || K <= 0 || (K % 4) != 0) return ORACLE_ERR_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int t = unpack_one(W_p, K, n, k);
            if (t > 1) return ORACLE_ERR_ARG;
            T[n * K + k] = (int8_t)t;
        }
    return ORACLE_OK;
}

/* ----------------------------------------------------- integer matmul */

/*
 * acc[m, c] = sum_k x_q[m,k] * T[cols[c], k], accumulated in int64 and stored
 * as int32 (ORACLE_ERR_OVERFLOW if it does not fit).  cols == NULL means all
 * N columns in order (then ncols must equal N).
 * [FT158] 計算パラダイム: the matmul becomes integer additions; each ternary
 * product is +x, 0 or -x.
 */
int oracle_ternary_matmul_cols(const int8_t *x_q, const uint8_t *W_p, int64_t M,
                               int64_t N, int64_t K, const int64_t *cols,
                               int64_t ncols, int32_t *acc) {
    if (!x_q || !W_p || !acc || M < 0 || N <= 0 || K <= 0 || (K % 4) != 0)
        return ORACLE_ERR_ARG;
    if (!cols && ncols != N) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) reduction(max : err)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t n = cols ? cols[c] : c;
            if (n < 0 || n >= N) { err = ORACLE_ERR_ARG; continue; }
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) {
                int t = unpack_one(W_p, K, n, k);
                int xv = x_q[m * K + k];
                if (t > 0) s += xv;
                else if (t < 0) s -= xv;
            }
            if (s > INT32_MAX || s < INT32_MIN) { err = ORACLE_ERR_OVERFLOW; continue; }
            acc[m * ncols + c] = (int32_t)s;
        }
    }
    return err;
}

/*
 * Dequantization, y = (float)acc / (s_x[m] * s_w): the product of the two
 * scales rounded to fp32 first, then one correctly rounded division.
 * [FT158] 量子化の仕組み: quantized weights are rescaled; [BNCPP] 数学的基礎
 * item 3: the output is multiplied back by the weight and activation scale
 * factors (garbled formula; reading: divide by both multiplicative scales).
 * y_f32 and y_bf16 (RNE of y) may each be NULL.
 */
int oracle_dequant(const int32_t *acc, const float *s_x, float s_w, int64_t M,
                   int64_t ncols, float *y_f32, uint16_t *y_bf16) {
    if (!acc || !s_x || M < 0 || ncols < 0) return ORACLE_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        float denom = s_x[m] * s_w;
        for (int64_t c = 0; c < ncols; ++c) {
            float y = (float)acc[m * ncols + c] / denom;
            if (y_f32) y_f32[m * ncols + c] = y;
            if (y_bf16) y_bf16[m * ncols + c] = float_to_bf16_bits_rne(y);
        }
    }
    return ORACLE_OK;
}

/* fp32 -> bf16 bits (RNE) for a whole buffer; used by the tests to express
 * bf16 expectations. */
void oracle_f32_to_bf16(const float *src, uint16_t *dst, int64_t n) {
    for (int64_t i = 0; i < n; ++i) dst[i] = float_to_bf16_bits_rne(src[i]);
}

/*
 * The whole forward for columns `cols` (NULL = all): RMSNorm + activation
 * quant, integer matmul against the packed ternary weights, dequant.
 * x_q / s_x / acc are caller buffers ([M,K], [M], [M,ncols]).
 */
int oracle_linear_forward(const void *x, int x_is_bf16, const float *gamma,
                          float eps, const uint8_t *W_p, float s_w, int64_t M,
                          int64_t N, int64_t K, const int64_t *cols,
                          int64_t ncols, int8_t *x_q, float *s_x, int32_t *acc,
                          float *y_f32, uint16_t *y_bf16) {
    int e = oracle_rmsnorm_quant_act(x, x_is_bf16, gamma, eps, M, K, x_q, s_x,
                                     NULL, NULL);
    if (e) return e;
    e = oracle_ternary_matmul_cols(x_q, W_p, M, N, K, cols, ncols, acc);
    if (e) return e;
    return oracle_dequant(acc, s_x, s_w, M, ncols, y_f32, y_bf16);
}

/* Thread count for the OpenMP loop of the matmul (1 when built without
 * OpenMP).  Returns the count in effect. */
int oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
