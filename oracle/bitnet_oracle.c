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
#include <stdlib.h>
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

/* ===================================================================== */
/* Variants of the forward (the "next" rows of the hot path).             */
/* ===================================================================== */

/* ------------------------------------------------- SwiGLU of two outputs */

/*
 * out = silu(g) * u, silu(z) = z / (1 + exp(-z)).
 * [ERA1B] 提案手法: the LLaMA-like block of BitNet b1.58 uses SwiGLU; its
 * gate and up projections are two BitLinear forwards of the same input and
 * the feed-forward multiplies silu(gate) by up.  g and u are those two fp32
 * outputs.  Arithmetic: fp64 from the fp32 inputs, one rounding to fp32 (and
 * RNE to bf16) at the end.  Either output may be NULL.
 */
int oracle_swiglu(const float *g, const float *u, int64_t n, float *out_f32,
                  uint16_t *out_bf16) {
    if (!g || !u || n < 0) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        double z = (double)g[i];
        double s = z / (1.0 + exp(-z));
        float o = (float)(s * (double)u[i]);
        if (out_f32) out_f32[i] = o;
        if (out_bf16) out_bf16[i] = float_to_bf16_bits_rne(o);
    }
    return ORACLE_OK;
}

/* ------------------------------------- lambda-warmup fake-quant forward */

/*
 * The training-time BitLinear forward with the warm-up of [FT158]
 * 動的ウォームアップ量子化: lambda = min(step / total_steps, 1) scales the
 * difference between the original and the quantized values, so the layer
 * moves from full precision (lambda = 0) to full quantization (lambda = 1).
 * Reading: the blend applies to both operands the page quantizes (weights
 * and activations, [FT158] 量子化の仕組み), each "quantized value" being the
 * rescaled fake-quant value:
 *
 *   x_n        RMSNorm of x, as oracle_rmsnorm_quant_act (fp32)
 *   xt[k]      = x_q[k] / s_x                   (fp32, correctly rounded)
 *   x_lam[k]   = x_n[k] + lambda * (xt[k] - x_n[k])   (three rounded fp32 ops)
 *   Wt[n,k]    = t[n,k] / s_w                   (t, s_w as the weight quant)
 *   W_lam[n,k] = W[n,k] + lambda * (Wt[n,k] - W[n,k])
 *   y[m,n]     = sum_k x_lam[m,k] * W_lam[n,k]
 *
 * The GPU computes the product on bf16 tensor cores (the training dtype of
 * the fine-tuning the page describes), so this function also returns the
 * sum over the bf16-rounded (RNE) operands, y_b, which is what such a kernel
 * approximates up to its fp32 accumulation, and sum |products| (absdot) for
 * the accumulation bound.  Sums run in fp64 (products of bf16 values are
 * exact in fp64).  Columns `cols` (NULL = all N); outputs [M][ncols]; any
 * of x_lam_out ([M][K]), y, y_b, absdot may be NULL.
 */
int oracle_warmup_forward(const void *x, int x_is_bf16, const float *gamma,
                          float eps, const float *W, int64_t M, int64_t N,
                          int64_t K, float lambda, const int64_t *cols,
                          int64_t ncols, float *x_lam_out, double *y,
                          double *y_b, double *absdot) {
    if (!x || !W || M < 0 || N <= 0 || K <= 0 || !(lambda >= 0.0f) || lambda > 1.0f)
        return ORACLE_ERR_ARG;
    if (!cols && ncols != N) return ORACLE_ERR_ARG;
    float s_w;
    int e = oracle_weight_scale(W, N, K, &s_w, NULL);
    if (e) return e;
    int8_t *xq = (int8_t *)malloc((size_t)(M > 0 ? M : 1) * (size_t)K);
    float *sx = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
    float *xn = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1) * (size_t)K);
    float *xl = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1) * (size_t)K);
    float *wl = (float *)malloc(sizeof(float) * (size_t)K);
    if (!xq || !sx || !xn || !xl || !wl) {
        free(xq); free(sx); free(xn); free(xl); free(wl);
        return ORACLE_ERR_ARG;
    }
    e = oracle_rmsnorm_quant_act(x, x_is_bf16, gamma, eps, M, K, xq, sx, xn, NULL);
    if (!e) {
        for (int64_t m = 0; m < M; ++m)
            for (int64_t k = 0; k < K; ++k) {
                float v = xn[m * K + k];
                float qt = (float)xq[m * K + k] / sx[m];
                float d = qt - v;
                float l = lambda * d;
                xl[m * K + k] = v + l;
            }
        if (x_lam_out) memcpy(x_lam_out, xl, sizeof(float) * (size_t)M * (size_t)K);
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t n = cols ? cols[c] : c;
            if (n < 0 || n >= N) { e = ORACLE_ERR_ARG; break; }
            for (int64_t k = 0; k < K; ++k) {
                float w = W[n * K + k];
                float wt = (float)ternary_of(w, s_w) / s_w;
                float d = wt - w;
                float l = lambda * d;
                wl[k] = w + l;
            }
            for (int64_t m = 0; m < M; ++m) {
                double s = 0.0, sb = 0.0, sa = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    float a = xl[m * K + k], b = wl[k];
                    s += (double)a * (double)b;
                    double pb = (double)bf16_bits_to_float(float_to_bf16_bits_rne(a)) *
                                (double)bf16_bits_to_float(float_to_bf16_bits_rne(b));
                    sb += pb;
                    sa += fabs(pb);
                }
                if (y) y[m * ncols + c] = s;
                if (y_b) y_b[m * ncols + c] = sb;
                if (absdot) absdot[m * ncols + c] = sa;
            }
        }
    }
    free(xq); free(sx); free(xn); free(xl); free(wl);
    return e;
}

/*
 * The weight operand of the warm-up forward on its own: W_lam [N][K] fp32 as
 * oracle_warmup_forward forms it per column (t and s_w of the per-tensor
 * weight quantization; t / s_w correctly rounded, then the three rounded
 * fp32 steps of the blend).  s_w_out may be NULL.
 */
int oracle_warmup_weights(const float *W, int64_t N, int64_t K, float lambda,
                          float *W_lam, float *s_w_out) {
    if (!W || !W_lam || N <= 0 || K <= 0 || !(lambda >= 0.0f) || lambda > 1.0f)
        return ORACLE_ERR_ARG;
    float s_w;
    int e = oracle_weight_scale(W, N, K, &s_w, NULL);
    if (e) return e;
    for (int64_t i = 0; i < N * K; ++i) {
        float w = W[i];
        float wt = (float)ternary_of(w, s_w) / s_w;
        float d = wt - w;
        float l = lambda * d;
        W_lam[i] = w + l;
    }
    if (s_w_out) *s_w_out = s_w;
    return ORACLE_OK;
}

/* -------------------------------------------- BitDelta: 1-bit deltas */

/*
 * Compression of one fine-tuned matrix against its base
 * ("【論文要約】BitDelta: Your Fine-Tune May Only Be Worth One Bit", Eq. 1-4):
 *   Delta = W_fine - W_base                       (fp64, exact here)
 *   Sign(Delta) = +1 if Delta > 0, else -1        (Eq. 2: zero maps to -1)
 *   alpha = (1 / (N K)) sum |Delta|               (Eq. 4, the L2-optimal scale)
 * W_base and W_fine are bf16 bit patterns [N][K] (a half-precision base
 * model, the page's Table 4 setting; bf16 is the activation type used
 * throughout this library).  The page's kernel packs the sign bits 32 per
 * integer without a bit order; reading: bit j (least significant first) of
 * word w of row n is 1 when Sign(Delta[n, 32 w + j]) = +1; rows back to
 * back, K/32 words each.  The sum for alpha uses the order of the weight
 * scale: per row, element k to partial (k/4) mod 256, tree; row sums to
 * partial n mod 256, tree; alpha = (float)(S / (N K)).  K % 32 == 0.
 */
int oracle_bitdelta_compress(const uint16_t *W_base, const uint16_t *W_fine,
                             int64_t N, int64_t K, uint32_t *signs, float *alpha,
                             double *S_out) {
    if (!W_base || !W_fine || !signs || !alpha || N <= 0 || K <= 0 || (K % 32) != 0)
        return ORACLE_ERR_ARG;
    double q[NPART];
    for (int i = 0; i < NPART; ++i) q[i] = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double p[NPART];
        for (int i = 0; i < NPART; ++i) p[i] = 0.0;
        for (int64_t w = 0; w < K / 32; ++w) {
            uint32_t word = 0;
            for (int j = 0; j < 32; ++j) {
                int64_t k = 32 * w + j;
                double d = (double)bf16_bits_to_float(W_fine[n * K + k]) -
                           (double)bf16_bits_to_float(W_base[n * K + k]);
                if (d > 0.0) word |= 1u << j;
                int idx = (int)((k / 4) % NPART);
                p[idx] = p[idx] + fabs(d);
            }
            signs[n * (K / 32) + w] = word;
        }
        double Rn = tree_f64(p);
        int j = (int)(n % NPART);
        q[j] = q[j] + Rn;
    }
    double S = tree_f64(q);
    if (S_out) *S_out = S;
    *alpha = (float)(S / (double)(N * K));
    return ORACLE_OK;
}

/*
 * Batched multi-tenant forward (Eq. 6): tenant b's input x_b (one token)
 * through its fine-tuned layer approximated as W_base + alpha_b Sign(Delta_b):
 *   y[b][n] = sum_k x[b][k] W_base[n][k] + alpha_b * sum_k x[b][k] s_b[n][k]
 * x: bf16 bits [B][K]; W_base: bf16 bits [N][K]; signs: [B][N][K/32] words
 * (layout of oracle_bitdelta_compress); alpha: [B].  fp64 sums of exact
 * products.  absdot (may be NULL) receives sum_k |x W_base| + alpha_b
 * sum_k |x| for the accumulation bound.  Columns `cols` (NULL = all);
 * outputs [B][ncols].
 */
int oracle_bitdelta_forward(const uint16_t *x, const uint16_t *W_base,
                            const uint32_t *signs, const float *alpha, int64_t B,
                            int64_t N, int64_t K, const int64_t *cols,
                            int64_t ncols, double *y, double *absdot) {
    if (!x || !W_base || !signs || !alpha || !y || B < 0 || N <= 0 || K <= 0 ||
        (K % 32) != 0)
        return ORACLE_ERR_ARG;
    if (!cols && ncols != N) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) reduction(max : err)
#endif
    for (int64_t c = 0; c < ncols; ++c) {
        int64_t n = cols ? cols[c] : c;
        if (n < 0 || n >= N) { err = ORACLE_ERR_ARG; continue; }
        for (int64_t b = 0; b < B; ++b) {
            double base = 0.0, delta = 0.0, ab = 0.0, ax = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double xv = (double)bf16_bits_to_float(x[b * K + k]);
                double wv = (double)bf16_bits_to_float(W_base[n * K + k]);
                uint32_t word = signs[(b * N + n) * (K / 32) + k / 32];
                double s = ((word >> (k % 32)) & 1u) ? 1.0 : -1.0;
                base += xv * wv;
                delta += xv * s;
                ab += fabs(xv * wv);
                ax += fabs(xv);
            }
            y[b * ncols + c] = base + (double)alpha[b] * delta;
            if (absdot) absdot[b * ncols + c] = ab + (double)alpha[b] * ax;
        }
    }
    return err;
}

/* ------------------------------------------------ group-wise scales */

/*
 * Group quantization ([BNCPP] グループ量子化と正規化): the weights and the
 * activations are split into groups that are quantized independently, so
 * that the groups (e.g. the K slices of a model-parallel layer) need no
 * communication for their scales.  Reading: G = K / group_k contiguous
 * groups along K (the reduction dimension, the one a row-parallel split
 * shares); every group has its own absmean weight scale and every
 * (token, group) its own absmax activation scale; the RMSNorm itself stays
 * over the whole row.
 *
 *   s_w[g]   = 1 / max(mean over all N rows and the group's columns of |W|, 1e-5)
 *              fp64 sum in the order of oracle_weight_scale applied to the
 *              N x group_k block (element k - g*group_k of a row to partial
 *              ((k - g*group_k)/4) mod 256, tree; rows to n mod 256, tree)
 *   t[n,k]   = clamp(rint(W[n,k] * s_w[g(k)]), -1, 1), packed as before
 *   s_x[m,g] = 127 / max(max_{k in g} |x_n[m,k]|, 1e-5)
 *   x_q[m,k] = clamp(rint(x_n[m,k] * s_x[m,g(k)]), -128, 127)
 *   acc[m,n,g] = sum_{k in g} x_q t
 *   term_g   = (float)acc[m,n,g] / (s_x[m,g] * s_w[g])   (fp32 as oracle_dequant)
 *   y[m,n]   = sum_g term_g, summed in fp64 and rounded once to fp32.
 * With group_k = K this is exactly the per-tensor forward.
 */
int oracle_group_weight_scale(const float *W, int64_t N, int64_t K, int64_t group_k,
                              float *s_w) {
    if (!W || !s_w || N <= 0 || K <= 0 || group_k <= 0 || (K % group_k) != 0)
        return ORACLE_ERR_ARG;
    const int64_t G = K / group_k;
    for (int64_t g = 0; g < G; ++g) {
        double q[NPART];
        for (int i = 0; i < NPART; ++i) q[i] = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double p[NPART];
            for (int i = 0; i < NPART; ++i) p[i] = 0.0;
            for (int64_t kl = 0; kl < group_k; ++kl) {
                int idx = (int)((kl / 4) % NPART);
                p[idx] = p[idx] + fabs((double)W[n * K + g * group_k + kl]);
            }
            double Rn = tree_f64(p);
            int j = (int)(n % NPART);
            q[j] = q[j] + Rn;
        }
        double S = tree_f64(q);
        float mean = (float)(S / (double)(N * group_k));
        if (mean < 1e-5f) mean = 1e-5f;
        s_w[g] = 1.0f / mean;
    }
    return ORACLE_OK;
}

int oracle_group_quantize_pack(const float *W, int64_t N, int64_t K, int64_t group_k,
                               const float *s_w, uint8_t *W_p) {
    if (!W || !s_w || !W_p || N <= 0 || K <= 0 || group_k <= 0 || (K % group_k) != 0 ||
        (K % 4) != 0)
        return ORACLE_ERR_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < K / 4; ++b) {
            unsigned byte = 0;
            for (int j = 0; j < 4; ++j) {
                int64_t k = 4 * b + j;
                int t = ternary_of(W[n * K + k], s_w[k / group_k]);
                byte |= (unsigned)(t + 1) << (2 * j);
            }
            W_p[n * (K / 4) + b] = (uint8_t)byte;
        }
    return ORACLE_OK;
}

int oracle_group_rmsnorm_quant_act(const void *x, int x_is_bf16, const float *gamma,
                                   float eps, int64_t M, int64_t K, int64_t group_k,
                                   int8_t *x_q, float *s_x) {
    if (!x || !x_q || !s_x || M < 0 || K <= 0 || eps < 0.0f || group_k <= 0 ||
        (K % group_k) != 0)
        return ORACLE_ERR_ARG;
    const int64_t G = K / group_k;
    for (int64_t m = 0; m < M; ++m) {
        float r = 0.0f;
        int zero_row = rms_inverse(x, x_is_bf16, m, K, eps, &r);
        for (int64_t g = 0; g < G; ++g) {
            float amax = 0.0f;
            for (int64_t k = g * group_k; k < (g + 1) * group_k; ++k) {
                float xn = 0.0f;
                if (!zero_row) {
                    float gm = gamma ? gamma[k] : 1.0f;
                    xn = (load_x(x, x_is_bf16, m * K + k) * r) * gm;
                }
                float a = fabsf(xn);
                if (a > amax) amax = a;
            }
            if (amax < 1e-5f) amax = 1e-5f;
            float sx = 127.0f / amax;
            s_x[m * G + g] = sx;
            for (int64_t k = g * group_k; k < (g + 1) * group_k; ++k) {
                float xn = 0.0f;
                if (!zero_row) {
                    float gm = gamma ? gamma[k] : 1.0f;
                    xn = (load_x(x, x_is_bf16, m * K + k) * r) * gm;
                }
                float q = rintf(xn * sx);
                if (q > 127.0f) q = 127.0f;
                if (q < -128.0f) q = -128.0f;
                x_q[m * K + k] = (int8_t)q;
            }
        }
    }
    return ORACLE_OK;
}

/* acc per group [M][ncols][G] and y [M][ncols] (fp32 and bf16, either may
 * be NULL) from already quantized activations and packed weights. */
int oracle_group_matmul_dequant(const int8_t *x_q, const float *s_x, const uint8_t *W_p,
                                const float *s_w, int64_t M, int64_t N, int64_t K,
                                int64_t group_k, const int64_t *cols, int64_t ncols,
                                int32_t *acc, float *y_f32, uint16_t *y_bf16) {
    if (!x_q || !s_x || !W_p || !s_w || M < 0 || N <= 0 || K <= 0 || group_k <= 0 ||
        (K % group_k) != 0 || (K % 4) != 0)
        return ORACLE_ERR_ARG;
    if (!cols && ncols != N) return ORACLE_ERR_ARG;
    const int64_t G = K / group_k;
    int err = ORACLE_OK;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) reduction(max : err)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t n = cols ? cols[c] : c;
            if (n < 0 || n >= N) { err = ORACLE_ERR_ARG; continue; }
            double ysum = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                int64_t s = 0;
                for (int64_t k = g * group_k; k < (g + 1) * group_k; ++k) {
                    int t = unpack_one(W_p, K, n, k);
                    int xv = x_q[m * K + k];
                    if (t > 0) s += xv;
                    else if (t < 0) s -= xv;
                }
                if (acc) acc[(m * ncols + c) * G + g] = (int32_t)s;
                float denom = s_x[m * G + g] * s_w[g];
                float term = (float)s / denom;
                ysum += (double)term;
            }
            float yv = (float)ysum;
            if (y_f32) y_f32[m * ncols + c] = yv;
            if (y_bf16) y_bf16[m * ncols + c] = float_to_bf16_bits_rne(yv);
        }
    }
    return err;
}
