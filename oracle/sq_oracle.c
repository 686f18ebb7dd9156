/*
 * sq_oracle.c -- plain, slow CPU oracle for the SmoothQuant smoothed W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load or run this code. It shares nothing with the CUDA library: no header, no helper,
 * no table. Every step is written the way the pages state it, in plain loops, so that a reader
 * can check it against them by eye.
 *
 * Pages cited (title, then section / equation / figure):
 *   [MIGRATE] "06 -- SmoothQuant: Migrating Difficulty from Activations to Weights"
 *   [TAMING]  "Taming the Outliers: A Deep Dive into SmoothQuant for LLM Quantization"
 *   [W8A8]    "SmoothQuant and W8A8: Quantizing Activations Too"
 *   [WOVS]    "SmoothQuant: Weight-Only vs W8A8"
 *
 * Readings where the pages are silent or disagree:
 *   - Quantiser: symmetric, delta = max|v| / 127, code = round-half-away-from-zero(v * (127/max|v|)),
 *     clamped to [-127, 127]. The pages leave the tie rule open ([TAMING], "Why Outliers Break
 *     Quantization") or use half-to-even in a listing; half-away is the fixed reading. The
 *     reciprocal-multiply form (v * fl32(127/m)) is the fixed reading of dividing v by delta, and
 *     the product is rounded once, to the integer (not first to binary32).
 *   - All per-element arithmetic is binary32 with each operation rounded (compile with
 *     -ffp-contract=off, no fast-math); the RMSNorm sum of squares is accumulated in binary64.
 *   - RMSNorm is the standard x / sqrt(mean(x^2) + eps) * gamma (the pages name RMSNorm but do not
 *     print it).
 *   - Scale floors: both abs-maxima and s itself are floored at 1e-5 (binary32 constant).
 *   - Static per-tensor scale: the maximum of the smoothed activation over the calibration tokens,
 *     delta = m / 127, codes clamped at +-127 (see the static-scale section below).
 *   - FP8: the OCP E4M3 "FN" format, scale m / 448, round to nearest even with saturation at
 *     +-448, the sign kept on zero (see the FP8 section below).
 *   - LayerNorm (not printed on the pages): the standard per-token form, mean and centred sum of
 *     squares in binary64, every other step rounded to binary32 (see the LayerNorm section below).
 *
 * bf16 tensors are passed as uint16_t bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_FLOOR 1e-5f
#define ORC_QMAX 127

/* bf16 -> binary32 is exact: the bf16 bits are the high half of the binary32 pattern. */
static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even. The 16 dropped bits are the remainder:
 * more than half an ulp rounds the magnitude up, exactly half rounds to the even neighbour.
 * A carry out of the mantissa moves into the exponent, which is the correct next value. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays a quiet NaN */
    uint32_t kept = u & 0xFFFF0000u;
    uint32_t rem = u & 0x0000FFFFu;
    if (rem > 0x8000u || (rem == 0x8000u && (kept & 0x00010000u) != 0u))
        kept += 0x00010000u;
    return (uint16_t)(kept >> 16);
}

uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
float orc_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }

/* Symmetric INT8 code of one value, [TAMING] "Why Outliers Break Quantization" (quantisation
 * equation): v / delta rounded to the nearest integer, with v / delta taken as v * fl32(127 / m).
 * The product of two binary32 values is exact in binary64 (48 significant bits), so the integer
 * rounding is applied to the exact product, once; C99's round() is round-half-away-from-zero.
 * An infinite inv_delta (a static scale whose 127 / m overflowed) makes t = 0 * inf = NaN for a zero
 * value: the code of a zero value is 0 whatever the scale. */
static int8_t quantize_one(float v, float inv_delta)
{
    double t = (double)v * (double)inv_delta;
    if (isnan(t)) return 0;
    double r = round(t);
    if (r > (double)ORC_QMAX) r = (double)ORC_QMAX;
    if (r < -(double)ORC_QMAX) r = -(double)ORC_QMAX;
    return (int8_t)r;
}

/* Quantise one row of already-smoothed binary32 values with one symmetric scale:
 * m = max|v|, delta = m / 127, codes = round(v * (127 / m)). A zero row gives delta 0, codes 0.
 * [MIGRATE] section 7 (one scale per output row / per token), [W8A8] "One layer, measured".
 * When 127 / m overflows binary32 (m below 127 / FLT_MAX, about 3.7e-37), the row is first scaled by
 * 2^64 -- exact, and the quantiser is scale-free -- so that the reciprocal is finite:
 * codes = round((v * 2^64) * (127 / (m * 2^64))); delta stays m / 127. */
static void quantize_row(const float *v, int64_t n, int8_t *q, float *delta_out)
{
    float m = 0.0f;
    for (int64_t k = 0; k < n; ++k) {
        float a = fabsf(v[k]);
        if (a > m) m = a;
    }
    if (m == 0.0f) {
        for (int64_t k = 0; k < n; ++k) q[k] = 0;
        *delta_out = 0.0f;
        return;
    }
    float delta = m / (float)ORC_QMAX;
    float inv = (float)ORC_QMAX / m;
    float pre = 1.0f;
    if (isinf(inv)) {
        pre = 0x1p64f;
        inv = (float)ORC_QMAX / (m * pre);
    }
    for (int64_t k = 0; k < n; ++k) q[k] = quantize_one(v[k] * pre, inv);
    *delta_out = delta;
}

/* Inverse RMS of one bf16 row: 1 / sqrt(mean(x^2) + eps), sum of squares in binary64 taken in
 * index order, then each later step rounded to binary32. */
static float row_inv_rms(const uint16_t *x, int64_t K, float eps)
{
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double v = (double)bf16_to_f32(x[k]);
        ss += v * v;
    }
    float ms = (float)(ss / (double)K);
    float r = sqrtf(ms + eps);
    return 1.0f / r;
}

/*
 * Per-input-channel abs-max over the rows of a row-major bf16 matrix a[rows, cols] (leading
 * dimension ld elements): amax[j] = max_r |a[r, j]|.
 *   [MIGRATE] section 3 (max|X_j| from calibration samples); [TAMING] "System Architecture"
 *   (the flowchart's per-channel maximum of |X| and of |W|).
 * With norm_gamma non-null each row is first replaced by its RMSNorm output
 *   y = (x * inv_rms) * gamma_j,
 * the input the linear layer actually sees (per [W8A8] "The trick: move the range into the weights",
 * the smoothed layers read the output of a norm).
 * accumulate != 0 keeps a running maximum with the values already in amax (calibration over
 * several batches); otherwise amax is overwritten.
 * For a weight stored [N, K] (output channel n, input channel k) the same call over rows n gives
 * max|W_k| per input channel.
 */
void orc_calibrate_absmax(const uint16_t *a, int64_t rows, int64_t cols, int64_t ld,
                          const float *norm_gamma, float eps, float *amax, int accumulate)
{
    if (!accumulate)
        for (int64_t j = 0; j < cols; ++j) amax[j] = 0.0f;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *row = a + r * ld;
        float ir = norm_gamma ? row_inv_rms(row, cols, eps) : 1.0f;
        for (int64_t j = 0; j < cols; ++j) {
            float v = bf16_to_f32(row[j]);
            if (norm_gamma) v = (v * ir) * norm_gamma[j];
            float av = fabsf(v);
            if (av > amax[j]) amax[j] = av;
        }
    }
}

/*
 * Smoothing factors, [MIGRATE] section 3 and [W8A8] "The trick: move the range into the weights":
 *   s_j = max|X_j|^alpha / max|W_j|^(1 - alpha),
 * evaluated in binary64 and rounded once to binary32, then floored at 1e-5 as in the
 * [TAMING] "Implementation in PyTorch" listing (clamp of s). Both abs-maxima are floored at 1e-5
 * first so that an all-zero channel gives a finite s.
 * The fold into the preceding norm, [W8A8] "The trick..." (s folded into the norm weights):
 *   fold_j = gamma_j / s_j, or 1 / s_j when gamma is null (no norm: the activations are divided
 *   by s directly, the smoothing node of the [TAMING] flowchart).
 * fold may be null.
 */
void orc_compute_scales(const float *amax_x, const float *amax_w, int64_t K, float alpha,
                        const float *gamma, float *s, float *fold)
{
    double ea = (double)alpha;
    double eb = 1.0 - (double)alpha;
    for (int64_t j = 0; j < K; ++j) {
        double a = (double)fmaxf(amax_x[j], ORC_FLOOR);
        double b = (double)fmaxf(amax_w[j], ORC_FLOOR);
        float sj = (float)(pow(a, ea) / pow(b, eb));
        sj = fmaxf(sj, ORC_FLOOR);
        s[j] = sj;
        if (fold) fold[j] = gamma ? gamma[j] / sj : 1.0f / sj;
    }
}

/*
 * Weight smoothing and per-output-channel INT8 quantisation.
 *   W_hat = diag(s) * W ([MIGRATE] section 2; the weight-update node of the [TAMING] flowchart): the weights
 *   that read input channel k are multiplied by s_k. Stored [N, K], that is column k.
 *   Then one symmetric scale per output row n ([MIGRATE] section 7).
 * s null means unsmoothed (s = 1).
 */
void orc_smooth_quantize_weight(const uint16_t *w, int64_t N, int64_t K, const float *s,
                                int8_t *wq, float *w_scale, float *work /* [K] */)
{
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *row = w + n * K;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_f32(row[k]);
            work[k] = s ? v * s[k] : v;
        }
        quantize_row(work, K, wq + n * K, &w_scale[n]);
    }
}

/*
 * Online activation path for T tokens of width K.
 *   apply_norm != 0: y = (x * inv_rms) * fold_k with fold = gamma / s folded into the RMSNorm
 *   weight ([W8A8] "The trick..."); apply_norm == 0: y = x * fold_k with fold = 1 / s
 *   (the smoothing node of the [TAMING] flowchart).
 *   Then one dynamic symmetric scale per token ([MIGRATE] section 7; [W8A8] "The full model,
 *   served": each token's maximum is found before the matrix product).
 */
void orc_rmsnorm_smooth_quant(const uint16_t *x, int64_t T, int64_t K, const float *fold,
                              float eps, int apply_norm, int8_t *xq, float *x_scale,
                              float *work /* [K] */)
{
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *row = x + t * K;
        float ir = apply_norm ? row_inv_rms(row, K, eps) : 1.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_f32(row[k]);
            work[k] = apply_norm ? (v * ir) * fold[k] : v * fold[k];
        }
        quantize_row(work, K, xq + t * K, &x_scale[t]);
    }
}

/*
 * Static per-tensor activation scale, [W8A8] "One layer, measured" (one static scale per tensor,
 * taken from the calibration tokens' maximum) and "Gotchas" (values past the calibrated maximum are
 * clipped). amax_y[k] is the per-channel maximum, over the calibration tokens, of the smoothed
 * activation exactly as the online quantiser forms it (the calibration abs-max with the fold in
 * place of gamma). The tensor maximum is m = max_k amax_y[k]; scale2[0] = delta = m / 127 and
 * scale2[1] = 127 / m, the same two values the per-token quantiser derives from a row maximum
 * (m == 0 gives 0 and 0).
 */
void orc_static_scale(const float *amax_y, int64_t K, float *scale2)
{
    float m = 0.0f;
    for (int64_t k = 0; k < K; ++k)
        if (amax_y[k] > m) m = amax_y[k];
    if (m == 0.0f) {
        scale2[0] = 0.0f;
        scale2[1] = 0.0f;
        return;
    }
    scale2[0] = m / (float)ORC_QMAX;
    scale2[1] = (float)ORC_QMAX / m;
}

/*
 * Online activation quantisation with the static per-tensor scale: the smoothed (and, with
 * apply_norm, normalised) activation y is formed exactly as in orc_rmsnorm_smooth_quant, then
 * every value is coded with the one calibrated scale: q = clamp(round_half_away(y * scale2[1]),
 * -127, 127) (values beyond the calibrated maximum saturate), and every token's scale is
 * scale2[0], so the dequantisation is the scalar step times the per-channel weight scale.
 *   [W8A8] "One layer, measured" and "Gotchas"; the quantiser of [TAMING] "Why Outliers Break
 *   Quantization".
 */
void orc_rmsnorm_smooth_quant_static(const uint16_t *x, int64_t T, int64_t K, const float *fold,
                                     float eps, int apply_norm, const float *scale2, int8_t *xq,
                                     float *x_scale)
{
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *row = x + t * K;
        float ir = apply_norm ? row_inv_rms(row, K, eps) : 1.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_f32(row[k]);
            float y = apply_norm ? (v * ir) * fold[k] : v * fold[k];
            xq[t * K + k] = quantize_one(y, scale2[1]);
        }
        x_scale[t] = scale2[0];
    }
}

/*
 * Fold of the smoothing into the previous linear layer, [MIGRATE] section 7 (the division X / s is
 * absorbed by multiplying the previous layer's output-column-j weights by 1 / s_j, so the smoothed
 * layer's input arrives already divided). The previous layer's weight is stored [K, Kp] (output
 * channel j of that layer = input channel j of the smoothed one), bf16:
 *   w_out[j, i] = bf16_rn(w[j, i] * f[j]),  b_out[j] = bf16_rn(b[j] * f[j]),  f = fl32(1 / s) (the
 *   fold vector of orc_compute_scales without gamma).
 * For an INT8 previous layer the same factor goes into its per-output-channel dequantisation:
 *   w_scale_out[j] = w_scale[j] * f[j] (binary32); its bias as above.
 */
void orc_fold_into_prev_linear(const uint16_t *w, const uint16_t *b, int64_t K, int64_t Kp, const float *f,
                               uint16_t *w_out, uint16_t *b_out)
{
    for (int64_t j = 0; j < K; ++j) {
        for (int64_t i = 0; i < Kp; ++i)
            w_out[j * Kp + i] = f32_to_bf16_rne(bf16_to_f32(w[j * Kp + i]) * f[j]);
        if (b) b_out[j] = f32_to_bf16_rne(bf16_to_f32(b[j]) * f[j]);
    }
}

void orc_fold_into_w_scale(const float *w_scale, int64_t K, const float *f, float *w_scale_out)
{
    for (int64_t j = 0; j < K; ++j) w_scale_out[j] = w_scale[j] * f[j];
}

/* ---------------------------------------------------------------------------------------------
 * LayerNorm-fed layers, [WOVS] "Integration with Transformers" (the run-time division by S costs
 * nothing: S^-1 is folded into the scale gamma and the bias beta of the preceding LayerNorm, so
 * activations leave the norm already smoothed). LayerNorm is not printed on the pages; the standard form is used:
 *   mu = (sum_k x_k) / K in binary64, m = fl32(mu);  c_k = fl32(x_k - m);
 *   var = (sum_k c_k^2) / K in binary64 (each square exact), ms = fl32(var);
 *   r = fl32(sqrt(fl32(ms + eps))), ir = fl32(1 / r);
 *   y_k = fl32(fl32(fl32(c_k * ir) * g_k) + b_k)
 * with g = gamma, b = beta for calibration, and g = fold = fl32(gamma / s), b = fl32(beta / s) online.
 */
static float row_layernorm(const uint16_t *x, int64_t K, float eps, float *c)
{
    double sum = 0.0;
    for (int64_t k = 0; k < K; ++k) sum += (double)bf16_to_f32(x[k]);
    float m = (float)(sum / (double)K);
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        c[k] = bf16_to_f32(x[k]) - m;
        ss += (double)c[k] * (double)c[k];
    }
    float ms = (float)(ss / (double)K);
    float r = sqrtf(ms + eps);
    return 1.0f / r;
}

/* Per-channel abs-max of the LayerNorm output y = LN(x) * gamma + beta over the rows (running maximum
 * with accumulate != 0). work holds K floats. */
void orc_calibrate_absmax_layernorm(const uint16_t *a, int64_t rows, int64_t cols, int64_t ld, const float *gamma,
                                    const float *beta, float eps, float *amax, int accumulate, float *work)
{
    if (!accumulate)
        for (int64_t j = 0; j < cols; ++j) amax[j] = 0.0f;
    for (int64_t r = 0; r < rows; ++r) {
        float ir = row_layernorm(a + r * ld, cols, eps, work);
        for (int64_t j = 0; j < cols; ++j) {
            float y = (work[j] * ir) * gamma[j] + beta[j];
            float v = fabsf(y);
            if (v > amax[j]) amax[j] = v;
        }
    }
}

/* The LayerNorm bias with S^-1 folded in: beta_fold[k] = fl32(beta[k] / s[k]). */
void orc_fold_layernorm_bias(const float *beta, const float *s, int64_t K, float *beta_fold)
{
    for (int64_t k = 0; k < K; ++k) beta_fold[k] = beta[k] / s[k];
}

/* LayerNorm with the folded scale and bias, then per-token symmetric INT8 (the quantiser above). */
void orc_layernorm_smooth_quant(const uint16_t *x, int64_t T, int64_t K, const float *fold, const float *beta_fold,
                                float eps, int8_t *xq, float *x_scale, float *work /* [2K] */)
{
    float *c = work, *y = work + K;
    for (int64_t t = 0; t < T; ++t) {
        float ir = row_layernorm(x + t * K, K, eps, c);
        for (int64_t k = 0; k < K; ++k) y[k] = (c[k] * ir) * fold[k] + beta_fold[k];
        quantize_row(y, K, xq + t * K, &x_scale[t]);
    }
}

/* ---------------------------------------------------------------------------------------------
 * FP8 E4M3 variant, [W8A8] "One layer, measured" (the same sweep in FP8 E4M3) and "FP8's exponent
 * gives each value its own scale". E4M3 (the OCP "FN" form): 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits; normals (1 + m/8) * 2^(e-7) for e = 1..15 except the pattern S.1111.111
 * (NaN), so the largest finite value is 448; subnormals (m/8) * 2^-6. Reading: scales are
 * delta = max|v| / 448 with codes e4m3(v * fl32(448 / max|v|)), rounded to nearest (ties to even)
 * with saturation to +-448, the FP8 counterpart of the INT8 quantiser above.
 */
#define ORC_F8MAX 448.0f

/* Nearest E4M3 value to a (a >= 0, finite), ties to even, saturating at 448; returned as its code
 * (exponent and mantissa bits, sign bit clear). */
static uint8_t e4m3_code_abs(float a)
{
    if (a >= ORC_F8MAX) return 0x7E;                      /* 448 (anything above saturates) */
    if (a < 0x1p-6f) {                                     /* subnormal grid, step 2^-9 */
        float q = nearbyintf(a * 0x1p9f);                  /* exact scaling; default mode is nearest-even */
        return (uint8_t)q;                                 /* q = 8 is the smallest normal, code 0x08 */
    }
    int e;
    frexpf(a, &e);                                         /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                                /* a in [2^e, 2^(e+1)) */
    float q = nearbyintf(ldexpf(a, 3 - e));                /* multiples of 2^(e-3): q in [8, 16] */
    int ee = e + 7, m = (int)q - 8;
    if (m == 8) { ee += 1; m = 0; }                        /* rounded up into the next binade */
    if (ee > 15 || (ee == 15 && m > 6)) return 0x7E;       /* beyond 448 after rounding: saturate */
    return (uint8_t)((ee << 3) | m);
}

static uint8_t e4m3_encode(float v)
{
    uint8_t c = e4m3_code_abs(fabsf(v));
    return signbit(v) ? (uint8_t)(c | 0x80) : c;           /* the sign is kept, also on a zero */
}

static float e4m3_decode(uint8_t c)
{
    int e = (c >> 3) & 15, m = c & 7;
    float a = e == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
    return (c & 0x80) ? -a : a;
}

uint8_t orc_e4m3_encode(float v) { return e4m3_encode(v); }
float orc_e4m3_decode(uint8_t c) { return e4m3_decode(c); }

/* One row of smoothed binary32 values to E4M3 with one scale: m = max|v|, delta = m / 448,
 * codes e4m3(v * fl32(448 / m)); a zero row gives delta 0 and codes 0. When 448 / m overflows
 * binary32 (m below 448 / FLT_MAX), the row is first scaled by 2^64 (exact), as in the INT8 quantiser. */
static void quantize_row_f8(const float *v, int64_t n, uint8_t *q, float *delta_out)
{
    float m = 0.0f;
    for (int64_t k = 0; k < n; ++k) {
        float a = fabsf(v[k]);
        if (a > m) m = a;
    }
    if (m == 0.0f) {
        for (int64_t k = 0; k < n; ++k) q[k] = 0;
        *delta_out = 0.0f;
        return;
    }
    float inv = ORC_F8MAX / m;
    float pre = 1.0f;
    if (isinf(inv)) {
        pre = 0x1p64f;
        inv = ORC_F8MAX / (m * pre);
    }
    for (int64_t k = 0; k < n; ++k) q[k] = e4m3_encode((v[k] * pre) * inv);
    *delta_out = m / ORC_F8MAX;
}

/* Smoothed weight in E4M3, one scale per output channel (the FP8 form of orc_smooth_quantize_weight). */
void orc_smooth_quantize_weight_f8(const uint16_t *w, int64_t N, int64_t K, const float *s, uint8_t *wq,
                                   float *w_scale, float *work)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_f32(w[n * K + k]);
            work[k] = s ? v * s[k] : v;
        }
        quantize_row_f8(work, K, wq + n * K, &w_scale[n]);
    }
}

/* RMSNorm with the folded weight (or x * fold), then E4M3 with one dynamic scale per token. */
void orc_rmsnorm_smooth_quant_f8(const uint16_t *x, int64_t T, int64_t K, const float *fold, float eps,
                                 int apply_norm, uint8_t *xq, float *x_scale, float *work)
{
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *row = x + t * K;
        float ir = apply_norm ? row_inv_rms(row, K, eps) : 1.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_to_f32(row[k]);
            work[k] = apply_norm ? (v * ir) * fold[k] : v * fold[k];
        }
        quantize_row_f8(work, K, xq + t * K, &x_scale[t]);
    }
}

/* FP8 product accumulated exactly: acc[t, n] = sum_k e4m3(xq[t,k]) * e4m3(wq[n,k]) in binary64.
 * Each product has at most 8 significant bits and lies in [2^-18, 2^18], so for K <= 2^20 the
 * binary64 sum is exact (the tensor cores accumulate in binary32; tests bound that difference). */
void orc_gemm_f8(const uint8_t *xq, int64_t T, const uint8_t *wq, int64_t N, int64_t K, const int64_t *row_idx,
                 int64_t nrows, const int64_t *col_idx, int64_t ncols, double *acc)
{
    if (!row_idx) nrows = T;
    if (!col_idx) ncols = N;
    double table[256];                                     /* the value of every code */
    for (int c = 0; c < 256; ++c) table[c] = (double)e4m3_decode((uint8_t)c);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t t = row_idx ? row_idx[i] : i;
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t n = col_idx ? col_idx[c] : c;
            double sum = 0.0;
            for (int64_t k = 0; k < K; ++k) sum += table[xq[t * K + k]] * table[wq[n * K + k]];
            acc[i * ncols + c] = sum;
        }
    }
}

/* Dequantisation of binary32 accumulators (the FP8 form): y = bf16(acc * (x_scale * w_scale) + bias),
 * the same steps as orc_dequant. */
void orc_dequant_f32(const float *acc, const float *x_scale, const float *w_scale, const uint16_t *bias,
                     const int64_t *row_idx, int64_t nrows, const int64_t *col_idx, int64_t ncols, uint16_t *y)
{
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t t = row_idx ? row_idx[i] : i;
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t n = col_idx ? col_idx[c] : c;
            float sc = x_scale[t] * w_scale[n];
            float v = acc[i * ncols + c] * sc;
            if (bias) v = v + bf16_to_f32(bias[n]);
            y[i * ncols + c] = f32_to_bf16_rne(v);
        }
    }
}

/*
 * INT8 x INT8 -> INT32 product of the quantised activations xq[T, K] and weights wq[N, K]
 * (both stored with K contiguous): acc[t, n] = sum_k xq[t, k] * wq[n, k].
 * [MIGRATE] section 7 (an integer product accumulated in 32 bits on the tensor cores); the GEMM
 * node of the [TAMING] flowchart. Exact: |acc| <= K * 127^2 < 2^31 for K <= 133,000.
 * Computed for the listed token rows and output columns only (all of them when the lists are
 * null); acc is [nrows, ncols].
 */
void orc_gemm_s8(const int8_t *xq, int64_t T, const int8_t *wq, int64_t N, int64_t K,
                 const int64_t *row_idx, int64_t nrows, const int64_t *col_idx, int64_t ncols,
                 int32_t *acc)
{
    if (!row_idx) nrows = T;
    if (!col_idx) ncols = N;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t t = row_idx ? row_idx[i] : i;
        const int8_t *xr = xq + t * K;
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t n = col_idx ? col_idx[c] : c;
            const int8_t *wr = wq + n * K;
            int32_t sum = 0;
            for (int64_t k = 0; k < K; ++k) sum += (int32_t)xr[k] * (int32_t)wr[k];
            acc[i * ncols + c] = sum;
        }
    }
}

/*
 * Dequantisation epilogue, [MIGRATE] section 7 (Y = scale_x * scale_w * Y_int32) and the
 * bias-and-dequantise node of the [TAMING] flowchart:
 *   y[t, n] = bf16( float(acc) * (x_scale[t] * w_scale[n]) + bias[n] ),
 * each operation rounded to binary32, the bias (bf16, optional) added last.
 * acc is [nrows, ncols] for the listed rows / columns (all when the lists are null).
 */
void orc_dequant(const int32_t *acc, const float *x_scale, const float *w_scale,
                 const uint16_t *bias, const int64_t *row_idx, int64_t nrows,
                 const int64_t *col_idx, int64_t ncols, uint16_t *y)
{
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t t = row_idx ? row_idx[i] : i;
        for (int64_t c = 0; c < ncols; ++c) {
            int64_t n = col_idx ? col_idx[c] : c;
            float sc = x_scale[t] * w_scale[n];
            float v = (float)acc[i * ncols + c] * sc;
            if (bias) v = v + bf16_to_f32(bias[n]);
            y[i * ncols + c] = f32_to_bf16_rne(v);
        }
    }
}
