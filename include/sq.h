/*
 * sq.h -- C ABI of libsq, the SmoothQuant smoothed W8A8 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer, as the pages describe it:
 *   offline  per-input-channel abs-maxima of calibration activations and of the weight,
 *            smoothing factors s_j = max|X_j|^alpha / max|W_j|^(1-alpha), the smoothed weight
 *            diag(s) * W quantised to INT8 with one scale per output channel;
 *   online   1/s folded into the preceding RMSNorm weight (or a LayerNorm's gamma and beta, or
 *            the previous linear layer), per-token dynamic symmetric INT8 quantisation of the
 *            normalised activations (or one static per-tensor scale), INT8 x INT8 -> INT32 GEMM, and
 *            a dequantisation epilogue (per-token scale x per-channel scale, plus bias) to bf16;
 *            the same path in FP8 E4M3.
 *
 * Pages cited (title, then section / equation / figure):
 *   [MIGRATE] "06 -- SmoothQuant: Migrating Difficulty from Activations to Weights"
 *   [TAMING]  "Taming the Outliers: A Deep Dive into SmoothQuant for LLM Quantization"
 *   [W8A8]    "SmoothQuant and W8A8: Quantizing Activations Too"
 *   [WOVS]    "SmoothQuant: Weight-Only vs W8A8"
 *
 * Conventions for every entry point
 *   - Tensor pointers are caller-owned DEVICE memory on the current CUDA device. The library
 *     allocates nothing and keeps no pointer after a call returns.
 *   - Matrices are row-major. bf16 data is passed as `const void *` (IEEE bfloat16 bit patterns).
 *     Sizes are element counts (int64_t).
 *   - `stream` is a cudaStream_t passed as `void *` (NULL = the legacy default stream). Each call
 *     enqueues its kernels on that stream and returns without synchronising; only
 *     sq_device_status() synchronises. Kernels are launched as programmatic dependent launches:
 *     one may be scheduled while the previous kernel of the stream is finishing, but it reads and
 *     writes no global memory before that kernel has completed (griddepcontrol.wait), so stream
 *     order holds for every input and output, whoever wrote them.
 *   - Outputs must not alias inputs.
 *   - Arguments are validated before anything is launched; a failed check returns its code and
 *     launches nothing. sq_last_error() then gives a one-line reason (per host thread).
 *   - Arithmetic: binary32 with every operation separately rounded (no contraction into fused
 *     multiply-adds), except the norm sums (binary64: the RMSNorm sum of squares, the LayerNorm sum
 *     and centred sum of squares) and the smoothing-factor power (binary64, rounded once to
 *     binary32). INT8 codes use round-half-away-from-zero and are clamped to [-127, 127].
 *   - Rows of very small values: every per-row quantiser (weights, tokens, INT8 and FP8) codes a row
 *     with m = max|v| as round(v * fl(qmax / m)), qmax = 127 (448 for FP8). When qmax / m overflows
 *     binary32 (m below about 3.7e-37 for INT8, 1.3e-36 for FP8), the row is first multiplied by 2^64
 *     (exact) and coded as round(fl(v * 2^64) * fl(qmax / fl(m * 2^64))); its scale is still m / qmax.
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SQ_OK = 0,
    SQ_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size, alpha outside [0,1] */
    SQ_ERR_UNSUPPORTED = 2,   /* a size the library does not handle (limits stated per call) */
    SQ_ERR_MISALIGNED = 3,    /* pointer or leading dimension not aligned as required */
    SQ_ERR_ARCH = 4,          /* current device is not compute capability 10.0 (B200 class) */
    SQ_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
    SQ_ERR_TIMEOUT = 6,       /* a bounded device-side wait ran out (reported by sq_device_status) */
    SQ_ERR_BOUNDS = 7         /* checked build only: a device-side bounds check failed and its access
                                 was skipped (reported by sq_device_status) */
} sq_status;

/* Name of a status code ("SQ_OK", ...). Never NULL. */
const char *sq_status_string(int status);

/* One-line reason for the last non-SQ_OK status returned on this host thread ("" if none). */
const char *sq_last_error(void);

/* Library version string. */
const char *sq_version(void);

/*
 * Per-input-channel abs-max: amax[j] = max over rows r of |a[r, j]|.
 *   [MIGRATE] section 3 "How to choose s" (max|X_j| from calibration samples);
 *   [TAMING] "System Architecture" (the flowchart's per-channel maximum of |X| and of |W|).
 * a          bf16 [rows, cols], row stride `ld` elements. For activations: calibration tokens x
 *            channels. For a weight stored [N, K] (nn.Linear orientation), rows = N, cols = K gives
 *            max|W_k| per input channel k.
 * norm_gamma nullable fp32 [cols]. When given, each row is replaced by its RMSNorm output
 *            (x / sqrt(mean(x^2) + eps)) * gamma before the reduction -- the input the linear
 *            layer actually sees when it is fed by a norm ([W8A8] "The trick: move the range into
 *            the weights").
 * amax       fp32 [cols], in/out. accumulate = 0 overwrites it; accumulate = 1 keeps a running
 *            maximum with its current contents (calibration streamed in batches).
 * Requirements: rows >= 0, 8 <= cols <= 16384 (else SQ_ERR_UNSUPPORTED), cols % 8 == 0, ld % 8 == 0,
 * ld >= cols, `a` and norm_gamma 16-byte aligned, amax 4-byte aligned.
 * rows == 0 with accumulate = 0 sets amax to 0. With norm_gamma, rows whose values all lie below
 * 2^-100 in magnitude (or contain subnormal bf16) may see the inexact squares of those values.
 */
sq_status sq_calibrate_absmax(const void *a, int64_t rows, int64_t cols, int64_t ld,
                              const float *norm_gamma, float eps, float *amax, int accumulate,
                              void *stream);

/*
 * Both maxima of one smoothing group in one launch: the same result as
 *   sq_calibrate_absmax(a, rows, cols, ld, norm_gamma, eps, amax, accumulate, stream) and then
 *   sq_calibrate_absmax(w, w_rows, cols, w_ld, NULL, 0, amax_w, accumulate, stream),
 * the activation maxima max|X_j| and the weight maxima max|W_j| that the smoothing factor of
 * [MIGRATE] section 3 combines. The two reductions are independent. When cols > 2048 and both inputs
 * have rows, one kernel reduces both: part of its CTAs streams the weight rows while the rest stream
 * the activation rows (the split follows the inputs' sizes). Otherwise the two reductions are
 * launched one after the other.
 * a, rows, ld, norm_gamma, eps, amax: as in sq_calibrate_absmax.
 * w          bf16 [w_rows, cols], row stride w_ld elements (a weight stored [N, K]); never normalised.
 * amax_w     fp32 [cols], in/out; must not overlap amax.
 * accumulate applies to both outputs (0 overwrites both, 1 keeps both running maxima).
 * Requirements: those of sq_calibrate_absmax for each input; amax and amax_w disjoint (else
 * SQ_ERR_INVALID_ARG).
 */
sq_status sq_calibrate_absmax_pair(const void *a, int64_t rows, int64_t cols, int64_t ld, const float *norm_gamma,
                                   float eps, float *amax, const void *w, int64_t w_rows, int64_t w_ld, float *amax_w,
                                   int accumulate, void *stream);

/*
 * Smoothing factors and the folded norm weight.
 *   [MIGRATE] section 3; [W8A8] "The trick: move the range into the weights" (formula and the
 *   fold into the norm's weights); clamp of s from [TAMING] "Implementation in PyTorch".
 *   s[j]    = max(fl32(pow(a_j, alpha) / pow(b_j, 1 - alpha)), 1e-5) with a_j = max(amax_x[j], 1e-5),
 *             b_j = max(amax_w[j], 1e-5), the powers and the quotient in binary64.
 *   fold[j] = gamma[j] / s[j]  (gamma non-null: the RMSNorm weight with 1/s folded in), or
 *             1 / s[j]         (gamma null: a layer fed directly, x is multiplied by 1/s).
 * amax_x, amax_w fp32 [K]; gamma nullable fp32 [K]; s fp32 [K] out; fold nullable fp32 [K] out.
 * 0 <= alpha <= 1 (alpha = 1: s = max|X_j|; alpha = 0: s = 1/max|W_j|). K >= 1.
 */
sq_status sq_compute_scales(const float *amax_x, const float *amax_w, int64_t K, float alpha,
                            const float *gamma, float *s, float *fold, void *stream);

/*
 * Smoothed weight, quantised to INT8 with one symmetric scale per output channel.
 *   W_hat = diag(s) * W: [MIGRATE] section 2 and section 7 (one scale per output row);
 *   [TAMING] "System Architecture" (the flowchart's weight-update and weight-quantisation nodes).
 *   w'[n,k] = w[n,k] * s[k]; m_n = max_k |w'[n,k]|; w_scale[n] = m_n / 127;
 *   wq[n,k] = clamp(round_half_away(w'[n,k] * (127 / m_n)), -127, 127); a zero row gives scale 0.
 * w bf16 [N, K]; s nullable fp32 [K] (null = unsmoothed); wq int8 [N, K] out; w_scale fp32 [N] out.
 * Requirements: N >= 0, K >= 8, K % 8 == 0, K <= 16384, w 16-byte aligned, wq 8-byte aligned.
 */
sq_status sq_smooth_quantize_weight(const void *w, int64_t N, int64_t K, const float *s,
                                    int8_t *wq, float *w_scale, void *stream);

/*
 * Online activation quantisation, fused with the RMSNorm that carries the folded 1/s.
 *   [W8A8] "The trick: move the range into the weights" (1/s folded into the norm weight);
 *   [MIGRATE] section 7 (X' INT8 with one scale per token); [W8A8] "The full model, served"
 *   (a dynamic scale means finding each token's maximum before every matrix product).
 *   apply_norm = 1: y[t,k] = (x[t,k] * inv_rms_t) * fold[k], inv_rms_t = 1 / sqrt(mean_k x^2 + eps)
 *   apply_norm = 0: y[t,k] = x[t,k] * fold[k]            (fold = 1/s; eps ignored)
 *   m_t = max_k |y[t,k]|; x_scale[t] = m_t / 127; xq[t,k] = clamp(round_half_away(y * (127/m_t)), +-127).
 * x bf16 [T, K]; fold fp32 [K]; xq int8 [T, K] out; x_scale fp32 [T] out.
 * Requirements: T >= 0, K >= 8, K % 8 == 0, K <= 16384, x 16-byte aligned, xq 8-byte aligned.
 */
sq_status sq_rmsnorm_smooth_quant(const void *x, int64_t T, int64_t K, const float *fold, float eps,
                                  int apply_norm, int8_t *xq, float *x_scale, void *stream);

/*
 * Static per-tensor activation scale (the alternative to per-token scales):
 *   [W8A8] "One layer, measured" (one static scale per tensor, from the calibration tokens' maximum)
 *   and "Gotchas" (values past the calibrated maximum are clipped).
 *   m = max_k fl32(amax[k] * |factor[k]|)  (factor null: m = max_k amax[k]);
 *   scale2[0] = fl32(m / 127), scale2[1] = fl32(127 / m); both 0 when m = 0.
 * amax is the per-channel calibration maximum of the activation as the quantiser will form it:
 *   norm-fed layer: sq_calibrate_absmax(calibration tokens, norm_gamma = fold) (the RMSNorm output
 *   times the folded weight), factor = NULL;
 *   layer fed directly: sq_calibrate_absmax(calibration tokens) and factor = fold (= 1/s).
 * Rounding is monotone, so either way m equals the largest |y| the quantiser would form on the
 * calibration tokens. amax fp32 [K]; factor nullable fp32 [K]; scale2 fp32 [2] out (device memory).
 * K >= 1. When 127 / m overflows binary32 (m below about 3.7e-37), scale2[1] is +infinity: the static
 * quantiser then codes every zero value 0 and saturates every other value at +-127.
 */
sq_status sq_static_scale(const float *amax, const float *factor, int64_t K, float *scale2, void *stream);

/*
 * Online activation quantisation with the static per-tensor scale: y as in
 * sq_rmsnorm_smooth_quant, then xq[t,k] = clamp(round_half_away(y * scale2[1]), -127, 127) (values
 * beyond the calibrated maximum saturate) and x_scale[t] = scale2[0] for every token, so
 * sq_w8a8_linear dequantises with the scalar step times the per-channel weight scale. No per-token
 * maximum is taken. scale2 fp32 [2] from sq_static_scale (device memory, read by the kernel).
 * Same arguments and requirements as sq_rmsnorm_smooth_quant otherwise; scale2 4-byte aligned.
 */
sq_status sq_rmsnorm_smooth_quant_static(const void *x, int64_t T, int64_t K, const float *fold, float eps,
                                         int apply_norm, const float *scale2, int8_t *xq, float *x_scale,
                                         void *stream);

/*
 * Fold of the smoothing into the previous linear layer instead of a norm:
 *   [MIGRATE] section 7 (multiply the previous layer's output-column-j weights by 1/s_j; the
 *   smoothed layer's input then arrives divided by s, at no run-time cost).
 * The previous layer's weight w is bf16 [K, Kp] row-major (row j = its output channel j = input
 * channel j of the smoothed layer), its bias b nullable bf16 [K]; fold fp32 [K] = fl32(1/s) (from
 * sq_compute_scales with gamma = NULL):
 *   w_out[j, i] = bf16_rn(w[j, i] * fold[j]),  b_out[j] = bf16_rn(b[j] * fold[j]).
 * The smoothed layer then quantises its input with fold = 1 (sq_rmsnorm_smooth_quant, apply_norm 0).
 * w_out / b_out may equal w / b (in place). Requirements: K >= 0, Kp >= 8, Kp % 8 == 0; w, w_out
 * 16-byte aligned; b_out required when b is given.
 */
sq_status sq_fold_into_prev_linear(const void *w, const void *b, int64_t K, int64_t Kp, const float *fold,
                                   void *w_out, void *b_out, void *stream);

/*
 * The same fold for an INT8 previous layer: its per-output-channel dequantisation scale absorbs it,
 * w_scale_out[j] = fl32(w_scale[j] * fold[j]) (its bf16 bias as in sq_fold_into_prev_linear).
 * fp32 [K] arrays, K >= 1; w_scale_out may equal w_scale.
 */
sq_status sq_fold_into_w_scale(const float *w_scale, int64_t K, const float *fold, float *w_scale_out, void *stream);

/*
 * LayerNorm-fed layers: the fold of S^-1 into the scale gamma and the bias beta of the LayerNorm in
 * front of the smoothed layer ([WOVS] "Integration with Transformers": its output then leaves the
 * norm already smoothed, at no run-time cost). The pages do not write LayerNorm out; the standard
 * per-token form is used, each step rounded as listed (fl32 = round to nearest binary32):
 *   m = fl32(sum_k x_k / K);  c_k = fl32(x_k - m);  ms = fl32(sum_k c_k^2 / K)   (sums in binary64)
 *   ir = fl32(1 / fl32(sqrt(fl32(ms + eps))));   y_k = fl32(fl32(fl32(c_k * ir) * g_k) + b_k)
 *
 * sq_calibrate_absmax_layernorm: per-column abs-max of y over the rows of bf16 a [rows, cols]
 *   (row stride ld elements) with g = gamma, b = beta (fp32 [cols]; beta nullable = no bias), into
 *   amax fp32 [cols]; accumulate != 0 keeps the running maximum (amax must then hold non-negative
 *   values). Requirements as sq_calibrate_absmax; gamma and beta 16-byte aligned; cols <= 16384.
 * sq_fold_layernorm_bias: beta_fold[k] = fl32(beta[k] / s[k]), fp32 [K], K >= 1 (the scale side,
 *   fl32(gamma / s), is the fold sq_compute_scales writes when given gamma).
 * sq_layernorm_smooth_quant: y with g = fold, b = beta_fold (nullable = no bias), then per-token
 *   symmetric INT8 exactly as sq_rmsnorm_smooth_quant: x bf16 [T, K] -> xq int8 [T, K], x_scale fp32
 *   [T]. Requirements: T >= 0, 8 <= K <= 16384, K % 8 == 0; x, fold, beta_fold 16-byte aligned, xq
 *   8-byte aligned.
 * The binary64 sums are taken in a tree order (see the library's LayerNorm source for when that can
 * differ from index order).
 */
sq_status sq_calibrate_absmax_layernorm(const void *a, int64_t rows, int64_t cols, int64_t ld, const float *gamma,
                                        const float *beta, float eps, float *amax, int accumulate, void *stream);
sq_status sq_fold_layernorm_bias(const float *beta, const float *s, int64_t K, float *beta_fold, void *stream);
sq_status sq_layernorm_smooth_quant(const void *x, int64_t T, int64_t K, const float *fold, const float *beta_fold,
                                    float eps, int8_t *xq, float *x_scale, void *stream);

/*
 * W8A8 linear: INT8 x INT8 -> INT32 GEMM with the dequantisation fused into its epilogue.
 *   [MIGRATE] section 7 (the integer product accumulated in 32 bits on the tensor cores, then
 *   scaled by the activation and weight scales); [TAMING] "System Architecture" (the flowchart's
 *   GEMM node and its bias-and-dequantise node).
 *   acc[t,n] = sum_k xq[t,k] * wq[n,k]   (exact in int32)
 *   y[t,n]   = bf16_rn( float(acc) * (x_scale[t] * w_scale[n]) + bias[n] )
 * xq int8 [T, K]; x_scale fp32 [T]; wq int8 [N, K]; w_scale fp32 [N]; bias nullable bf16 [N];
 * y bf16 [T, N] out; acc_out nullable int32 [T, N] out (raw accumulators, for verification).
 * workspace / workspace_bytes: reserved; pass NULL / 0 (sq_w8a8_linear_workspace_size returns 0).
 * Requirements: T >= 0, N >= 8, N % 8 == 0, K >= 16, K % 16 == 0, K <= 131072; xq, wq, y 16-byte
 * aligned; acc_out 16-byte aligned. The GEMM runs on the tensor cores (tcgen05, TMEM accumulators,
 * TMA-fed shared-memory pipeline); its device-side waits are bounded and report SQ_ERR_TIMEOUT
 * through sq_device_status() instead of hanging. Output tiles are 128 tokens x 256 channels (64
 * channels when 256-wide tiles would leave SMs idle), or, for T <= 128, 128 channels x 16..128
 * tokens; every form computes the same bits.
 */
sq_status sq_w8a8_linear(const int8_t *xq, const float *x_scale, int64_t T, const int8_t *wq,
                         const float *w_scale, int64_t N, int64_t K, const void *bias, void *y,
                         int32_t *acc_out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Tile shape of sq_w8a8_linear for the calls that follow, in this process, on every device.
 *   enable = 0 (default): one SM per 128-token x 256-channel tile (tcgen05.mma.cta_group::1).
 *   enable = 1: pairs of SMs (a two-CTA cluster, tcgen05.mma.cta_group::2) per 256 x 256 tile when
 *               T >= 256; smaller T keeps the single-SM form.
 * Both forms compute the same bits. The pair form moves half the weight bytes per SM and needs fewer
 * SM cycles, but on B200 under its power limit it ran at lower clocks and was no faster, hence the
 * default. Any other value returns SQ_ERR_INVALID_ARG. Not synchronised with calls in flight on
 * other host threads.
 */
sq_status sq_set_gemm_cta_pair(int enable);

/*
 * FP8 E4M3 variant of the weight and activation quantisers and of the linear layer:
 *   [W8A8] "One layer, measured" (the same layer quantised to FP8 E4M3, weights per output channel,
 *   activations per token) and its explanation that FP8's exponent gives each value its own scale.
 * E4M3 is the OCP "FN" form (largest finite value 448). Codes are e4m3(v * fl32(448 / m)) rounded to
 * nearest (ties to even) with saturation at +-448, the sign kept on zeros; the scale is m / 448
 * (m = the row maximum); an all-zero row gives scale 0 and codes +0 (0x00). Codes are stored one byte
 * per value (uint8, the E4M3 bit pattern). Same arguments and requirements as the INT8 calls.
 */
sq_status sq_smooth_quantize_weight_fp8(const void *w, int64_t N, int64_t K, const float *s, uint8_t *wq,
                                        float *w_scale, void *stream);
sq_status sq_rmsnorm_smooth_quant_fp8(const void *x, int64_t T, int64_t K, const float *fold, float eps,
                                      int apply_norm, uint8_t *xq, float *x_scale, void *stream);

/*
 * FP8 linear: E4M3 x E4M3 products accumulated in binary32 on the tensor cores
 * (tcgen05.mma.kind::f8f6f4), then y[t,n] = bf16_rn(acc * (x_scale[t] * w_scale[n]) + bias[n]) in
 * binary32 as in sq_w8a8_linear. The products are exact; the order and precision of the tensor-core
 * accumulation are the hardware's, so acc differs from the exact sum by rounding only. acc_out
 * nullable fp32 [T, N] (the accumulators). Same arguments and requirements as sq_w8a8_linear (the
 * CTA-pair setting does not apply).
 */
sq_status sq_w8a8_linear_fp8(const uint8_t *xq, const float *x_scale, int64_t T, const uint8_t *wq,
                             const float *w_scale, int64_t N, int64_t K, const void *bias, void *y,
                             float *acc_out, void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace sq_w8a8_linear needs for these sizes: always 0 (no form of the GEMM uses one). */
size_t sq_w8a8_linear_workspace_size(int64_t T, int64_t N, int64_t K);

/*
 * Synchronises `stream`, then reports the device-side status word of the current device:
 * SQ_OK, SQ_ERR_TIMEOUT (a bounded wait in a kernel ran out; the kernel stopped its work and
 * returned, the context stays usable), SQ_ERR_BOUNDS (libsq_checked.so only: a device-side bounds
 * check failed and the access it guards was skipped) or SQ_ERR_CUDA (an asynchronous CUDA error).
 * The first error recorded is kept. The word is shared by every stream on the device; it is read and
 * cleared in one atomic exchange ordered on `stream` (a one-thread kernel), so an error that a kernel
 * on another stream records meanwhile is either reported by this call or kept for the next one.
 */
sq_status sq_device_status(void *stream);

/*
 * Sets the limit, in nanoseconds, of every bounded device-side wait launched afterwards on the
 * current device (default 2e9 = 2 s). Values below 1000 are raised to 1000.
 */
sq_status sq_set_wait_timeout_ns(uint64_t ns);

/*
 * Self-test of the timeout path: launches one small kernel whose thread waits, with the bounded
 * wait the GEMM uses, on a shared-memory barrier that nothing ever completes. The wait runs out
 * after the configured limit, the kernel records SQ_ERR_TIMEOUT in the status word and returns.
 * Used by the test suite to show that an expired wait ends in a status, not a hang.
 */
sq_status sq_selftest_wait_timeout(void *stream);

/*
 * Self-test of the device-side bounds checks of libsq_checked.so (the library built with
 * SQ_DEVICE_CHECKS): launches one small kernel whose store fails its check, so the kernel records
 * SQ_ERR_BOUNDS in the status word and skips the store (the store's target lies inside the kernel's
 * own array either way). Returns SQ_ERR_UNSUPPORTED, launching nothing, in the product libsq.so.
 * Neither the checks nor this call has a counterpart in SmoothQuant: they are a debugging aid.
 */
sq_status sq_selftest_bounds_check(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H */
