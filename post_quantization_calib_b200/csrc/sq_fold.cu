// sq_fold.cu -- fold of the smoothing factor 1/s into the previous linear layer, the alternative to
// folding it into a norm's weight.
//
// Pages cited: [MIGRATE] "06 -- SmoothQuant: Migrating Difficulty from Activations to Weights",
// section 7 (the division X / s is absorbed by multiplying the previous layer's output-column-j
// weights by 1 / s_j; zero run-time cost); [WOVS] "SmoothQuant: Weight-Only vs W8A8", "Integration
// with Transformers" (S^-1 folded into a LayerNorm's gamma and beta: beta / s here, gamma / s is
// the fold the smoothing-factor kernel writes).
//
// The previous layer's weight is bf16 [K, Kp] (its output channel j feeds input channel j of the
// smoothed layer): row j is multiplied by fold[j] = fl32(1 / s_j) and rounded to bf16 (nearest,
// ties to even), and so is its bias. For an INT8 previous layer the factor goes into its binary32
// per-output-channel dequantisation scale instead. Both are HBM-bound elementwise passes: a CTA
// takes whole rows, 16-byte vectors (8 bf16) per thread, one binary32 multiply per element.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_device.cuh"
#include "sq_internal.h"

using namespace sqdev;

namespace {

__device__ __forceinline__ uint32_t scale_pair(uint32_t w, float f) {
    const float lo = __fmul_rn(__uint_as_float(w << 16), f);
    const float hi = __fmul_rn(__uint_as_float(w & 0xFFFF0000u), f);
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// w_out / b_out may alias w / b (each element is read, then written, by the same thread; plain loads).
__global__ void __launch_bounds__(256) k_fold_rows(const uint4 *w, const uint16_t *b, int64_t K, int64_t vrow,
                                                   const float *__restrict__ fold, uint4 *w_out, uint16_t *b_out)
{
    pdl_wait();
    pdl_trigger();
    for (int64_t j = blockIdx.x; j < K; j += gridDim.x) {
        const float f = __ldg(fold + j);
        const uint4 *src = w + j * vrow;
        uint4 *dst = w_out + j * vrow;
        for (int64_t v = threadIdx.x; v < vrow; v += blockDim.x) {
            const uint4 q = src[v];
            dst[v] = make_uint4(scale_pair(q.x, f), scale_pair(q.y, f), scale_pair(q.z, f), scale_pair(q.w, f));
        }
        if (b != nullptr && threadIdx.x == 0) {
            const float r = __fmul_rn(__uint_as_float(static_cast<uint32_t>(b[j]) << 16), f);
            const __nv_bfloat16 h = __float2bfloat16_rn(r);
            b_out[j] = *reinterpret_cast<const uint16_t *>(&h);
        }
    }
}

__global__ void k_fold_w_scale(const float *ws, int64_t K, const float *__restrict__ fold, float *out)
{
    pdl_wait();
    pdl_trigger();
    for (int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < K;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[j] = __fmul_rn(ws[j], fold[j]);
}

// beta_fold[k] = fl32(beta[k] / s[k]): the LayerNorm bias with S^-1 folded in.
__global__ void k_fold_ln_bias(const float *__restrict__ beta, const float *__restrict__ s, int64_t K,
                               float *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < K;
         k += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[k] = __fdiv_rn(beta[k], s[k]);
}

}  // namespace

extern "C" {

sq_status sq_fold_into_prev_linear(const void *w, const void *b, int64_t K, int64_t Kp, const float *fold,
                                   void *w_out, void *b_out, void *stream)
{
    using sq::fail;
    if (K < 0 || Kp < 8) return fail(SQ_ERR_INVALID_ARG, "sq_fold_into_prev_linear: need K >= 0 and Kp >= 8");
    if (K > 0 && (!w || !fold || !w_out)) return fail(SQ_ERR_INVALID_ARG, "sq_fold_into_prev_linear: w, fold and w_out are required");
    if (b && !b_out) return fail(SQ_ERR_INVALID_ARG, "sq_fold_into_prev_linear: b_out is required with a bias");
    if (Kp % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_fold_into_prev_linear: Kp must be a multiple of 8");
    if ((w && !sq::aligned(w, 16)) || (w_out && !sq::aligned(w_out, 16)) || (fold && !sq::aligned(fold, 4)) ||
        (b && !sq::aligned(b, 2)) || (b_out && !sq::aligned(b_out, 2)))
        return fail(SQ_ERR_MISALIGNED, "sq_fold_into_prev_linear: w and w_out 16-byte, fold 4-byte, biases 2-byte alignment required");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    if (K == 0) return SQ_OK;
    const int64_t grid = K < 8L * sq::sm_count(dev) ? K : 8L * sq::sm_count(dev);
    return sq::cuda_status(sq::launch_pdl(k_fold_rows, dim3(static_cast<unsigned>(grid)), dim3(256), 0, sq::as_stream(stream),
                                          nullptr, static_cast<const uint4 *>(w), static_cast<const uint16_t *>(b), K, Kp / 8,
                                          fold, static_cast<uint4 *>(w_out), static_cast<uint16_t *>(b_out)),
                           "launch(fold_rows)");
}

sq_status sq_fold_into_w_scale(const float *w_scale, int64_t K, const float *fold, float *w_scale_out, void *stream)
{
    using sq::fail;
    if (K < 1 || !w_scale || !fold || !w_scale_out) return fail(SQ_ERR_INVALID_ARG, "sq_fold_into_w_scale: need K >= 1 and all arrays");
    if (!sq::aligned(w_scale, 4) || !sq::aligned(fold, 4) || !sq::aligned(w_scale_out, 4))
        return fail(SQ_ERR_MISALIGNED, "sq_fold_into_w_scale: fp32 arrays must be 4-byte aligned");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    return sq::cuda_status(sq::launch_pdl(k_fold_w_scale, dim3(static_cast<unsigned>((K + 255) / 256 < 1024 ? (K + 255) / 256 : 1024)),
                                          dim3(256), 0, sq::as_stream(stream), nullptr, w_scale, K, fold, w_scale_out),
                           "launch(fold_w_scale)");
}

sq_status sq_fold_layernorm_bias(const float *beta, const float *s, int64_t K, float *beta_fold, void *stream)
{
    using sq::fail;
    if (K < 1 || !beta || !s || !beta_fold) return fail(SQ_ERR_INVALID_ARG, "sq_fold_layernorm_bias: need K >= 1 and all arrays");
    if (!sq::aligned(beta, 4) || !sq::aligned(s, 4) || !sq::aligned(beta_fold, 4))
        return fail(SQ_ERR_MISALIGNED, "sq_fold_layernorm_bias: fp32 arrays must be 4-byte aligned");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    return sq::cuda_status(sq::launch_pdl(k_fold_ln_bias, dim3(static_cast<unsigned>((K + 255) / 256 < 1024 ? (K + 255) / 256 : 1024)),
                                          dim3(256), 0, sq::as_stream(stream), nullptr, beta, s, K, beta_fold),
                           "launch(fold_layernorm_bias)");
}

}  // extern "C"
