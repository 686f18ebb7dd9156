// sq_layernorm.cu -- LayerNorm-fed layers: the calibration abs-max of a LayerNorm's output and the
// fused LayerNorm + per-token INT8 quantiser with the smoothing factors folded into the LayerNorm.
//
// Page cited: [WOVS] "SmoothQuant: Weight-Only vs W8A8", "Integration with Transformers" (the
// division of the activations by S costs nothing at run time: S^-1 goes into the scale gamma and the
// bias beta of the LayerNorm in front of the projection, so its output is already smoothed, while
// the weight rows carry S).
//
// The pages do not write LayerNorm out; the standard per-token form is used, each step rounded as
// listed (fl32 = round to nearest binary32):
//   m   = fl32(sum_k x_k / K)               the sum in binary64
//   c_k = fl32(x_k - m)
//   ms  = fl32(sum_k c_k^2 / K)             each square exact in binary64, the sum in binary64
//   ir  = fl32(1 / fl32(sqrt(fl32(ms + eps))))
//   y_k = fl32(fl32(fl32(c_k * ir) * g_k) + b_k)
// Calibration takes g = gamma, b = beta; the online quantiser takes g = fold = fl32(gamma / s) (the
// fold sq_compute_scales writes) and b = fl32(beta / s) (sq_fold_layernorm_bias). The two binary64
// sums are taken in a tree order. The sum of x is exact unless a row's nonzero magnitudes span more
// than about 2^31; the sum of squares differs from any other order by at most a few binary64
// roundings, which can move ms only when the exact value lies that close to a binary32 rounding
// boundary.
//
// Design (B200). HBM-bound, one read of x. A CTA of 32..512 threads takes one row at a time
// (grid-stride over rows; the grid is SMs x resident CTAs); thread t holds the 16-byte vectors
// t, t + blockDim, ... of the row (VPT of them) as binary32 in registers, so the mean, the centred
// values, the variance and the outputs all come from one load. Block sums go through warp
// butterflies and one shared-memory slot per warp that every thread then adds in warp order, so all
// threads hold the same binary64 total. The squares are formed without a conversion instruction:
// one 64-bit integer multiply-add places |c|'s exponent and mantissa in the binary64 fields with
// exponent bias +485, which is exactly |c| * 2^-411 for every normal |c| >= 2^-100 (a zero becomes
// 2^-538, whose square rounds away inside the fused multiply-add), and the total is rescaled by
// 2^822.
// The calibration keeps per-column running maxima in registers over the rows its CTA takes and ends
// with one atomic max per column. Unlike the RMSNorm calibration it cannot apply gamma once per
// column at the end: the beta term makes each element's |y| depend on its own row.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_internal.h"

namespace {

constexpr int kLnMaxK = 16384;         // widest row held in registers (512 threads x 4 vectors)
constexpr int kLnMaxThreads = 512;
constexpr float kLnQmax = 127.0f;      // symmetric INT8 range [-127, 127]
constexpr uint64_t kSqBias64 = static_cast<uint64_t>(485u << 20) << 32;
constexpr unsigned kAll = 0xFFFFFFFFu;

struct LnArgs {
    const uint4 *x;     // row r starts at x + r * ldv (16-byte vectors of 8 bf16)
    int64_t rows;
    int64_t ldv;        // row stride in vectors
    int nvec;           // vectors per row (K / 8)
    int K;
    double inv_k;       // 1 / K when K is a power of two (exact), else 0
    const float *g;     // [K] gamma (calibration) or fold = gamma / s (online)
    const float *b;     // [K] beta or beta / s; NULL = no bias
    float eps;
    float *amax;        // calibration output [K] (running maximum)
    int8_t *q;          // online output [rows, K]
    float *scale;       // online output [rows]
};

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// |c| * 2^-411 in binary64 from the binary32 bits of |c| (see the file comment).
__device__ __forceinline__ double scaled_operand(float c) {
    double d;
    asm("{\n\t.reg .u64 t;\n\tmad.wide.u32 t, %1, 536870912, %2;\n\tmov.b64 %0, t;\n\t}"
        : "=d"(d) : "r"(__float_as_uint(c) & 0x7FFFFFFFu), "l"(kSqBias64));
    return d;
}

// Total over the CTA of one value per thread, identical in every thread: a warp butterfly (both
// partners of an exchange form the same sum), one slot per warp, the slots added in warp order.
__device__ __forceinline__ double block_sum(double v, double *slot) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kAll, v, o);
    if ((threadIdx.x & 31) == 0) slot[threadIdx.x >> 5] = v;
    __syncthreads();
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += slot[i];
    return t;
}

__device__ __forceinline__ float block_max(float v, float *slot) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kAll, v, o));
    if ((threadIdx.x & 31) == 0) slot[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = 0.0f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t = fmaxf(t, slot[i]);
    return t;
}

// Round half away from zero for |t| <= 127.00001: v = rz(t + copysign(1/2, t)) keeps the integer part
// of the exactly rounded sum (rounding toward zero cannot carry it past an integer); the conversion
// truncates it.
__device__ __forceinline__ uint32_t code_of(float t) {
    const float v = __fadd_rz(t, copysignf(0.5f, t));
    return static_cast<uint32_t>(__float2int_rz(v)) & 0xFFu;
}

// CALIB: per-column running abs-max of y (g = gamma, b = beta) into amax.
// Otherwise: y with g = fold, b = beta_fold, then one symmetric INT8 scale per row.
template <int VPT, bool CALIB>
__global__ void __launch_bounds__(kLnMaxThreads) k_layernorm(const LnArgs p)
{
    // one slot array per reduction of a row, so that no barrier is needed between rows
    __shared__ double s_sum[kLnMaxThreads / 32];
    __shared__ double s_ss[kLnMaxThreads / 32];
    __shared__ float s_max[kLnMaxThreads / 32];
    const int tid = threadIdx.x;
    const int bt = blockDim.x;
    float run[CALIB ? VPT * 8 : 1];
#pragma unroll
    for (int e = 0; e < (CALIB ? VPT * 8 : 1); ++e) run[e] = 0.0f;

    for (int64_t r = blockIdx.x; r < p.rows; r += gridDim.x) {
        const uint4 *row = p.x + r * p.ldv;
        float x[VPT * 8];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = i * bt + tid;
            const uint4 u = v < p.nvec ? ld_stream(row + v) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t w = k == 0 ? u.x : k == 1 ? u.y : k == 2 ? u.z : u.w;
                x[i * 8 + 2 * k] = __uint_as_float(w << 16);
                x[i * 8 + 2 * k + 1] = __uint_as_float(w & 0xFFFF0000u);
            }
        }
        // mean: absent vectors hold zeros and add nothing
        double s = 0.0;
#pragma unroll
        for (int e = 0; e < VPT * 8; ++e) s = __dadd_rn(s, static_cast<double>(x[e]));
        const double tot = block_sum(s, s_sum);
        const float m = __double2float_rn(p.inv_k != 0.0 ? __dmul_rn(tot, p.inv_k)
                                                         : __ddiv_rn(tot, static_cast<double>(p.K)));
        // centred values (kept in x) and the scaled sum of their squares
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const bool ok = i * bt + tid < p.nvec;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float c = __fsub_rn(x[i * 8 + k], m);
                x[i * 8 + k] = c;
                if (ok) {
                    const double d = scaled_operand(c);
                    ss = __fma_rn(d, d, ss);
                }
            }
        }
        const double var = __dmul_rn(block_sum(ss, s_ss), 0x1p822);
        const float ms = __double2float_rn(p.inv_k != 0.0 ? __dmul_rn(var, p.inv_k)
                                                          : __ddiv_rn(var, static_cast<double>(p.K)));
        const float ir = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, p.eps)));

        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = i * bt + tid;
            if (v < p.nvec) {
                const float4 g0 = __ldg(reinterpret_cast<const float4 *>(p.g) + 2 * v);
                const float4 g1 = __ldg(reinterpret_cast<const float4 *>(p.g) + 2 * v + 1);
                float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = b0;
                if (p.b != nullptr) {
                    b0 = __ldg(reinterpret_cast<const float4 *>(p.b) + 2 * v);
                    b1 = __ldg(reinterpret_cast<const float4 *>(p.b) + 2 * v + 1);
                }
                const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float y = __fadd_rn(__fmul_rn(__fmul_rn(x[i * 8 + k], ir), gg[k]), bb[k]);
                    x[i * 8 + k] = y;
                    if (CALIB) run[i * 8 + k] = fmaxf(run[i * 8 + k], fabsf(y));
                    else am = fmaxf(am, fabsf(y));
                }
            }
        }
        if (!CALIB) {
            const float mx = block_max(am, s_max);
            const float inv = mx > 0.0f ? __fdiv_rn(kLnQmax, mx) : 0.0f;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = i * bt + tid;
                if (v < p.nvec) {
                    uint32_t lo = 0, hi = 0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        lo |= code_of(__fmul_rn(x[i * 8 + k], inv)) << (8 * k);
                        hi |= code_of(__fmul_rn(x[i * 8 + 4 + k], inv)) << (8 * k);
                    }
                    *reinterpret_cast<uint2 *>(p.q + r * p.K + static_cast<int64_t>(v) * 8) = make_uint2(lo, hi);
                }
            }
            if (tid == 0) p.scale[r] = mx > 0.0f ? __fdiv_rn(mx, kLnQmax) : 0.0f;
        }
    }
    if (CALIB) {
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = i * bt + tid;
            if (v < p.nvec) {
#pragma unroll
                for (int k = 0; k < 8; ++k)   // non-negative binary32 order = unsigned integer order
                    if (run[i * 8 + k] > 0.0f)
                        atomicMax(reinterpret_cast<unsigned int *>(p.amax + static_cast<int64_t>(v) * 8 + k),
                                  __float_as_uint(run[i * 8 + k]));
            }
        }
    }
}

__global__ void k_fold_ln_bias(const float *__restrict__ beta, const float *__restrict__ s, int64_t K,
                               float *__restrict__ out)
{
    for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < K;
         k += static_cast<int64_t>(gridDim.x) * blockDim.x)
        out[k] = __fdiv_rn(beta[k], s[k]);
}

template <int VPT, bool CALIB>
sq_status launch_ln(const LnArgs &a, int dev, cudaStream_t st) {
    const int per = (a.nvec + VPT - 1) / VPT;
    const int threads = (per + 31) / 32 * 32;
    int occ = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_layernorm<VPT, CALIB>, threads, 0);
    if (e != cudaSuccess) return sq::cuda_status(e, "occupancy(layernorm)");
    const int64_t cap = static_cast<int64_t>(occ < 1 ? 1 : occ) * sq::sm_count(dev);
    const int64_t grid = a.rows < cap ? a.rows : cap;
    k_layernorm<VPT, CALIB><<<static_cast<unsigned>(grid), threads, 0, st>>>(a);
    return sq::cuda_status(cudaGetLastError(), CALIB ? "launch(layernorm_absmax)" : "launch(layernorm_quant)");
}

template <bool CALIB>
sq_status dispatch_ln(const LnArgs &a, int dev, cudaStream_t st) {
    if (a.nvec <= 256) return launch_ln<1, CALIB>(a, dev, st);
    if (a.nvec <= 512) return launch_ln<2, CALIB>(a, dev, st);
    return launch_ln<4, CALIB>(a, dev, st);
}

double exact_inv(int64_t K) { return (K & (K - 1)) == 0 ? 1.0 / static_cast<double>(K) : 0.0; }

}  // namespace

extern "C" {

sq_status sq_calibrate_absmax_layernorm(const void *a, int64_t rows, int64_t cols, int64_t ld, const float *gamma,
                                        const float *beta, float eps, float *amax, int accumulate, void *stream)
{
    using sq::fail;
    if (!amax || !gamma) return fail(SQ_ERR_INVALID_ARG, "sq_calibrate_absmax_layernorm: amax and gamma are required");
    if (rows < 0 || cols < 8 || ld < cols)
        return fail(SQ_ERR_INVALID_ARG, "sq_calibrate_absmax_layernorm: need rows >= 0, cols >= 8, ld >= cols (rows=%lld cols=%lld ld=%lld)",
                    (long long)rows, (long long)cols, (long long)ld);
    if (rows > 0 && !a) return fail(SQ_ERR_INVALID_ARG, "sq_calibrate_absmax_layernorm: a is NULL");
    if (cols % 8 != 0 || ld % 8 != 0)
        return fail(SQ_ERR_MISALIGNED, "sq_calibrate_absmax_layernorm: cols and ld must be multiples of 8");
    if ((a && !sq::aligned(a, 16)) || !sq::aligned(gamma, 16) || (beta && !sq::aligned(beta, 16)) || !sq::aligned(amax, 4))
        return fail(SQ_ERR_MISALIGNED, "sq_calibrate_absmax_layernorm: a, gamma and beta 16-byte, amax 4-byte alignment required");
    if (cols > kLnMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_calibrate_absmax_layernorm: cols must be <= %d", kLnMaxK);
    int dev = 0;
    SQ_TRY_ARCH(dev);
    cudaStream_t st = sq::as_stream(stream);
    if (!accumulate) {
        const sq_status s0 = sq::cuda_status(cudaMemsetAsync(amax, 0, static_cast<size_t>(cols) * 4, st), "memset(amax)");
        if (s0 != SQ_OK) return s0;
    }
    if (rows == 0) return SQ_OK;
    LnArgs la = {};
    la.x = static_cast<const uint4 *>(a);
    la.rows = rows;
    la.ldv = ld / 8;
    la.nvec = static_cast<int>(cols / 8);
    la.K = static_cast<int>(cols);
    la.inv_k = exact_inv(cols);
    la.g = gamma;
    la.b = beta;
    la.eps = eps;
    la.amax = amax;
    return dispatch_ln<true>(la, dev, st);
}

sq_status sq_fold_layernorm_bias(const float *beta, const float *s, int64_t K, float *beta_fold, void *stream)
{
    using sq::fail;
    if (K < 1 || !beta || !s || !beta_fold) return fail(SQ_ERR_INVALID_ARG, "sq_fold_layernorm_bias: need K >= 1 and all arrays");
    if (!sq::aligned(beta, 4) || !sq::aligned(s, 4) || !sq::aligned(beta_fold, 4))
        return fail(SQ_ERR_MISALIGNED, "sq_fold_layernorm_bias: fp32 arrays must be 4-byte aligned");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    k_fold_ln_bias<<<static_cast<unsigned>((K + 255) / 256 < 1024 ? (K + 255) / 256 : 1024), 256, 0, sq::as_stream(stream)>>>(
        beta, s, K, beta_fold);
    return sq::cuda_status(cudaGetLastError(), "launch(fold_layernorm_bias)");
}

sq_status sq_layernorm_smooth_quant(const void *x, int64_t T, int64_t K, const float *fold, const float *beta_fold,
                                    float eps, int8_t *xq, float *x_scale, void *stream)
{
    using sq::fail;
    if (T < 0 || K < 8) return fail(SQ_ERR_INVALID_ARG, "sq_layernorm_smooth_quant: need T >= 0 and K >= 8");
    if (!fold) return fail(SQ_ERR_INVALID_ARG, "sq_layernorm_smooth_quant: fold is required");
    if (T > 0 && (!x || !xq || !x_scale)) return fail(SQ_ERR_INVALID_ARG, "sq_layernorm_smooth_quant: x, xq and x_scale are required");
    if (K % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_layernorm_smooth_quant: K must be a multiple of 8");
    if (K > kLnMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_layernorm_smooth_quant: K must be <= %d", kLnMaxK);
    if ((x && !sq::aligned(x, 16)) || (xq && !sq::aligned(xq, 8)) || !sq::aligned(fold, 16) ||
        (beta_fold && !sq::aligned(beta_fold, 16)) || (x_scale && !sq::aligned(x_scale, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_layernorm_smooth_quant: x, fold and beta_fold 16-byte, xq 8-byte, x_scale 4-byte alignment required");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    if (T == 0) return SQ_OK;
    LnArgs la = {};
    la.x = static_cast<const uint4 *>(x);
    la.rows = T;
    la.ldv = K / 8;
    la.nvec = static_cast<int>(K / 8);
    la.K = static_cast<int>(K);
    la.inv_k = exact_inv(K);
    la.g = fold;
    la.b = beta_fold;
    la.eps = eps;
    la.q = xq;
    la.scale = x_scale;
    return dispatch_ln<false>(la, dev, sq::as_stream(stream));
}

}  // extern "C"
