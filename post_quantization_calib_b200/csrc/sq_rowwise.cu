// sq_rowwise.cu -- the HBM-bound steps of the smoothed W8A8 linear on sm_100a:
//   per-input-channel abs-max (calibration activations and weights), smoothing factors with the
//   fold into the norm weight, and the row quantisers (weights per output channel, activations per
//   token with the RMSNorm fused in).
//
// Pages cited (title, then section / equation / figure):
//   [MIGRATE] "06 -- SmoothQuant: Migrating Difficulty from Activations to Weights"
//   [TAMING]  "Taming the Outliers: A Deep Dive into SmoothQuant for LLM Quantization"
//   [W8A8]    "SmoothQuant and W8A8: Quantizing Activations Too"
//
// Design (B200): every kernel streams its input once with 16-byte loads, keeps a whole row of a
// CTA's work in registers, reduces with warp shuffles plus one shared-memory step, and writes
// coalesced outputs. The column abs-max reduces across CTAs first inside an 8-CTA thread-block
// cluster through distributed shared memory, so only one global atomic max per column per cluster
// reaches L2. Arithmetic is binary32 with explicit round-to-nearest intrinsics (nothing is
// contracted into fused multiply-adds); the RMSNorm sum of squares is binary64.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_internal.h"

namespace cg = cooperative_groups;

namespace {

constexpr float kFloor = 1e-5f;   // floor of abs-maxima and of s ([TAMING] listing clamps s at 1e-5)
constexpr float kQmax = 127.0f;   // symmetric INT8 range [-127, 127]
constexpr int kCluster = 8;       // CTAs per cluster in the column abs-max
constexpr int kMaxK = 16384;      // widest row held on chip by the row kernels

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ void load8f(const float *__restrict__ p, float (&f)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Round half away from zero. t - trunc(t) is exact in binary32, so the comparison decides ties
// exactly.
__device__ __forceinline__ float round_half_away(float t) {
    const float r = truncf(t);
    return fabsf(__fsub_rn(t, r)) >= 0.5f ? __fadd_rn(r, copysignf(1.0f, t)) : r;
}

// INT8 code of one smoothed value: clamp(round_half_away(y * inv_delta), -127, 127).
__device__ __forceinline__ uint32_t code8(float y, float inv_delta) {
    float r = round_half_away(__fmul_rn(y, inv_delta));
    r = fminf(fmaxf(r, -kQmax), kQmax);
    return static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu;
}

__device__ __forceinline__ uint2 pack8(const float (&y)[8], float inv) {
    uint2 o;
    o.x = code8(y[0], inv) | (code8(y[1], inv) << 8) | (code8(y[2], inv) << 16) | (code8(y[3], inv) << 24);
    o.y = code8(y[4], inv) | (code8(y[5], inv) << 8) | (code8(y[6], inv) << 16) | (code8(y[7], inv) << 24);
    return o;
}

// 1 / sqrt(ss / K + eps) with each step rounded as the RMSNorm definition orders it.
__device__ __forceinline__ float inv_rms(double ss, int K, float eps) {
    const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
    const float r = __fsqrt_rn(__fadd_rn(ms, eps));
    return __fdiv_rn(1.0f, r);
}

__device__ __forceinline__ double sumsq8(const float (&f)[8]) {
    double s = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) s += static_cast<double>(f[e]) * static_cast<double>(f[e]);
    return s;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// ---------------------------------------------------------------------------------------------
// Column abs-max, [MIGRATE] section 3 / [TAMING] "System Architecture" (max|X| and max|W| per
// channel). Each CTA owns a contiguous block of rows and a slab of THREADS*VPT*8 columns, holds the
// running maxima of its columns in registers, and (with NORM) normalises each row by its inverse
// RMS and the norm weight first. Two rows are in flight per iteration.
template <int THREADS, int VPT, bool NORM>
__global__ void __launch_bounds__(THREADS)
k_absmax(const uint4 *__restrict__ a, int64_t rows, int nvec, int64_t ldv,
         const float *__restrict__ gamma, float eps, int cols, int64_t rows_per_cta,
         float *__restrict__ amax)
{
    constexpr int WARPS = THREADS / 32;
    extern __shared__ float s_red[];               // [THREADS * VPT * 8] this CTA's maxima
    __shared__ double s_ss[2][WARPS][2];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slab0 = blockIdx.y * THREADS * VPT;   // first 8-column vector of the slab
    const int slab_vecs = min(THREADS * VPT, nvec - slab0);
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
    const int64_t r1 = min(rows, r0 + rows_per_cta);

    float g[VPT][8];
    float mx[VPT][8];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = tid + i * THREADS;
#pragma unroll
        for (int e = 0; e < 8; ++e) { mx[i][e] = 0.0f; g[i][e] = 1.0f; }
        if (NORM && vi < slab_vecs) load8f(gamma + (slab0 + vi) * 8, g[i]);
    }

    int it = 0;
    for (int64_t r = r0; r < r1; r += 2, ++it) {
        const bool two = (r + 1) < r1;
        const uint4 *p0 = a + r * ldv + slab0;
        const uint4 *p1 = p0 + ldv;
        uint4 v0[VPT], v1[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int vi = tid + i * THREADS;
            const bool ok = vi < slab_vecs;
            v0[i] = ok ? __ldcs(p0 + vi) : make_uint4(0u, 0u, 0u, 0u);
            v1[i] = (ok && two) ? __ldcs(p1 + vi) : make_uint4(0u, 0u, 0u, 0u);
        }
        float ir0 = 1.0f, ir1 = 1.0f;
        if (NORM) {
            double ss0 = 0.0, ss1 = 0.0;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float f[8];
                unpack8(v0[i], f); ss0 += sumsq8(f);
                unpack8(v1[i], f); ss1 += sumsq8(f);
            }
            ss0 = warp_sum(ss0);
            ss1 = warp_sum(ss1);
            if (lane == 0) { s_ss[it & 1][warp][0] = ss0; s_ss[it & 1][warp][1] = ss1; }
            __syncthreads();
            double t0 = 0.0, t1 = 0.0;
#pragma unroll
            for (int w = 0; w < WARPS; ++w) { t0 += s_ss[it & 1][w][0]; t1 += s_ss[it & 1][w][1]; }
            ir0 = inv_rms(t0, cols, eps);
            ir1 = inv_rms(t1, cols, eps);
        }
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            float f[8];
            unpack8(v0[i], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float y = NORM ? __fmul_rn(__fmul_rn(f[e], ir0), g[i][e]) : f[e];
                mx[i][e] = fmaxf(mx[i][e], fabsf(y));
            }
            if (two) {
                unpack8(v1[i], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float y = NORM ? __fmul_rn(__fmul_rn(f[e], ir1), g[i][e]) : f[e];
                    mx[i][e] = fmaxf(mx[i][e], fabsf(y));
                }
            }
        }
    }

    // Cluster-wide reduction through distributed shared memory, then one atomic max per column.
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = tid + i * THREADS;
        if (vi < slab_vecs) {
#pragma unroll
            for (int e = 0; e < 8; ++e) s_red[vi * 8 + e] = mx[i][e];
        }
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int slab_cols = slab_vecs * 8;
    const int share = (slab_cols + kCluster - 1) / kCluster;
    const int c0 = static_cast<int>(cluster.block_rank()) * share;
    const int c1 = min(slab_cols, c0 + share);
    for (int j = c0 + tid; j < c1; j += THREADS) {
        float m = 0.0f;
#pragma unroll
        for (int q = 0; q < kCluster; ++q) m = fmaxf(m, cluster.map_shared_rank(s_red, q)[j]);
        // abs-maxima are non-negative, where IEEE order equals unsigned integer order
        if (m > 0.0f) atomicMax(reinterpret_cast<unsigned int *>(amax + slab0 * 8 + j), __float_as_uint(m));
    }
    cluster.sync();
}

__global__ void k_fill_zero(float *__restrict__ p, int64_t n) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = 0.0f;
}

// ---------------------------------------------------------------------------------------------
// Smoothing factors and fold, [MIGRATE] section 3 and [W8A8] "The trick: move the range into the
// weights": s = max|X|^alpha / max|W|^(1-alpha) in binary64, rounded once, floored at 1e-5;
// fold = gamma / s (or 1 / s).
__global__ void k_scales(const float *__restrict__ ax, const float *__restrict__ aw, int64_t K,
                         double ea, double eb, const float *__restrict__ gamma,
                         float *__restrict__ s, float *__restrict__ fold)
{
    const int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (j >= K) return;
    const double a = static_cast<double>(fmaxf(ax[j], kFloor));
    const double b = static_cast<double>(fmaxf(aw[j], kFloor));
    float sj = __double2float_rn(__ddiv_rn(pow(a, ea), pow(b, eb)));
    sj = fmaxf(sj, kFloor);
    s[j] = sj;
    if (fold) fold[j] = __fdiv_rn(gamma ? gamma[j] : 1.0f, sj);
}

// ---------------------------------------------------------------------------------------------
// Row quantiser, one CTA per row. Without NORM it quantises y = x * c (weights: c = s, the
// smoothed weight diag(s) W, [MIGRATE] sections 2 and 7; activations fed directly: c = 1/s).
// With NORM it fuses the RMSNorm whose weight carries the folded 1/s ([W8A8] "The trick..."),
// y = (x * inv_rms) * c, and quantises per token ([MIGRATE] section 7; [W8A8] "The full model,
// served"). The row stays in registers between the reductions and the quantisation.
template <int THREADS, int VPT, bool NORM>
__global__ void __launch_bounds__(THREADS)
k_rowquant(const uint4 *__restrict__ x, int nvec, const float *__restrict__ c, float eps,
           int K, int8_t *__restrict__ q, float *__restrict__ scale)
{
    constexpr int WARPS = THREADS / 32;
    __shared__ double s_ss[WARPS];
    __shared__ float s_mx[WARPS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.x;
    const uint4 *xr = x + row * static_cast<int64_t>(nvec);

    uint4 v[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = tid + i * THREADS;
        v[i] = vi < nvec ? __ldcs(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
    }

    float ir = 1.0f;
    if (NORM) {
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            float f[8];
            unpack8(v[i], f);
            ss += sumsq8(f);
        }
        ss = warp_sum(ss);
        if (lane == 0) s_ss[warp] = ss;
        __syncthreads();
        double t = 0.0;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) t += s_ss[w];
        ir = inv_rms(t, K, eps);
    }

    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = tid + i * THREADS;
        if (vi < nvec) {
            float f[8], cc[8];
            unpack8(v[i], f);
            if (c) load8f(c + vi * 8, cc);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float y = NORM ? __fmul_rn(__fmul_rn(f[e], ir), cc[e]) : (c ? __fmul_rn(f[e], cc[e]) : f[e]);
                m = fmaxf(m, fabsf(y));
            }
        }
    }
    m = warp_max(m);
    if (lane == 0) s_mx[warp] = m;
    __syncthreads();
    m = 0.0f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) m = fmaxf(m, s_mx[w]);

    const float delta = m > 0.0f ? __fdiv_rn(m, kQmax) : 0.0f;
    const float inv = m > 0.0f ? __fdiv_rn(kQmax, m) : 0.0f;
    uint2 *qr = reinterpret_cast<uint2 *>(q + row * static_cast<int64_t>(K));
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = tid + i * THREADS;
        if (vi < nvec) {
            float f[8], cc[8], y[8];
            unpack8(v[i], f);
            if (c) load8f(c + vi * 8, cc);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                y[e] = NORM ? __fmul_rn(__fmul_rn(f[e], ir), cc[e]) : (c ? __fmul_rn(f[e], cc[e]) : f[e]);
            qr[vi] = pack8(y, inv);
        }
    }
    if (tid == 0) scale[row] = delta;
}

// ---------------------------------------------------------------------------------------------
// Launch helpers.

struct RowCfg {
    int threads;
    int vpt;
};

// Smallest (threads, vectors-per-thread) pair covering nvec 8-element vectors.
RowCfg row_cfg(int64_t nvec) {
    if (nvec <= 128) return {128, 1};
    if (nvec <= 256) return {256, 1};
    if (nvec <= 512) return {256, 2};
    if (nvec <= 1024) return {256, 4};
    return {256, 8};
}

template <int THREADS, int VPT, bool NORM>
sq_status launch_absmax_t(const void *a, int64_t rows, int64_t cols, int64_t ld, const float *gamma,
                          float eps, float *amax, int dev, cudaStream_t st)
{
    auto kern = k_absmax<THREADS, VPT, NORM>;
    const int nvec = static_cast<int>(cols / 8);
    const int slab = THREADS * VPT;
    const int slabs = (nvec + slab - 1) / slab;
    const size_t smem = static_cast<size_t>(slab) * 8 * sizeof(float);
    static int configured[64];
    static int per_sm[64];
    if (!configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaFuncSetAttribute(absmax)");
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, THREADS, smem);
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor(absmax)");
        per_sm[dev] = nb > 0 ? nb : 1;
        configured[dev] = 1;
    }
    const int64_t target = static_cast<int64_t>(sq::sm_count(dev)) * per_sm[dev] / slabs;
    int64_t gx = (rows + 15) / 16;                               // at least ~16 rows per CTA
    if (gx > target) gx = target;
    gx = ((gx + kCluster - 1) / kCluster) * kCluster;
    if (gx < kCluster) gx = kCluster;
    int64_t rpc = (rows + gx - 1) / gx;
    rpc += rpc & 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(slabs), 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const uint4 *>(a), rows, nvec,
                                       static_cast<int64_t>(ld / 8), gamma, eps, static_cast<int>(cols), rpc, amax);
    return sq::cuda_status(e, "launch(absmax)");
}

template <int THREADS, int VPT, bool NORM>
sq_status launch_rowquant_t(const void *x, int64_t rows, int64_t K, const float *c, float eps,
                            int8_t *q, float *scale, cudaStream_t st)
{
    if (rows == 0) return SQ_OK;
    k_rowquant<THREADS, VPT, NORM><<<static_cast<unsigned>(rows), THREADS, 0, st>>>(
        reinterpret_cast<const uint4 *>(x), static_cast<int>(K / 8), c, eps, static_cast<int>(K), q, scale);
    return sq::cuda_status(cudaGetLastError(), "launch(rowquant)");
}

template <bool NORM>
sq_status dispatch_rowquant(const void *x, int64_t rows, int64_t K, const float *c, float eps,
                            int8_t *q, float *scale, cudaStream_t st)
{
    const RowCfg rc = row_cfg(K / 8);
    switch (rc.threads * 16 + rc.vpt) {
        case 128 * 16 + 1: return launch_rowquant_t<128, 1, NORM>(x, rows, K, c, eps, q, scale, st);
        case 256 * 16 + 1: return launch_rowquant_t<256, 1, NORM>(x, rows, K, c, eps, q, scale, st);
        case 256 * 16 + 2: return launch_rowquant_t<256, 2, NORM>(x, rows, K, c, eps, q, scale, st);
        case 256 * 16 + 4: return launch_rowquant_t<256, 4, NORM>(x, rows, K, c, eps, q, scale, st);
        default: return launch_rowquant_t<256, 8, NORM>(x, rows, K, c, eps, q, scale, st);
    }
}

template <bool NORM>
sq_status dispatch_absmax(const void *a, int64_t rows, int64_t cols, int64_t ld, const float *gamma,
                          float eps, float *amax, int dev, cudaStream_t st)
{
    const RowCfg rc = row_cfg(cols / 8);
    switch (rc.threads * 16 + rc.vpt) {
        case 128 * 16 + 1: return launch_absmax_t<128, 1, NORM>(a, rows, cols, ld, gamma, eps, amax, dev, st);
        case 256 * 16 + 1: return launch_absmax_t<256, 1, NORM>(a, rows, cols, ld, gamma, eps, amax, dev, st);
        case 256 * 16 + 2: return launch_absmax_t<256, 2, NORM>(a, rows, cols, ld, gamma, eps, amax, dev, st);
        case 256 * 16 + 4: return launch_absmax_t<256, 4, NORM>(a, rows, cols, ld, gamma, eps, amax, dev, st);
        default: return launch_absmax_t<256, 8, NORM>(a, rows, cols, ld, gamma, eps, amax, dev, st);
    }
}

}  // namespace

extern "C" {

sq_status sq_calibrate_absmax(const void *a, int64_t rows, int64_t cols, int64_t ld,
                              const float *norm_gamma, float eps, float *amax, int accumulate,
                              void *stream)
{
    using sq::fail;
    if (!amax) return fail(SQ_ERR_INVALID_ARG, "sq_calibrate_absmax: amax is NULL");
    if (rows < 0 || cols < 8 || ld < cols)
        return fail(SQ_ERR_INVALID_ARG, "sq_calibrate_absmax: need rows >= 0, cols >= 8, ld >= cols (rows=%lld cols=%lld ld=%lld)",
                    (long long)rows, (long long)cols, (long long)ld);
    if (rows > 0 && !a) return fail(SQ_ERR_INVALID_ARG, "sq_calibrate_absmax: a is NULL");
    if (cols % 8 != 0 || ld % 8 != 0)
        return fail(SQ_ERR_MISALIGNED, "sq_calibrate_absmax: cols and ld must be multiples of 8");
    if ((a && !sq::aligned(a, 16)) || !sq::aligned(amax, 4) || (norm_gamma && !sq::aligned(norm_gamma, 16)))
        return fail(SQ_ERR_MISALIGNED, "sq_calibrate_absmax: a and norm_gamma must be 16-byte aligned, amax 4-byte aligned");
    if (norm_gamma && cols > kMaxK)
        return fail(SQ_ERR_UNSUPPORTED, "sq_calibrate_absmax: with norm_gamma, cols must be <= %d", kMaxK);
    if (cols / 8 > (int64_t)1 << 30) return fail(SQ_ERR_UNSUPPORTED, "sq_calibrate_absmax: cols too large");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    cudaStream_t st = sq::as_stream(stream);
    if (!accumulate) {
        k_fill_zero<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(amax, cols);
        sq_status s0 = sq::cuda_status(cudaGetLastError(), "launch(fill)");
        if (s0 != SQ_OK) return s0;
    }
    if (rows == 0) return SQ_OK;
    return norm_gamma ? dispatch_absmax<true>(a, rows, cols, ld, norm_gamma, eps, amax, dev, st)
                      : dispatch_absmax<false>(a, rows, cols, ld, nullptr, eps, amax, dev, st);
}

sq_status sq_compute_scales(const float *amax_x, const float *amax_w, int64_t K, float alpha,
                            const float *gamma, float *s, float *fold, void *stream)
{
    using sq::fail;
    if (!amax_x || !amax_w || !s) return fail(SQ_ERR_INVALID_ARG, "sq_compute_scales: amax_x, amax_w and s are required");
    if (K < 1) return fail(SQ_ERR_INVALID_ARG, "sq_compute_scales: K must be >= 1");
    if (!(alpha >= 0.0f && alpha <= 1.0f)) return fail(SQ_ERR_INVALID_ARG, "sq_compute_scales: alpha must be in [0, 1]");
    if (!sq::aligned(amax_x, 4) || !sq::aligned(amax_w, 4) || !sq::aligned(s, 4) ||
        (gamma && !sq::aligned(gamma, 4)) || (fold && !sq::aligned(fold, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_compute_scales: fp32 arrays must be 4-byte aligned");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    const double ea = static_cast<double>(alpha);
    const double eb = 1.0 - static_cast<double>(alpha);
    k_scales<<<static_cast<unsigned>((K + 255) / 256), 256, 0, sq::as_stream(stream)>>>(amax_x, amax_w, K, ea, eb, gamma, s, fold);
    return sq::cuda_status(cudaGetLastError(), "launch(scales)");
}

sq_status sq_smooth_quantize_weight(const void *w, int64_t N, int64_t K, const float *s,
                                    int8_t *wq, float *w_scale, void *stream)
{
    using sq::fail;
    if (N < 0 || K < 8) return fail(SQ_ERR_INVALID_ARG, "sq_smooth_quantize_weight: need N >= 0 and K >= 8");
    if (N > 0 && (!w || !wq || !w_scale)) return fail(SQ_ERR_INVALID_ARG, "sq_smooth_quantize_weight: w, wq and w_scale are required");
    if (K % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_smooth_quantize_weight: K must be a multiple of 8");
    if (K > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_smooth_quantize_weight: K must be <= %d", kMaxK);
    if ((w && !sq::aligned(w, 16)) || (wq && !sq::aligned(wq, 8)) || (s && !sq::aligned(s, 16)) ||
        (w_scale && !sq::aligned(w_scale, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_smooth_quantize_weight: w and s 16-byte, wq 8-byte, w_scale 4-byte alignment required");
    if (N > 0x7FFFFFFF) return fail(SQ_ERR_UNSUPPORTED, "sq_smooth_quantize_weight: N too large");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    return dispatch_rowquant<false>(w, N, K, s, 0.0f, wq, w_scale, sq::as_stream(stream));
}

sq_status sq_rmsnorm_smooth_quant(const void *x, int64_t T, int64_t K, const float *fold, float eps,
                                  int apply_norm, int8_t *xq, float *x_scale, void *stream)
{
    using sq::fail;
    if (T < 0 || K < 8) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant: need T >= 0 and K >= 8");
    if (!fold) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant: fold is required");
    if (T > 0 && (!x || !xq || !x_scale)) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant: x, xq and x_scale are required");
    if (K % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_rmsnorm_smooth_quant: K must be a multiple of 8");
    if (K > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_rmsnorm_smooth_quant: K must be <= %d", kMaxK);
    if ((x && !sq::aligned(x, 16)) || (xq && !sq::aligned(xq, 8)) || !sq::aligned(fold, 16) ||
        (x_scale && !sq::aligned(x_scale, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_rmsnorm_smooth_quant: x and fold 16-byte, xq 8-byte, x_scale 4-byte alignment required");
    if (T > 0x7FFFFFFF) return fail(SQ_ERR_UNSUPPORTED, "sq_rmsnorm_smooth_quant: T too large");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    cudaStream_t st = sq::as_stream(stream);
    return apply_norm ? dispatch_rowquant<true>(x, T, K, fold, eps, xq, x_scale, st)
                      : dispatch_rowquant<false>(x, T, K, fold, eps, xq, x_scale, st);
}

}  // extern "C"
