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
// Design (B200). One kernel template serves the abs-max (MODE_ABSMAX) and the quantisers
// (MODE_QUANT). A CTA of 8 warps is split into row groups of 1, 2, 4 or 8 warps (enough lanes to hold
// one row of up to 16384 bf16 in registers, 64 per lane). Each group streams its own rows through a
// 2-6 slot shared-memory ring filled by TMA bulk copies (one 1-D copy per row, completion on an
// mbarrier), so several rows per group are in flight while the group computes on the current one.
// Per row, the group's lanes hold the row in registers; reductions are warp shuffles plus, for
// groups of several warps, one named barrier that also releases the ring slot.
//
// Instruction budget. These kernels must retire about 8-12 bf16 elements per SM cycle to keep up
// with HBM, so each element gets only a dozen instructions and none on the quarter-rate conversion
// pipe:
//   * the RMSNorm sum of squares is binary64, but each operand is built with integer operations:
//     the bf16 exponent and mantissa are placed in the binary64 fields with exponent bias +485, which
//     is exactly x * 2^-411 for every normal |x| >= 2^-100 (and a zero becomes 2^-538, whose square
//     2^-1076 rounds away inside the fused multiply-add); the binary64 accumulator is rescaled by
//     2^822 at the end. Squares of |x| < 2^-100 (and of subnormal bf16) are not exact; they are
//     below 2^-200 and cannot move a binary32 result unless the whole row is that small.
//   * INT8 codes use round-toward-zero adds instead of conversions: r = rz(|t| + 0.5) and
//     w = rz(r + 2^23) give 2^23 + round_half_away(|t|) exactly; the sign is applied with one exact
//     fused multiply-add that leaves the two's-complement code in the low byte of the result.
//     |t| <= fl(m * fl(127/m)) <= 127.00001, so the code never leaves [-127, 127].
//   * pairs of binary32 values use the packed f32x2 instructions of sm_100.
// Arithmetic otherwise follows the RMSNorm / quantiser definitions step by step with explicit
// round-to-nearest operations (nothing is contracted into fused multiply-adds), so results are
// bit-identical to the definitions.
//
// The column abs-max keeps per-column running maxima in registers, combines the groups of a CTA in
// shared memory and the 8 CTAs of a thread-block cluster through distributed shared memory, then
// issues one atomic max per column per cluster. For a norm-fed input the maximum of
// fl(fl(|x| * inv_rms) * |gamma|) over rows equals fl(max(fl(|x| * inv_rms)) * |gamma|) because
// rounding is monotone, so gamma is applied once per column at the end.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace cg = cooperative_groups;
using namespace sqdev;

namespace {

constexpr float kFloor = 1e-5f;   // floor of abs-maxima and of s ([TAMING] listing clamps s at 1e-5)
constexpr float kQmax = 127.0f;   // symmetric INT8 range [-127, 127]
constexpr int kCluster = 8;       // CTAs per cluster in the column abs-max
constexpr int kMaxK = 16384;      // widest row held on chip by the row kernels
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxStages = 6;
constexpr uint32_t kSqBias = 485u << 20;   // binary64 exponent bias mapping bf16 x to x * 2^-411

enum { MODE_ABSMAX = 0, MODE_QUANT = 1 };

struct RowArgs {
    const uint8_t *src;     // row r starts at src + r * ld_bytes (16-byte aligned)
    int64_t rows;
    int64_t ld_bytes;
    int K;                  // bf16 elements per row (multiple of 8)
    int stages;             // ring slots per row group
    const float *vec;       // ABSMAX: norm gamma (NORM) ; QUANT: per-column factor c (nullable)
    float eps;
    double inv_k;           // 1 / K when K is a power of two (exact), else 0
    float *amax;            // ABSMAX output [K] (running maximum; pre-zeroed when overwriting)
    int8_t *q;              // QUANT output [rows, K]
    float *scale;           // QUANT output [rows]
    unsigned int *status;   // device status word
    uint64_t limit_ns;      // bound of every wait
};

// 1 / sqrt(ss / K + eps) with each step rounded as the RMSNorm definition orders it. When K is a
// power of two (inv_k != 0) the division ss / K is the exact multiplication by inv_k = 1 / K.
__device__ __forceinline__ float inv_rms(double ss, int K, double inv_k, float eps) {
    const double q = inv_k != 0.0 ? __dmul_rn(ss, inv_k) : __ddiv_rn(ss, static_cast<double>(K));
    const float ms = __double2float_rn(q);
    const float r = __fsqrt_rn(__fadd_rn(ms, eps));
    return __frcp_rn(r);
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

// Adds the squares of the two bf16 values of `w` to the scaled binary64 accumulator.
__device__ __forceinline__ double add_squares(uint32_t w, double ss) {
    const double a_hi = __hiloint2double(static_cast<int>(mad_hi(w & 0x7FFF0000u, 1u << 29, kSqBias)), 0);
    const double a_lo = __hiloint2double(static_cast<int>((w & 0x7FFFu) * 8192u + kSqBias), 0);
    ss = __fma_rn(a_hi, a_hi, ss);
    return __fma_rn(a_lo, a_lo, ss);
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int k) {
    return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}

// Signed INT8 codes of the two values of `y` (scaled by inv): the code of the low element in the
// low byte, of the high element in the next byte.
__device__ __forceinline__ uint32_t codes2(uint64_t y, uint64_t inv2) {
    const uint64_t t = mul2_rn(y, inv2);
    uint32_t tl, th;
    unpack2(t, tl, th);
    const uint64_t sgn = pack2u((tl & 0x80000000u) | 0x3F800000u, (th & 0x80000000u) | 0x3F800000u);   // +-1
    const uint64_t at = mul2_rn(t, sgn);                                                  // |t|
    const uint64_t r = add2_rz(at, pack2(0.5f, 0.5f));                                    // rz(|t| + 1/2)
    const uint64_t w = add2_rz(r, pack2(8388608.0f, 8388608.0f));                         // 2^23 + q
    const uint64_t qm = add2_rn(w, pack2(-8388736.0f, -8388736.0f));                      // q - 128
    const uint64_t f = fma2_rn(sgn, qm, pack2(8388736.0f, 8388736.0f));                   // 2^23 + 128 +- (q - 128)
    uint32_t fl, fh;
    unpack2(f, fl, fh);
    return __byte_perm(fl, fh, 0x0040);
}

template <int WPR, int VPL, int MODE, bool NORM>
__global__ void __launch_bounds__(kThreads, 2) k_rows(const RowArgs p)
{
    constexpr int G = kWarps / WPR;   // row groups per CTA
    constexpr int GT = 32 * WPR;      // threads per row group
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t s_full[G * kMaxStages];
    __shared__ double s_ss[2][kWarps];
    __shared__ float s_mx[2][kWarps];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int group = warp / WPR, wig = warp % WPR, gtid = wig * 32 + lane;
    const bool leader = gtid == 0;
    const int K = p.K, nvec = K >> 3;
    const uint32_t rowbytes = static_cast<uint32_t>(K) * 2u;
    const int stages = p.stages;
    uint8_t *ring = smem;
    const size_t ring_bytes = static_cast<size_t>(G) * stages * rowbytes;
    float4 *c_lo = reinterpret_cast<float4 *>(smem + ring_bytes);   // c[8v .. 8v+3]
    float4 *c_hi = c_lo + nvec;                                     // c[8v+4 .. 8v+7]

    const int64_t g0 = static_cast<int64_t>(blockIdx.x) * G + group;
    const int64_t gstride = static_cast<int64_t>(gridDim.x) * G;
    const int64_t nrows = g0 < p.rows ? (p.rows - 1 - g0) / gstride + 1 : 0;

    if (tid == 0) {
        for (int i = 0; i < G * stages; ++i) mbar_init(smem_u32(&s_full[i]), 1);
        mbar_init_fence();
    }
    if (MODE == MODE_QUANT && p.vec != nullptr) {
        const float4 *cv = reinterpret_cast<const float4 *>(p.vec);
        for (int v = tid; v < nvec; v += kThreads) { c_lo[v] = __ldg(cv + 2 * v); c_hi[v] = __ldg(cv + 2 * v + 1); }
    }
    __syncthreads();

    auto slot = [&](int s) { return ring + (static_cast<size_t>(group) * stages + s) * rowbytes; };
    auto full_bar = [&](int s) { return smem_u32(&s_full[group * stages + s]); };
    auto issue = [&](int64_t j) {
        const int s = static_cast<int>(j % stages);
        mbar_expect_tx(full_bar(s), rowbytes);
        bulk_g2s(smem_u32(slot(s)), p.src + (g0 + j * gstride) * p.ld_bytes, rowbytes, full_bar(s));
    };
    if (leader)
        for (int64_t j = 0; j < nrows && j < stages; ++j) issue(j);

    float mx[VPL][8];          // ABSMAX with norm: running max of fl(|x| * inv_rms) per column
    uint32_t mh[VPL][4];       // ABSMAX without norm: running max of |x| as bf16 pairs
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[i][e] = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) mh[i][k] = 0u;
    }

    // Row j of this group sits in slot j % stages. Every lane reads the slot twice (sum of squares,
    // then the values themselves) instead of keeping it in registers across the group barrier; the
    // slot of row j-1 is refilled at row j's barrier, after every lane has finished with it.
    int64_t consumed = 0, issued = nrows < stages ? nrows : stages;
    bool failed = false;
    for (int64_t j = 0; j < nrows; ++j) {
        const int s = static_cast<int>(j % stages);
        const bool ok = mbar_wait(full_bar(s), static_cast<uint32_t>((j / stages) & 1), p.limit_ns, nullptr);
        const uint4 *rp = reinterpret_cast<const uint4 *>(slot(s));
        double ss = 0.0;
        if (NORM) {
            double ss1 = 0.0;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int v = i * GT + gtid;
                const uint4 r = (ok && v < nvec) ? rp[v] : make_uint4(0u, 0u, 0u, 0u);
                ss = add_squares(r.x, ss);
                ss1 = add_squares(r.y, ss1);
                ss = add_squares(r.z, ss);
                ss1 = add_squares(r.w, ss1);
            }
            ss = warp_sum(ss + ss1);
        }
        // One group-wide step: partial sums become visible, every lane is done with row j-1, and a
        // failed wait anywhere in the group stops the whole group at the same row.
        bool any_fail;
        if (WPR == 1) {
            any_fail = __any_sync(0xFFFFFFFFu, !ok);
            __syncwarp();
        } else {
            if (NORM && lane == 0) s_ss[j & 1][warp] = ss;
            any_fail = named_sync_or(1 + group, GT, !ok);
            if (NORM) {
                ss = 0.0;
#pragma unroll
                for (int w = 0; w < WPR; ++w) ss += s_ss[j & 1][group * WPR + w];
            }
        }
        if (any_fail) { failed = true; break; }
        consumed = j + 1;
        if (leader && j >= 1 && issued < nrows) issue(issued++);
        const int64_t row = g0 + j * gstride;
        const float ir = NORM ? inv_rms(__dmul_rn(ss, 0x1p822), K, p.inv_k, p.eps) : 1.0f;
        const uint64_t ir2 = pack2(ir, ir);

        if (MODE == MODE_ABSMAX) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int v = i * GT + gtid;
                const uint4 r = v < nvec ? rp[v] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t w = word_of(r, k);
                    if (NORM) {
                        const uint64_t ay = mul2_rn(pack2u((w & 0x7FFFu) << 16, w & 0x7FFF0000u), ir2);
                        uint32_t al, ah;
                        unpack2(ay, al, ah);
                        mx[i][2 * k] = fmaxf(mx[i][2 * k], __uint_as_float(al));
                        mx[i][2 * k + 1] = fmaxf(mx[i][2 * k + 1], __uint_as_float(ah));
                    } else {
                        __nv_bfloat162 cur = *reinterpret_cast<__nv_bfloat162 *>(&mh[i][k]);
                        const uint32_t a = w & 0x7FFF7FFFu;
                        cur = __hmax2(cur, *reinterpret_cast<const __nv_bfloat162 *>(&a));
                        mh[i][k] = *reinterpret_cast<uint32_t *>(&cur);
                    }
                }
            }
        } else {
            // y = (x * inv_rms) * c  (or x * c, or x), kept in registers as element pairs
            uint64_t y[VPL][4];
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int v = i * GT + gtid;
                const uint4 r = v < nvec ? rp[v] : make_uint4(0u, 0u, 0u, 0u);
                float4 cl = make_float4(1.f, 1.f, 1.f, 1.f), ch = cl;
                if (p.vec != nullptr && v < nvec) { cl = c_lo[v]; ch = c_hi[v]; }
                const uint64_t c2[4] = {pack2(cl.x, cl.y), pack2(cl.z, cl.w), pack2(ch.x, ch.y), pack2(ch.z, ch.w)};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t w = word_of(r, k);
                    const uint64_t x2 = pack2u(w << 16, w & 0xFFFF0000u);
                    const uint64_t yy = NORM ? mul2_rn(mul2_rn(x2, ir2), c2[k]) : (p.vec != nullptr ? mul2_rn(x2, c2[k]) : x2);
                    y[i][k] = yy;
                    uint32_t yl, yh;
                    unpack2(yy, yl, yh);
                    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(yl)), fabsf(__uint_as_float(yh))));
                }
            }
            m = warp_max(m);
            if (WPR > 1) {
                if (lane == 0) s_mx[j & 1][warp] = m;
                named_sync(1 + group, GT);
                m = 0.0f;
#pragma unroll
                for (int w = 0; w < WPR; ++w) m = fmaxf(m, s_mx[j & 1][group * WPR + w]);
            }
            const float delta = m > 0.0f ? __fdiv_rn(m, kQmax) : 0.0f;
            const float inv = m > 0.0f ? __fdiv_rn(kQmax, m) : 0.0f;
            const uint64_t inv2 = pack2(inv, inv);
            uint2 *qrow = reinterpret_cast<uint2 *>(p.q + row * static_cast<int64_t>(K));
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int v = i * GT + gtid;
                if (v < nvec) {
                    const uint32_t c01 = codes2(y[i][0], inv2), c23 = codes2(y[i][1], inv2);
                    const uint32_t c45 = codes2(y[i][2], inv2), c67 = codes2(y[i][3], inv2);
                    qrow[v] = make_uint2(__byte_perm(c01, c23, 0x5410), __byte_perm(c45, c67, 0x5410));
                }
            }
            if (leader) p.scale[row] = delta;
        }
    }

    if (failed && leader) atomicCAS(p.status, 0u, static_cast<unsigned int>(SQ_ERR_TIMEOUT));
    // Copies issued but never consumed (only after a failed wait) must land before the CTA exits.
    if (leader) {
        for (int64_t j = consumed; j < issued; ++j)
            if (!mbar_wait(full_bar(static_cast<int>(j % stages)), static_cast<uint32_t>((j / stages) & 1), p.limit_ns, nullptr))
                atomicCAS(p.status, 0u, static_cast<unsigned int>(SQ_ERR_TIMEOUT));
    }

    if (MODE == MODE_ABSMAX) {
        __syncthreads();                                   // the ring is free: reuse it
        float *red = reinterpret_cast<float *>(smem);      // [G][K]
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int v = i * GT + gtid;
            if (v < nvec) {
                float *dst = red + static_cast<size_t>(group) * K + v * 8;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    dst[2 * k] = NORM ? mx[i][2 * k] : __uint_as_float(mh[i][k] << 16);
                    dst[2 * k + 1] = NORM ? mx[i][2 * k + 1] : __uint_as_float(mh[i][k] & 0xFFFF0000u);
                }
            }
        }
        __syncthreads();
        for (int c = tid; c < K; c += kThreads) {
            float m = red[c];
#pragma unroll
            for (int g = 1; g < G; ++g) m = fmaxf(m, red[static_cast<size_t>(g) * K + c]);
            if (NORM) m = __fmul_rn(m, fabsf(__ldg(p.vec + c)));
            red[c] = m;
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int share = (K + kCluster - 1) / kCluster;
        const int c0 = static_cast<int>(cluster.block_rank()) * share;
        const int c1 = min(K, c0 + share);
        for (int c = c0 + tid; c < c1; c += kThreads) {
            float m = 0.0f;
#pragma unroll
            for (int q = 0; q < kCluster; ++q) m = fmaxf(m, cluster.map_shared_rank(red, q)[c]);
            // abs-maxima are non-negative, where IEEE order equals unsigned integer order
            if (m > 0.0f) atomicMax(reinterpret_cast<unsigned int *>(p.amax + c), __float_as_uint(m));
        }
        cluster.sync();
    }
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
// Launch geometry and dispatch.

struct Geo {
    int wpr, vpl, groups, stages;
    size_t smem;
};

Geo row_geo(int K, int mode) {
    const int nvec = K / 8;
    Geo g;
    g.wpr = nvec <= 256 ? 1 : nvec <= 512 ? 2 : nvec <= 1024 ? 4 : 8;
    const int per = (nvec + 32 * g.wpr - 1) / (32 * g.wpr);
    g.vpl = g.wpr > 1 ? 8 : per <= 1 ? 1 : per <= 2 ? 2 : per <= 4 ? 4 : 8;
    g.groups = kWarps / g.wpr;
    const size_t rowbytes = static_cast<size_t>(K) * 2;
    const size_t extra = mode == MODE_QUANT ? static_cast<size_t>(K) * 4 : 0;
    const long budget = 96L * 1024 - static_cast<long>(extra);
    long st = budget / static_cast<long>(g.groups * rowbytes);
    g.stages = static_cast<int>(st < 2 ? 2 : st > kMaxStages ? kMaxStages : st);
    const size_t ring = static_cast<size_t>(g.groups) * g.stages * rowbytes;
    const size_t red = mode == MODE_ABSMAX ? static_cast<size_t>(g.groups) * K * 4 : 0;
    g.smem = (ring > red ? ring : red) + extra;
    return g;
}

template <int WPR, int VPL, int MODE, bool NORM>
sq_status launch_rows_t(RowArgs a, const Geo &geo, int dev, cudaStream_t st) {
    auto kern = k_rows<WPR, VPL, MODE, NORM>;
    constexpr int G = kWarps / WPR;
    static size_t configured_smem[64];
    static int per_sm[64];
    if (configured_smem[dev] < geo.smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(geo.smem));
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaFuncSetAttribute(rows)");
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, geo.smem);
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor(rows)");
        per_sm[dev] = nb > 0 ? nb : 1;
        configured_smem[dev] = geo.smem;
    }
    const int64_t full = static_cast<int64_t>(sq::sm_count(dev)) * per_sm[dev];
    a.stages = geo.stages;
    a.inv_k = (a.K & (a.K - 1)) == 0 ? 1.0 / static_cast<double>(a.K) : 0.0;
    a.status = sq::device_status_word(dev);
    a.limit_ns = sq::wait_timeout_ns(dev);
    if (a.status == nullptr) return sq::fail(SQ_ERR_CUDA, "device status word unavailable");
    if (MODE == MODE_QUANT) {
        int64_t ctas = (a.rows + G - 1) / G;
        if (ctas > full) ctas = full;
        kern<<<static_cast<unsigned>(ctas), kThreads, geo.smem, st>>>(a);
        return sq::cuda_status(cudaGetLastError(), "launch(rowquant)");
    }
    int64_t ctas = (a.rows + 8 * G - 1) / (8 * G);     // at least ~8 rows per group
    if (ctas > full) ctas = full;
    ctas = ((ctas + kCluster - 1) / kCluster) * kCluster;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = geo.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return sq::cuda_status(cudaLaunchKernelEx(&cfg, kern, a), "launch(absmax)");
}

template <int MODE, bool NORM>
sq_status dispatch_rows(const RowArgs &a, int dev, cudaStream_t st) {
    const Geo g = row_geo(a.K, MODE);
    switch (g.wpr * 16 + g.vpl) {
        case 1 * 16 + 1: return launch_rows_t<1, 1, MODE, NORM>(a, g, dev, st);
        case 1 * 16 + 2: return launch_rows_t<1, 2, MODE, NORM>(a, g, dev, st);
        case 1 * 16 + 4: return launch_rows_t<1, 4, MODE, NORM>(a, g, dev, st);
        case 1 * 16 + 8: return launch_rows_t<1, 8, MODE, NORM>(a, g, dev, st);
        case 2 * 16 + 8: return launch_rows_t<2, 8, MODE, NORM>(a, g, dev, st);
        case 4 * 16 + 8: return launch_rows_t<4, 8, MODE, NORM>(a, g, dev, st);
        default: return launch_rows_t<8, 8, MODE, NORM>(a, g, dev, st);
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
    if (cols > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_calibrate_absmax: cols must be <= %d", kMaxK);
    int dev = 0;
    SQ_TRY_ARCH(dev);
    cudaStream_t st = sq::as_stream(stream);
    if (!accumulate) {
        k_fill_zero<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(amax, cols);
        sq_status s0 = sq::cuda_status(cudaGetLastError(), "launch(fill)");
        if (s0 != SQ_OK) return s0;
    }
    if (rows == 0) return SQ_OK;
    RowArgs ra = {};
    ra.src = static_cast<const uint8_t *>(a);
    ra.rows = rows;
    ra.ld_bytes = ld * 2;
    ra.K = static_cast<int>(cols);
    ra.vec = norm_gamma;
    ra.eps = eps;
    ra.amax = amax;
    return norm_gamma ? dispatch_rows<MODE_ABSMAX, true>(ra, dev, st) : dispatch_rows<MODE_ABSMAX, false>(ra, dev, st);
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
    int dev = 0;
    SQ_TRY_ARCH(dev);
    if (N == 0) return SQ_OK;
    RowArgs ra = {};
    ra.src = static_cast<const uint8_t *>(w);
    ra.rows = N;
    ra.ld_bytes = K * 2;
    ra.K = static_cast<int>(K);
    ra.vec = s;
    ra.q = wq;
    ra.scale = w_scale;
    return dispatch_rows<MODE_QUANT, false>(ra, dev, sq::as_stream(stream));
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
    int dev = 0;
    SQ_TRY_ARCH(dev);
    if (T == 0) return SQ_OK;
    RowArgs ra = {};
    ra.src = static_cast<const uint8_t *>(x);
    ra.rows = T;
    ra.ld_bytes = K * 2;
    ra.K = static_cast<int>(K);
    ra.vec = fold;
    ra.eps = eps;
    ra.q = xq;
    ra.scale = x_scale;
    cudaStream_t st = sq::as_stream(stream);
    return apply_norm ? dispatch_rows<MODE_QUANT, true>(ra, dev, st) : dispatch_rows<MODE_QUANT, false>(ra, dev, st);
}

}  // extern "C"
