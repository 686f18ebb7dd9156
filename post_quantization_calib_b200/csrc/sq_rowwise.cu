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
constexpr int kMaxCluster = 8;    // largest cluster tried for the column abs-max
constexpr int kMaxK = 16384;      // widest row held on chip by the row kernels
constexpr int kWarps = 8;                   // consumer warps per CTA
constexpr int kThreads = 32 * (kWarps + 1); // plus one producer warp
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

// 3-input maximum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// One CTA = 8 consumer warps in row groups of WPR warps + 1 producer warp. A group processes units of
// R consecutive rows; lane l of warp w of the group holds 8-element vectors v = i * 32 * WPR +
// 32 * w + l (i < VPL) of every row of the unit.
template <int WPR, int VPL, int R, int MODE, bool NORM, bool FULL>
__global__ void __launch_bounds__(kThreads, 2) k_rows(const RowArgs p)
{
    constexpr int G = kWarps / WPR;   // row groups per CTA
    constexpr int GT = 32 * WPR;      // consumer threads per row group
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t s_full[G * kMaxStages];
    __shared__ __align__(8) uint64_t s_empty[G * kMaxStages];
    __shared__ double s_ss[2][kWarps][R];
    __shared__ float s_mx[2][kWarps][R];
    __shared__ int s_abort[G];
    __shared__ long long s_consumed[G];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool producer = warp == kWarps;                 // the last warp refills the rings
    const int group = producer ? lane : warp / WPR;        // producer lane g serves group g
    const int wig = warp % WPR, gtid = wig * 32 + lane;
    const bool leader = !producer && gtid == 0;
    const int K = p.K, nvec = K >> 3;
    const uint32_t rowbytes = static_cast<uint32_t>(K) * 2u;
    const uint32_t slotbytes = rowbytes * R;
    const int stages = p.stages;
    uint8_t *ring = smem;
    const size_t ring_bytes = static_cast<size_t>(G) * stages * slotbytes;
    float4 *c_lo = reinterpret_cast<float4 *>(smem + ring_bytes);   // c[8v .. 8v+3]
    float4 *c_hi = c_lo + nvec;                                     // c[8v+4 .. 8v+7]

    const int64_t units = (p.rows + R - 1) / R;
    const int64_t g0 = static_cast<int64_t>(blockIdx.x) * G + group;
    const int64_t gstride = static_cast<int64_t>(gridDim.x) * G;
    const int64_t nunits = (group < G && g0 < units) ? (units - 1 - g0) / gstride + 1 : 0;

    if (tid == 0) {
        for (int i = 0; i < G * stages; ++i) {
            mbar_init(smem_u32(&s_full[i]), 1);
            mbar_init(smem_u32(&s_empty[i]), WPR);
        }
        for (int g = 0; g < G; ++g) { s_abort[g] = 0; s_consumed[g] = 0; }
        mbar_init_fence();
    }
    if (MODE == MODE_QUANT && p.vec != nullptr) {
        const float4 *cv = reinterpret_cast<const float4 *>(p.vec);
        for (int v = tid; v < nvec; v += kThreads) { c_lo[v] = __ldg(cv + 2 * v); c_hi[v] = __ldg(cv + 2 * v + 1); }
    }
    __syncthreads();

    auto slot = [&](int s) { return ring + (static_cast<size_t>(group) * stages + s) * slotbytes; };
    auto full_bar = [&](int s) { return smem_u32(&s_full[group * stages + s]); };
    auto empty_bar = [&](int s) { return smem_u32(&s_empty[group * stages + s]); };
    volatile int *abort_flag = &s_abort[group < G ? group : 0];

    float mx[VPL][8];          // ABSMAX with norm: running max of fl(|x| * inv_rms) per column
    uint32_t mh[VPL][4];       // ABSMAX without norm: running max of |x| as bf16 pairs
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[i][e] = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) mh[i][k] = 0u;
    }

    int64_t issued = 0;
    bool failed = false;
    if (producer) {
        // Lane g keeps group g's ring full: a slot is refilled as soon as the group's warps have
        // released it, independently of the group's progress on later units.
        if (lane < G) {
            int s = 0;
            uint32_t phase = 0;
            for (int64_t j = 0; j < nunits; ++j) {
                if (!mbar_ready(empty_bar(s), phase ^ 1u, p.limit_ns, abort_flag)) {
                    if (!*abort_flag) failed = true;
                    *abort_flag = 1;
                    break;
                }
                const int64_t r0 = (g0 + j * gstride) * R;
                const int nr = static_cast<int>(p.rows - r0 < R ? p.rows - r0 : R);
                mbar_expect_tx(full_bar(s), rowbytes * static_cast<uint32_t>(nr));
                for (int r = 0; r < nr; ++r)
                    bulk_g2s(smem_u32(slot(s) + r * rowbytes), p.src + (r0 + r) * p.ld_bytes, rowbytes, full_bar(s));
                issued = j + 1;
                if (++s == stages) { s = 0; phase ^= 1u; }
            }
        }
    } else {
        int64_t consumed = 0;
        int s = 0;
        uint32_t phase = 0;
        for (int64_t j = 0; j < nunits; ++j) {
            const bool ok = mbar_ready(full_bar(s), phase, p.limit_ns, abort_flag);
            const int64_t r0 = (g0 + j * gstride) * R;
            const int nr = static_cast<int>(p.rows - r0 < R ? p.rows - r0 : R);   // uniform in the group
            const uint4 *rp = reinterpret_cast<const uint4 *>(slot(s));
            const int rv = static_cast<int>(rowbytes / 16);                           // vectors per row
            double ss[R];
#pragma unroll
            for (int r = 0; r < R; ++r) ss[r] = 0.0;
            if (NORM) {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (r < nr) {
                        double a = 0.0, b = 0.0;
#pragma unroll
                        for (int i = 0; i < VPL; ++i) {
                            const int v = i * GT + gtid;
                            const uint4 q = (ok && (FULL || v < nvec)) ? rp[r * rv + v] : make_uint4(0u, 0u, 0u, 0u);
                            a = add_squares(q.x, a);
                            b = add_squares(q.y, b);
                            a = add_squares(q.z, a);
                            b = add_squares(q.w, b);
                        }
                        ss[r] = warp_sum(a + b);
                    }
                }
            }
            // Group-wide step: partial sums become visible, and a failed wait anywhere in the group
            // stops the whole group at the same unit.
            bool any_fail;
            if (WPR == 1) {
                any_fail = __any_sync(0xFFFFFFFFu, !ok);
            } else {
                if (NORM && lane == 0) {
#pragma unroll
                    for (int r = 0; r < R; ++r) s_ss[j & 1][warp][r] = ss[r];
                }
                any_fail = named_sync_or(1 + group, GT, !ok);
                if (NORM) {
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        double t = 0.0;
#pragma unroll
                        for (int w = 0; w < WPR; ++w) t += s_ss[j & 1][group * WPR + w][r];
                        ss[r] = t;
                    }
                }
            }
            if (any_fail) {
                if (leader) { if (!*abort_flag) failed = true; *abort_flag = 1; }
                break;
            }
            uint64_t ir2[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float ir = NORM ? inv_rms(__dmul_rn(ss[r], 0x1p822), K, p.inv_k, p.eps) : 1.0f;
                ir2[r] = pack2(ir, ir);
            }

            if (MODE == MODE_ABSMAX) {
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int v = i * GT + gtid;
                    const bool in = FULL || v < nvec;
                    uint4 q[R];
#pragma unroll
                    for (int r = 0; r < R; ++r) q[r] = (in && r < nr) ? rp[r * rv + v] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (NORM) {
                            float yl[R], yh[R];
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                const uint32_t w = word_of(q[r], k);
                                uint32_t l, h;
                                unpack2(mul2_rn(pack2u(w << 16, w & 0xFFFF0000u), ir2[r]), l, h);
                                yl[r] = fabsf(__uint_as_float(l));
                                yh[r] = fabsf(__uint_as_float(h));
                            }
                            if (R == 2) {
                                mx[i][2 * k] = max3f(mx[i][2 * k], yl[0], yl[R - 1]);
                                mx[i][2 * k + 1] = max3f(mx[i][2 * k + 1], yh[0], yh[R - 1]);
                            } else {
                                mx[i][2 * k] = fmaxf(mx[i][2 * k], yl[0]);
                                mx[i][2 * k + 1] = fmaxf(mx[i][2 * k + 1], yh[0]);
                            }
                        } else {
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                __nv_bfloat162 cur = *reinterpret_cast<__nv_bfloat162 *>(&mh[i][k]);
                                const uint32_t a = word_of(q[r], k) & 0x7FFF7FFFu;
                                cur = __hmax2(cur, *reinterpret_cast<const __nv_bfloat162 *>(&a));
                                mh[i][k] = *reinterpret_cast<uint32_t *>(&cur);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(s));      // this warp is done with the slot
            } else {
                // y = (x * inv_rms) * c  (or x * c, or x), kept in registers as element pairs
                uint64_t y[R][VPL][4];
                float m[R];
#pragma unroll
                for (int r = 0; r < R; ++r) m[r] = 0.0f;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int v = i * GT + gtid;
                    const bool in = FULL || v < nvec;
                    float4 cl = make_float4(1.f, 1.f, 1.f, 1.f), ch = cl;
                    if (p.vec != nullptr && in) { cl = c_lo[v]; ch = c_hi[v]; }
                    const uint64_t c2[4] = {pack2(cl.x, cl.y), pack2(cl.z, cl.w), pack2(ch.x, ch.y), pack2(ch.z, ch.w)};
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint4 q = (in && r < nr) ? rp[r * rv + v] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t w = word_of(q, k);
                            const uint64_t x2 = pack2u(w << 16, w & 0xFFFF0000u);
                            const uint64_t yy = NORM ? mul2_rn(mul2_rn(x2, ir2[r]), c2[k]) : (p.vec != nullptr ? mul2_rn(x2, c2[k]) : x2);
                            y[r][i][k] = yy;
                            uint32_t yl, yh;
                            unpack2(yy, yl, yh);
                            m[r] = max3f(m[r], fabsf(__uint_as_float(yl)), fabsf(__uint_as_float(yh)));
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(s));      // the unit is in registers now
#pragma unroll
                for (int r = 0; r < R; ++r) m[r] = warp_max(m[r]);
                if (WPR > 1) {
                    if (lane == 0) {
#pragma unroll
                        for (int r = 0; r < R; ++r) s_mx[j & 1][warp][r] = m[r];
                    }
                    named_sync(1 + group, GT);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        float t = 0.0f;
#pragma unroll
                        for (int w = 0; w < WPR; ++w) t = fmaxf(t, s_mx[j & 1][group * WPR + w][r]);
                        m[r] = t;
                    }
                }
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (r < nr) {
                        const float delta = m[r] > 0.0f ? __fdiv_rn(m[r], kQmax) : 0.0f;
                        const float inv = m[r] > 0.0f ? __fdiv_rn(kQmax, m[r]) : 0.0f;
                        const uint64_t inv2 = pack2(inv, inv);
                        uint2 *qrow = reinterpret_cast<uint2 *>(p.q + (r0 + r) * static_cast<int64_t>(K));
#pragma unroll
                        for (int i = 0; i < VPL; ++i) {
                            const int v = i * GT + gtid;
                            if (FULL || v < nvec) {
                                const uint32_t c01 = codes2(y[r][i][0], inv2), c23 = codes2(y[r][i][1], inv2);
                                const uint32_t c45 = codes2(y[r][i][2], inv2), c67 = codes2(y[r][i][3], inv2);
                                qrow[v] = make_uint2(__byte_perm(c01, c23, 0x5410), __byte_perm(c45, c67, 0x5410));
                            }
                        }
                        if (leader) p.scale[r0 + r] = delta;
                    }
                }
            }
            consumed = j + 1;
            if (++s == stages) { s = 0; phase ^= 1u; }
        }
        if (leader) s_consumed[group] = consumed;
    }

    if (failed) atomicCAS(p.status, 0u, static_cast<unsigned int>(SQ_ERR_TIMEOUT));
    __syncthreads();
    // Copies issued but never consumed (only after a failed wait) must land before the CTA exits.
    if (producer && lane < G) {
        for (int64_t j = s_consumed[group]; j < issued; ++j)
            if (!mbar_wait(full_bar(static_cast<int>(j % stages)), static_cast<uint32_t>((j / stages) & 1), p.limit_ns, nullptr))
                atomicCAS(p.status, 0u, static_cast<unsigned int>(SQ_ERR_TIMEOUT));
    }

    if (MODE == MODE_ABSMAX) {
        __syncthreads();                                   // the ring is idle: reuse it
        float *red = reinterpret_cast<float *>(smem);      // [G][K]
        if (!producer) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int v = i * GT + gtid;
                if (FULL || v < nvec) {
                    float *dst = red + static_cast<size_t>(group) * K + v * 8;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        dst[2 * k] = NORM ? mx[i][2 * k] : __uint_as_float(mh[i][k] << 16);
                        dst[2 * k + 1] = NORM ? mx[i][2 * k + 1] : __uint_as_float(mh[i][k] & 0xFFFF0000u);
                    }
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
        const int csize = static_cast<int>(cluster.num_blocks());
        const int share = (K + csize - 1) / csize;
        const int c0 = static_cast<int>(cluster.block_rank()) * share;
        const int c1 = min(K, c0 + share);
        for (int c = c0 + tid; c < c1; c += kThreads) {
            float m = 0.0f;
            for (int q = 0; q < csize; ++q) m = fmaxf(m, cluster.map_shared_rank(red, q)[c]);
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
    int wpr, vpl, rpu, groups, stages;   // warps per row group, vectors per lane, rows per unit
    size_t smem;
};

// Row groups hold 64 values per lane per unit where possible (4 vectors x 2 rows).
Geo row_geo(int K, int mode) {
    const int nvec = K / 8;
    Geo g;
    if (nvec <= 128) {
        g.wpr = 1;
        const int per = (nvec + 31) / 32;
        g.vpl = per <= 1 ? 1 : per <= 2 ? 2 : 4;
        g.rpu = 2;
    } else if (nvec <= 1024) {
        g.wpr = nvec <= 256 ? 2 : nvec <= 512 ? 4 : 8;
        g.vpl = 4;
        g.rpu = 2;
    } else {
        g.wpr = 8;
        g.vpl = 8;
        g.rpu = 1;
    }
    g.groups = kWarps / g.wpr;
    const size_t slotbytes = static_cast<size_t>(K) * 2 * g.rpu;
    const size_t extra = mode == MODE_QUANT ? static_cast<size_t>(K) * 4 : 0;
    const long budget = 96L * 1024 - static_cast<long>(extra);
    long st = budget / static_cast<long>(g.groups * slotbytes);
    g.stages = static_cast<int>(st < 2 ? 2 : st > kMaxStages ? kMaxStages : st);
    const size_t ring = static_cast<size_t>(g.groups) * g.stages * slotbytes;
    const size_t red = mode == MODE_ABSMAX ? static_cast<size_t>(g.groups) * K * 4 : 0;
    g.smem = (ring > red ? ring : red) + extra;
    return g;
}

template <int WPR, int VPL, int R, int MODE, bool NORM, bool FULL>
sq_status launch_rows_t(RowArgs a, const Geo &geo, int dev, cudaStream_t st) {
    auto kern = k_rows<WPR, VPL, R, MODE, NORM, FULL>;
    constexpr int G = kWarps / WPR;
    static size_t configured_smem[64];
    static int per_sm[64];
    static int cluster_size[64], cluster_ctas[64];
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = geo.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (configured_smem[dev] < geo.smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(geo.smem));
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaFuncSetAttribute(rows)");
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, geo.smem);
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor(rows)");
        per_sm[dev] = nb > 0 ? nb : 1;
        if (MODE == MODE_ABSMAX) {
            // Whole clusters must fit on one GPU processing cluster; take the size that keeps the
            // most CTAs resident at once (ties: the larger cluster, fewer atomics).
            cluster_size[dev] = 1;
            cluster_ctas[dev] = 0;
            for (int c = kMaxCluster; c >= 2; c /= 2) {
                attr[0].val.clusterDim.x = c;
                cfg.gridDim = dim3(c, 1, 1);
                int nc = 0;
                if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess) { (void)cudaGetLastError(); continue; }
                if (nc * c > cluster_ctas[dev]) { cluster_ctas[dev] = nc * c; cluster_size[dev] = c; }
            }
            if (cluster_ctas[dev] == 0) return sq::fail(SQ_ERR_CUDA, "no cluster configuration fits the abs-max kernel");
        }
        configured_smem[dev] = geo.smem;
    }
    const int64_t full = static_cast<int64_t>(sq::sm_count(dev)) * per_sm[dev];
    a.stages = geo.stages;
    a.inv_k = (a.K & (a.K - 1)) == 0 ? 1.0 / static_cast<double>(a.K) : 0.0;
    a.status = sq::device_status_word(dev);
    a.limit_ns = sq::wait_timeout_ns(dev);
    if (a.status == nullptr) return sq::fail(SQ_ERR_CUDA, "device status word unavailable");
    const int64_t units = (a.rows + R - 1) / R;
    if (MODE == MODE_QUANT) {
        int64_t ctas = (units + G - 1) / G;
        if (ctas > full) ctas = full;
        kern<<<static_cast<unsigned>(ctas), kThreads, geo.smem, st>>>(a);
        return sq::cuda_status(cudaGetLastError(), "launch(rowquant)");
    }
    // one wave of resident clusters at most, at least ~4 units per group
    const int csz = cluster_size[dev];
    int64_t ctas = (units + 4 * G - 1) / (4 * G);
    if (ctas > cluster_ctas[dev]) ctas = cluster_ctas[dev];
    ctas = ((ctas + csz - 1) / csz) * csz;
    attr[0].val.clusterDim.x = csz;
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
    return sq::cuda_status(cudaLaunchKernelEx(&cfg, kern, a), "launch(absmax)");
}

template <int MODE, bool NORM, bool FULL>
sq_status dispatch_rows_f(const RowArgs &a, const Geo &g, int dev, cudaStream_t st) {
    switch (g.wpr * 100 + g.vpl * 10 + g.rpu) {
        case 112: return launch_rows_t<1, 1, 2, MODE, NORM, FULL>(a, g, dev, st);
        case 122: return launch_rows_t<1, 2, 2, MODE, NORM, FULL>(a, g, dev, st);
        case 142: return launch_rows_t<1, 4, 2, MODE, NORM, FULL>(a, g, dev, st);
        case 242: return launch_rows_t<2, 4, 2, MODE, NORM, FULL>(a, g, dev, st);
        case 442: return launch_rows_t<4, 4, 2, MODE, NORM, FULL>(a, g, dev, st);
        case 842: return launch_rows_t<8, 4, 2, MODE, NORM, FULL>(a, g, dev, st);
        default: return launch_rows_t<8, 8, 1, MODE, NORM, FULL>(a, g, dev, st);
    }
}

// FULL: the row is exactly VPL vectors per lane of the group (no bounds checks per vector).
template <int MODE, bool NORM>
sq_status dispatch_rows(const RowArgs &a, int dev, cudaStream_t st) {
    const Geo g = row_geo(a.K, MODE);
    const bool full = (a.K / 8) == g.vpl * 32 * g.wpr;
    return full ? dispatch_rows_f<MODE, NORM, true>(a, g, dev, st) : dispatch_rows_f<MODE, NORM, false>(a, g, dev, st);
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
