// sq_rowwise.cu -- the HBM-bound steps of the smoothed W8A8 linear on sm_100a:
//   per-input-channel abs-max (calibration activations and weights, optionally of their RMSNorm or
//   LayerNorm output), smoothing factors with the fold into the norm weight, the static per-tensor
//   scale, and the row quantisers (weights per output channel, activations per token with the RMSNorm
//   or LayerNorm fused in; INT8, INT8 with a static scale, or FP8 E4M3).
//
// Pages cited (title, then section / equation / figure):
//   [MIGRATE] "06 -- SmoothQuant: Migrating Difficulty from Activations to Weights"
//   [TAMING]  "Taming the Outliers: A Deep Dive into SmoothQuant for LLM Quantization"
//   [W8A8]    "SmoothQuant and W8A8: Quantizing Activations Too"
//   [WOVS]    "SmoothQuant: Weight-Only vs W8A8"
//
// Design (B200). One kernel template serves the abs-max and the quantisers (the MODE_* values below).
// A CTA (one per SM) has 16 warps, 4 per scheduler. Rows of up to 2048 elements are
// handled by a single warp each, wider rows by row groups of 2, 4 or 8 warps; narrower rows are
// batched R at a time, so that a unit always gives a lane 8 vectors of 8 elements (64 element-rows)
// against a fixed per-unit cost. Each row group streams its units through its own shared-memory ring
// of 2-4 slots, filled with TMA bulk copies (one 1-D copy per row, completion on an mbarrier): as
// soon as the group has read a slot for the last time, a lane issues the copies of the unit that goes
// there next (the leader once the quantiser holds the unit in registers; for the abs-max, which
// re-reads the slot, the last warp of the group to finish with it), so two or more units per group
// are in flight while the group computes on the current one. There is no separate producer warp, so
// all 16 warps compute. A column abs-max over few rows uses four-warp groups instead of two.
//
// Every kernel is launched as a dependent launch: it sets up shared memory, then waits
// (griddepcontrol.wait) for the previous kernel of the stream before it reads global memory. The
// abs-max that follows this library's own zero-fill of amax streams its rows at once and waits only
// before its atomics: the fill itself waited for all earlier work before it let the abs-max start.
//
// Per unit, sums and maxima of the R rows are reduced across the warp with one butterfly that
// halves the number of values at each exchange, so a lane ends up with the total of one row; the
// per-row scalar steps (1/rms, the quantisation step and its reciprocal) then run once, in parallel
// across lanes, and are broadcast with shuffles.
//
// Instruction budget. These kernels must retire about 8-12 bf16 elements per SM cycle to keep up
// with HBM, so each element gets only a few instructions:
//   * the RMSNorm sum of squares is binary64, but each operand is built with integer operations:
//     the bf16 exponent and mantissa are placed in the binary64 fields with exponent bias +485, which
//     is exactly x * 2^-411 for every normal |x| >= 2^-100 (and a zero becomes 2^-538, whose square
//     2^-1076 rounds away inside the fused multiply-add); the binary64 accumulator is rescaled by
//     2^822 at the end. Squares of |x| < 2^-100 (and of subnormal bf16) are not exact; they are
//     below 2^-200 and cannot move a binary32 result unless the whole row is that small.
//   * INT8 codes: v = rz(y * iv + copysign(1/2, y)) in one fused multiply-add (round toward zero
//     cannot carry the sum across an integer), then a truncating conversion gives
//     round_half_away(y * iv) of the exact product; |y * iv| <= m * fl(127/m) <= 127.00001, so the
//     code never leaves [-127, 127]; four codes are packed with two saturating conversions.
//   * the quantisers' per-element arithmetic is scalar binary32 (the packed f32x2 forms cost more
//     register moves than they save there); the abs-max keeps the packed forms.
// Arithmetic otherwise follows the RMSNorm / quantiser definitions step by step with explicit
// round-to-nearest operations (nothing is contracted into fused multiply-adds), so results are
// bit-identical to the definitions.
//
// The column abs-max keeps per-column running maxima in registers, combines the warps of a CTA in
// shared memory and the CTAs of a thread-block cluster through distributed shared memory, then
// issues one atomic max per column per cluster. For a norm-fed input the maximum of
// fl(fl(|x| * inv_rms) * |gamma|) over rows equals fl(max(fl(|x| * inv_rms)) * |gamma|) because
// rounding is monotone, so gamma is applied once per column at the end.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <mutex>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace cg = cooperative_groups;
using namespace sqdev;

namespace {

constexpr float kFloor = 1e-5f;   // floor of abs-maxima and of s ([TAMING] listing clamps s at 1e-5)
constexpr float kQmax = 127.0f;   // symmetric INT8 range [-127, 127]
constexpr int kMaxCluster = 8;    // largest cluster tried for the column abs-max
constexpr int kMaxK = 16384;      // widest row held on chip by the row kernels
constexpr int kWarps = 16;                  // warps per CTA
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxStages = 4;
constexpr uint32_t kSqBias = 485u << 20;   // binary64 exponent bias mapping bf16 x to x * 2^-411
constexpr unsigned kAll = 0xFFFFFFFFu;

// MODE_QSTATIC: the quantiser with one static per-tensor scale (no row maximum; codes clamped).
// MODE_QF8: the per-row quantiser with FP8 E4M3 codes (scale max/448).
// MODE_QLN / MODE_ALN: the per-row quantiser and the column abs-max of a LayerNorm's output
// y = fl(fl(fl(c * inv_std) * g) + b), c = fl(x - mean) (g from vec, b from vec2).
enum { MODE_ABSMAX = 0, MODE_QUANT = 1, MODE_QSTATIC = 2, MODE_QF8 = 3, MODE_QLN = 4, MODE_ALN = 5 };
constexpr float kF8Max = 448.0f;  // largest finite E4M3 value

struct RowArgs {
    const uint8_t *src;     // row r starts at src + r * ld_bytes (16-byte aligned)
    int64_t rows;
    int64_t ld_bytes;
    int K;                  // bf16 elements per row (multiple of 8)
    int stages;             // ring slots per row group
    const float *vec;       // ABSMAX: norm gamma (NORM) ; QUANT: per-column factor c (nullable)
    const float *vec2;      // LayerNorm modes: per-column bias b (nullable = none)
    float eps;
    double inv_k;           // 1 / K when K is a power of two (exact), else 0
    float *amax;            // ABSMAX output [K] (running maximum; pre-zeroed when overwriting)
    int8_t *q;              // QUANT output [rows, K]
    float *scale;           // QUANT output [rows]
    const float *scale2;    // QSTATIC: {delta, 127 / m} of the static per-tensor scale
    unsigned int *status;   // device status word
    uint64_t limit_ns;      // bound of every wait
    int stream_once;        // input larger than half the L2: its lines are evicted first
    int early;              // ABSMAX modes launched right after this library's zero-fill of amax: the
                            // rows may be read before pdl_wait(); amax is touched only after it
    int group_major;        // unit numbering across the grid: 1 = group by group over all CTAs (few units
                            // per group: each SM gets an equal share), 0 = CTA by CTA
};

// 1 / sqrt(ss / K + eps) with each step rounded as the RMSNorm definition orders it. When K is a
// power of two (inv_k != 0) the division ss / K is the exact multiplication by inv_k = 1 / K.
__device__ __forceinline__ float inv_rms(double ss, int K, double inv_k, float eps) {
    const double q = inv_k != 0.0 ? __dmul_rn(ss, inv_k) : __ddiv_rn(ss, static_cast<double>(K));
    const float ms = __double2float_rn(q);
    const float r = __fsqrt_rn(__fadd_rn(ms, eps));
    return __frcp_rn(r);
}

// Butterfly reduction of R per-lane values (one per row of a unit) across the warp. Each exchange
// halves the number of values a lane holds; when one is left the remaining exchanges are plain.
// Afterwards every lane holds the total of row (lane / (32 / R)).
template <int R>
__device__ __forceinline__ double rows_sum(double (&v)[R], int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int n = R >> step;
        if (n >= 2) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
                const double send = up ? v[i] : v[i + n / 2];
                const double keep = up ? v[i + n / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(kAll, send, o);
            }
        } else {
            v[0] += __shfl_xor_sync(kAll, v[0], o);
        }
    }
    return v[0];
}

template <int R>
__device__ __forceinline__ float rows_max(float (&v)[R], int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int n = R >> step;
        if (n >= 2) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < n / 2; ++i) {
                const float send = up ? v[i] : v[i + n / 2];
                const float keep = up ? v[i + n / 2] : v[i];
                v[i] = fmaxf(keep, __shfl_xor_sync(kAll, send, o));
            }
        } else {
            v[0] = fmaxf(v[0], __shfl_xor_sync(kAll, v[0], o));
        }
    }
    return v[0];
}

// |x| * 2^-411 in binary64 for the binary32 bits of |x| in `a` (a bf16 x: its bits in 30..16, the
// low half zero): one 64-bit multiply-add a * 2^29 + (485 << 52) writes both halves of the
// register pair.
__device__ __forceinline__ double sq_operand(uint32_t a) {
    double d;
    asm("{\n\t.reg .u64 t;\n\tmad.wide.u32 t, %1, 536870912, %2;\n\tmov.b64 %0, t;\n\t}"
        : "=d"(d) : "r"(a), "l"(static_cast<uint64_t>(kSqBias) << 32));
    return d;
}

// Adds the squares of the two bf16 values of `w` to the scaled binary64 accumulators a and b.
// WIDE: operands built with one 64-bit multiply-add each (fewer instructions, more registers; the
// quantiser, which keeps its unit in registers, uses the 32-bit form).
template <bool WIDE>
__device__ __forceinline__ void add_squares(uint32_t w, double &a, double &b) {
    double d_hi, d_lo;
    if (WIDE) {
        d_hi = sq_operand(w & 0x7FFF0000u);
        d_lo = sq_operand((w << 16) & 0x7FFF0000u);
    } else {
        d_hi = __hiloint2double(static_cast<int>(mad_hi(w & 0x7FFF0000u, 1u << 29, kSqBias)), 0);
        d_lo = __hiloint2double(static_cast<int>((w & 0x7FFFu) * 8192u + kSqBias), 0);
    }
    a = __fma_rn(d_hi, d_hi, a);
    b = __fma_rn(d_lo, d_lo, b);
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int k) {
    return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}

// bf16 pair -> packed binary32 pair (exact)
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) { return pack2u(w << 16, w & 0xFFFF0000u); }

// Adds the two bf16 values of `w` (exactly converted) to the binary64 sums a and b.
__device__ __forceinline__ void add_values(uint32_t w, double &a, double &b) {
    a = __dadd_rn(a, static_cast<double>(__uint_as_float(w << 16)));
    b = __dadd_rn(b, static_cast<double>(__uint_as_float(w & 0xFFFF0000u)));
}

// Adds the squares of c = fl(x - m) for the two bf16 values x of `w` (nm2 = {-m, -m}) to the
// scaled binary64 accumulators a and b: one 64-bit multiply-add places the binary32 |c| in the
// binary64 fields with exponent bias +485, i.e. |c| * 2^-411, exact for normal |c| >= 2^-100 (a zero
// becomes 2^-538, whose square rounds away in the fused multiply-add).
__device__ __forceinline__ void add_centred_squares(uint32_t w, uint64_t nm2, double &a, double &b) {
    uint32_t cl, ch;
    unpack2(add2_rn(bf2_to_f2(w), nm2), cl, ch);
    const double dl = sq_operand(cl & 0x7FFFFFFFu), dh = sq_operand(ch & 0x7FFFFFFFu);
    a = __fma_rn(dl, dl, a);
    b = __fma_rn(dh, dh, b);
}

// INT8 code of y with the reciprocal step iv: round half away from zero of the exact product y * iv.
// v = rz(y * iv + copysign(1/2, y)) in one fused multiply-add rounded toward zero cannot carry the
// sum across an integer (an integer is representable), so the truncating conversion of v gives
// round_half_away(y * iv) (iv > 0, so y * iv has the sign of y); |y * iv| <= 127.00001 on the
// dynamic path, so its code never leaves [-127, 127].
__device__ __forceinline__ int code_of(float y, float iv) {
    const float h = __uint_as_float((__float_as_uint(y) & 0x80000000u) | 0x3F000000u);
    return __float2int_rz(__fmaf_rz(y, iv, h));
}

// Clamp of x to [-q, q] that keeps a NaN a NaN (min/max with the .NaN modifier).
__device__ __forceinline__ float clamp_keep_nan(float x, float q) {
    float d;
    asm("{\n\t.reg .f32 t;\n\tmax.NaN.f32 t, %1, %2;\n\tmin.NaN.f32 %0, t, %3;\n\t}" : "=f"(d) : "f"(x), "f"(-q), "f"(q));
    return d;
}

// code_of for values that may lie beyond the calibrated range (static scale): v is clamped to
// [-127, 127] before the truncation, so a code saturates at +-127 (truncation is monotone). When the
// static reciprocal 127/m overflowed to infinity (a calibrated maximum below 127 / FLT_MAX), a zero
// value gives 0 * inf = NaN: the clamp keeps it and the conversion turns a NaN into the code 0.
__device__ __forceinline__ int code_of_clamped(float y, float iv) {
    const float h = __uint_as_float((__float_as_uint(y) & 0x80000000u) | 0x3F000000u);
    return __float2int_rz(clamp_keep_nan(__fmaf_rz(y, iv, h), kQmax));
}

// Four INT8 codes in one word, q0 in the low byte (saturating packs of two values each).
__device__ __forceinline__ uint32_t pack4_s8(int q0, int q1, int q2, int q3) {
    uint32_t t, d;
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(t) : "r"(q3), "r"(q2));
    asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q1), "r"(q0), "r"(t));
    return d;
}

// E4M3 codes of two values (round to nearest, ties to even, saturating at +-448, the sign kept on a
// zero): the first value's code in the low byte.
__device__ __forceinline__ uint32_t f8codes2(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// LayerNorm parameters of vector v (8 columns) as binary32 pairs: g from the shared-memory table,
// b from its shared-memory table (BTAB) or else from global memory (nullable: zeros).
template <bool BTAB>
__device__ __forceinline__ void ln_params(const float4 *c_lo, const float4 *c_hi, const float *b, int v,
                                          uint64_t (&g2)[4], uint64_t (&b2)[4]) {
    const float4 gl = c_lo[v], gh = c_hi[v];
    g2[0] = pack2(gl.x, gl.y); g2[1] = pack2(gl.z, gl.w); g2[2] = pack2(gh.x, gh.y); g2[3] = pack2(gh.z, gh.w);
    float4 bl = make_float4(0.f, 0.f, 0.f, 0.f), bh = bl;
    if (BTAB) {
        const int nvec = static_cast<int>(c_hi - c_lo);
        bl = c_hi[nvec + v];
        bh = c_hi[2 * nvec + v];
    } else if (b != nullptr) {
        bl = __ldg(reinterpret_cast<const float4 *>(b) + 2 * v);
        bh = __ldg(reinterpret_cast<const float4 *>(b) + 2 * v + 1);
    }
    b2[0] = pack2(bl.x, bl.y); b2[1] = pack2(bl.z, bl.w); b2[2] = pack2(bh.x, bh.y); b2[3] = pack2(bh.z, bh.w);
}

// y = fl(fl(fl(c * ir) * g) + b) with c = fl(x - m), for the two bf16 values x of `w` (nm2 = {-m, -m}).
// The bias goes in with scalar adds (add2_scalar): a packed add here was contracted with the
// multiply before it, which rounds y once instead of twice.
__device__ __forceinline__ uint64_t ln_y2(uint32_t w, uint64_t nm2, uint64_t ir2, uint64_t g2, uint64_t b2) {
    return add2_scalar(mul2_rn(mul2_rn(add2_rn(bf2_to_f2(w), nm2), ir2), g2), b2);
}

// 3-input maximum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Column vector v of a row lies inside it. A FULL geometry covers the row exactly, so the bound holds
// by construction there; the checked build verifies it.
#ifdef SQ_DEVICE_CHECKS
#define SQ_COL_IN(v) (FULL ? SQ_CHECK((v) < nvec, p.status) : (v) < nvec)
#else
#define SQ_COL_IN(v) (FULL || (v) < nvec)
#endif

// One CTA = 16 warps in row groups of WPR warps. A group processes units of R consecutive rows; lane l
// of warp w of the group covers the 8-element vectors v = i * 32 * WPR + 32 * w + l (i < VPL) of
// every row of the unit. R > 1 only with WPR == 1.
// The body of a row kernel: this CTA is number `cta` of the `nctas` CTAs that share problem p.
template <int WPR, int VPL, int R, int MODE, bool NORM, bool FULL>
__device__ __forceinline__ void rows_body(const RowArgs p, unsigned cta, unsigned nctas)
{
    constexpr int G = kWarps / WPR;   // row groups per CTA
    constexpr int GT = 32 * WPR;      // consumer threads per row group
    constexpr int SUB = 32 / R;       // lanes that hold one row's total after a butterfly
    static_assert(R >= 1 && R <= 8 && VPL * R <= 8, "a unit gives a lane at most 64 element-rows");
    constexpr bool LN = MODE == MODE_QLN || MODE == MODE_ALN;       // LayerNorm: mean removed, bias added
    constexpr bool ABS = MODE == MODE_ABSMAX || MODE == MODE_ALN;   // column abs-max: rows re-read from the slot
    static_assert(!LN || NORM, "the LayerNorm modes normalise");
    // LayerNorm with groups of up to four warps (rows of up to 8192 elements, and the column abs-max over
    // few rows): the bias b gets a shared-memory table beside the one of g; eight-warp groups (16384
    // elements) read it from global memory, since both tables and a ring of two slots per group would not
    // fit. At 8192 elements the table leaves the ring two slots instead of three and still measured
    // 17 % faster (16384 x 8192 in CUDA graphs of 8 calls: 131.8 against 159.6 us per call).
    constexpr bool BTAB = LN && WPR <= 4;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t s_full[G * kMaxStages];
    __shared__ double s_ss[2][kWarps][R];
    __shared__ double s_ss2[LN ? 2 : 1][kWarps][LN ? R : 1];   // LayerNorm: the centred sums of squares
    __shared__ float s_mx[2][kWarps][R];
    __shared__ int s_abort[G];
    // Column abs-max over multi-warp groups: the last warp of a group to finish reading a slot refills it
    // (s_done counts the group's warps per slot; s_issued counts the group's issued units).
    constexpr bool LAST_REFILLS = ABS && WPR > 1;
    __shared__ int s_done[LAST_REFILLS ? G * kMaxStages : 1];
    __shared__ int s_issued[G];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int group = warp / WPR;
    const int wig = warp % WPR, gtid = wig * 32 + lane;
    const bool leader = gtid == 0;
    const int K = p.K, nvec = K >> 3;
    const uint32_t rowbytes = static_cast<uint32_t>(K) * 2u;
    const uint32_t slotbytes = rowbytes * R;
    const int stages = p.stages;
    uint8_t *ring = smem;
    const size_t ring_bytes = static_cast<size_t>(G) * stages * slotbytes;
    const size_t red_bytes = ABS ? static_cast<size_t>(G) * K * 4 : 0;
    float4 *c_lo = reinterpret_cast<float4 *>(smem + (ring_bytes > red_bytes ? ring_bytes : red_bytes));   // c[8v .. 8v+3]
    float4 *c_hi = c_lo + nvec;                                                                              // c[8v+4 .. 8v+7]
    const bool has_vec = p.vec != nullptr;
    float sdelta = 0.0f, sinv = 0.0f;

    const int64_t units = (p.rows + R - 1) / R;
    // first unit of this group; the group then takes every gstride-th unit
    const int64_t g0 = p.group_major ? static_cast<int64_t>(group) * nctas + cta : static_cast<int64_t>(cta) * G + group;
    const int64_t gstride = static_cast<int64_t>(nctas) * G;
    const int64_t nunits = g0 < units ? (units - 1 - g0) / gstride + 1 : 0;

    if (tid == 0) {
        for (int i = 0; i < G * stages; ++i) mbar_init(smem_u32(&s_full[i]), 1);
        for (int g = 0; g < G; ++g) { s_abort[g] = 0; s_issued[g] = 0; }
        for (int i = 0; i < (LAST_REFILLS ? G * kMaxStages : 1); ++i) s_done[i] = 0;
        mbar_init_fence();
    }
    // Dependent launch: everything above touched shared memory only. After the library's own
    // zero-fill (early) every earlier grid is already complete, so the rows can stream at once and
    // only amax waits for the fill (below).
    if (!(ABS && p.early)) pdl_wait();
    pdl_trigger();
    if (MODE == MODE_QSTATIC) {
        // the static scale is written by the kernel before this one (after the wait: never stale)
        sdelta = __ldg(p.scale2);
        sinv = __ldg(p.scale2 + 1);
    }
    if (MODE != MODE_ABSMAX && has_vec) {
        const float4 *cv = reinterpret_cast<const float4 *>(p.vec);
        for (int v = tid; v < nvec; v += kThreads) { c_lo[v] = __ldg(cv + 2 * v); c_hi[v] = __ldg(cv + 2 * v + 1); }
    }
    if (BTAB) {   // b table: b[8v .. 8v+3] at c_hi[nvec + v], b[8v+4 .. 8v+7] at c_hi[2 nvec + v] (absent: zeros)
        const float4 *bv = reinterpret_cast<const float4 *>(p.vec2);
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int v = tid; v < nvec; v += kThreads) {
            c_hi[nvec + v] = bv != nullptr ? __ldg(bv + 2 * v) : z;
            c_hi[2 * nvec + v] = bv != nullptr ? __ldg(bv + 2 * v + 1) : z;
        }
    }
    __syncthreads();

    auto slot = [&](int st) { return ring + (static_cast<size_t>(group) * stages + st) * slotbytes; };
    auto full_bar = [&](int st) { return smem_u32(&s_full[group * stages + st]); };
    volatile int *abort_flag = &s_abort[group];
    // Leader only: the copies of unit j (nr rows) into slot st, counted on its full barrier.
    const uint64_t policy = l2_evict_first_policy();
    auto issue = [&](int64_t j, int st) {
        const int64_t r0 = (g0 + j * gstride) * R;
        const int nr = static_cast<int>(p.rows - r0 < R ? p.rows - r0 : R);
        mbar_expect_tx(full_bar(st), rowbytes * static_cast<uint32_t>(nr));
        // one copy for the whole unit when its rows are contiguous, else one per row
        const bool packed = p.ld_bytes == static_cast<int64_t>(rowbytes);
        const int ncopies = packed ? 1 : nr;
        const uint32_t bytes = packed ? rowbytes * static_cast<uint32_t>(nr) : rowbytes;
        for (int r = 0; r < ncopies; ++r) {
            // the copy lands inside the slot and reads rows of the input only
            if (!SQ_CHECK(st >= 0 && st < stages && r0 >= 0 && nr >= 1 && r0 + nr <= p.rows &&
                              static_cast<uint64_t>(r) * rowbytes + bytes <= slotbytes, p.status))
                continue;
            const uint32_t dst = smem_u32(slot(st) + r * rowbytes);
            const uint8_t *src = p.src + (r0 + r) * p.ld_bytes;
            if (p.stream_once) bulk_g2s_hint(dst, src, bytes, full_bar(st), policy);
            else bulk_g2s(dst, src, bytes, full_bar(st));
        }
    };

    float mx[VPL][8];          // ABSMAX with norm: running max of fl(|x| * inv_rms) per column
    uint32_t mh[VPL][4];       // ABSMAX without norm: running max of |x| as bf16 pairs
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[i][e] = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) mh[i][k] = 0u;
    }

    int64_t issued = 0, consumed = 0;
    bool failed = false;
    if (leader) {
        issued = nunits < stages ? nunits : stages;
        for (int64_t j = 0; j < issued; ++j) issue(j, static_cast<int>(j));
        if (LAST_REFILLS) atomicMax(&s_issued[group], static_cast<int>(issued));
    }
    // Leader only, after the group's last read of slot st (unit j): refill it with unit j + stages.
    auto refill = [&](int64_t j, int st) {
        if (j + stages < nunits && !*abort_flag) {
            fence_proxy_async_smem();
            issue(j + stages, st);
            issued = j + stages + 1;
            if (LAST_REFILLS) atomicMax(&s_issued[group], static_cast<int>(issued));
        }
    };
    {
        int st = 0;
        uint32_t phase = 0;
        const int rv = static_cast<int>(rowbytes / 16);   // vectors per row in a slot
        for (int64_t j = 0; j < nunits; ++j) {
            const bool ok = mbar_ready(full_bar(st), phase, p.limit_ns, abort_flag);
            const int64_t r0 = (g0 + j * gstride) * R;
            const int nr = static_cast<int>(p.rows - r0 < R ? p.rows - r0 : R);   // uniform in the group
            const uint4 *rp = reinterpret_cast<const uint4 *>(slot(st));
            // A failed wait anywhere in the group stops the whole group at the same unit (a warp
            // of a wider group learns it at the group step below, after reading a stale slot).
            if (WPR == 1 && __any_sync(kAll, !ok)) {
                if (leader) { if (!*abort_flag) failed = true; *abort_flag = 1; }
                break;
            }

            // ---- pass A: the unit's rows into registers (QUANT) and the sums of squares (NORM)
            uint4 xr[R][VPL];
            double ssr[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int v = i * GT + gtid;
                    const bool in = SQ_COL_IN(v) && r < nr;
                    if (MODE == MODE_ABSMAX && !NORM) continue;
                    const uint4 q = in ? rp[r * rv + v] : make_uint4(0u, 0u, 0u, 0u);
                    if (!ABS) xr[r][i] = q;
                    if (LN) {                                   // the row sums of x (absent: zeros)
                        if (i & 1) { add_values(q.x, a2, a3); add_values(q.y, a2, a3); add_values(q.z, a2, a3); add_values(q.w, a2, a3); }
                        else { add_values(q.x, a0, a1); add_values(q.y, a0, a1); add_values(q.z, a0, a1); add_values(q.w, a0, a1); }
                    } else if (NORM) {
                        if (i & 1) { add_squares<MODE == MODE_ABSMAX>(q.x, a2, a3); add_squares<MODE == MODE_ABSMAX>(q.y, a2, a3); add_squares<MODE == MODE_ABSMAX>(q.z, a2, a3); add_squares<MODE == MODE_ABSMAX>(q.w, a2, a3); }
                        else { add_squares<MODE == MODE_ABSMAX>(q.x, a0, a1); add_squares<MODE == MODE_ABSMAX>(q.y, a0, a1); add_squares<MODE == MODE_ABSMAX>(q.z, a0, a1); add_squares<MODE == MODE_ABSMAX>(q.w, a0, a1); }
                    }
                }
                ssr[r] = (a0 + a1) + (a2 + a3);
            }
            if (WPR > 1) {
                // Group step, the one barrier of the unit for abs-max: partial sums become visible,
                // failures propagate, and (quantiser) every warp holds the unit in registers, so its
                // slot can be refilled. The abs-max re-reads the slot; its last warp refills it.
                if (NORM) {
                    const double part = rows_sum<R>(ssr, lane);   // row lane / SUB, this warp's columns
                    if (lane % SUB == 0) s_ss[j & 1][warp][lane / SUB] = part;
                }
                if (named_sync_or(1 + group, GT, !ok)) {
                    if (leader) { if (!*abort_flag) failed = true; *abort_flag = 1; }
                    break;
                }
                if (leader && !ABS) refill(j, st);      // the unit is in registers: its slot is free
            } else if (!ABS) {
                __syncwarp();                                   // the unit is in registers now
                if (leader) refill(j, st);
            }

            // ---- 1 / rms (LayerNorm: the mean, then 1 / standard deviation) of every row of the
            // unit, broadcast to all lanes
            float ir[R];
            float mu[R];
            if (NORM) {
                double ss;
                if (WPR > 1) {
                    ss = 0.0;
#pragma unroll
                    for (int w = 0; w < WPR; ++w) ss += s_ss[j & 1][group * WPR + w][lane / SUB];
                } else {
                    ss = rows_sum<R>(ssr, lane);                // total of row lane / SUB
                }
                if (LN) {
                    // ss is the row's sum of x: its mean, then the scaled sum of the squares of
                    // c = fl(x - mean) (a second group step when the row spans several warps)
                    const float mean = __double2float_rn(p.inv_k != 0.0 ? __dmul_rn(ss, p.inv_k)
                                                                        : __ddiv_rn(ss, static_cast<double>(K)));
#pragma unroll
                    for (int r = 0; r < R; ++r) mu[r] = __shfl_sync(kAll, mean, r * SUB);
                    double sq2[R];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint64_t nm2 = pack2(-mu[r], -mu[r]);
                        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
#pragma unroll
                        for (int i = 0; i < VPL; ++i) {
                            const int v = i * GT + gtid;
                            if (!(SQ_COL_IN(v) && r < nr)) continue;
                            const uint4 q = ABS ? rp[r * rv + v] : xr[r][i];
                            if (i & 1) { add_centred_squares(q.x, nm2, a2, a3); add_centred_squares(q.y, nm2, a2, a3); add_centred_squares(q.z, nm2, a2, a3); add_centred_squares(q.w, nm2, a2, a3); }
                            else { add_centred_squares(q.x, nm2, a0, a1); add_centred_squares(q.y, nm2, a0, a1); add_centred_squares(q.z, nm2, a0, a1); add_centred_squares(q.w, nm2, a0, a1); }
                        }
                        sq2[r] = (a0 + a1) + (a2 + a3);
                    }
                    if (WPR > 1) {
                        const double part = rows_sum<R>(sq2, lane);
                        if (lane % SUB == 0) s_ss2[j & 1][warp][lane / SUB] = part;
                        named_sync(1 + group, GT);
                        ss = 0.0;
#pragma unroll
                        for (int w = 0; w < WPR; ++w) ss += s_ss2[j & 1][group * WPR + w][lane / SUB];
                    } else {
                        ss = rows_sum<R>(sq2, lane);
                    }
                }
                const float mine = inv_rms(__dmul_rn(ss, 0x1p822), K, p.inv_k, p.eps);
#pragma unroll
                for (int r = 0; r < R; ++r) ir[r] = __shfl_sync(kAll, mine, r * SUB);
            } else {
#pragma unroll
                for (int r = 0; r < R; ++r) ir[r] = 1.0f;
            }

            if (ABS) {
                // ---- pass B: running column maxima
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int v = i * GT + gtid;
                    uint64_t g2[4], b2[4];                      // LayerNorm: gamma and beta pairs
                    if (LN && SQ_COL_IN(v)) ln_params<BTAB>(c_lo, c_hi, p.vec2, v, g2, b2);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        if (!(SQ_COL_IN(v) && r < nr)) continue;
                        if (LN) {
                            const uint64_t ir2 = pack2(ir[r], ir[r]), nm2 = pack2(-mu[r], -mu[r]);
                            const uint4 q = rp[r * rv + v];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                uint32_t l, h;
                                unpack2(ln_y2(word_of(q, k), nm2, ir2, g2[k], b2[k]), l, h);
                                mx[i][2 * k] = fmaxf(mx[i][2 * k], fabsf(__uint_as_float(l)));
                                mx[i][2 * k + 1] = fmaxf(mx[i][2 * k + 1], fabsf(__uint_as_float(h)));
                            }
                        } else if (NORM) {
                            const uint64_t ir2 = pack2(ir[r], ir[r]);
                            const uint4 q = rp[r * rv + v];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                uint32_t l, h;
                                unpack2(mul2_rn(bf2_to_f2(word_of(q, k)), ir2), l, h);
                                mx[i][2 * k] = fmaxf(mx[i][2 * k], fabsf(__uint_as_float(l)));
                                mx[i][2 * k + 1] = fmaxf(mx[i][2 * k + 1], fabsf(__uint_as_float(h)));
                            }
                        } else {
                            const uint4 q = rp[r * rv + v];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                __nv_bfloat162 cur = *reinterpret_cast<__nv_bfloat162 *>(&mh[i][k]);
                                const uint32_t a = word_of(q, k) & 0x7FFF7FFFu;
                                cur = __hmax2(cur, *reinterpret_cast<const __nv_bfloat162 *>(&a));
                                mh[i][k] = *reinterpret_cast<uint32_t *>(&cur);
                            }
                        }
                    }
                }
                // this warp is done with the slot: a single warp refills it; in a wider group the last of
                // its warps to get here does (the count orders every warp's reads before the copy)
                __syncwarp();
                if (WPR == 1) {
                    if (leader) refill(j, st);
                } else if (lane == 0) {
                    if (atomicAdd(&s_done[group * kMaxStages + st], 1) == WPR - 1) {
                        s_done[group * kMaxStages + st] = 0;
                        refill(j, st);
                    }
                }
            } else if (MODE == MODE_QSTATIC) {
                // ---- one pass: y = (x * inv_rms) * c (or x * c, or x), coded with the static scale
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (r < nr) {
                        uint2 *qrow = reinterpret_cast<uint2 *>(p.q + (r0 + r) * static_cast<int64_t>(K));
#pragma unroll
                        for (int i = 0; i < VPL; ++i) {
                            const int v = i * GT + gtid;
                            if (!SQ_COL_IN(v)) continue;
                            float4 cl = make_float4(1.f, 1.f, 1.f, 1.f), ch = cl;
                            if (has_vec) { cl = c_lo[v]; ch = c_hi[v]; }
                            const float cf[8] = {cl.x, cl.y, cl.z, cl.w, ch.x, ch.y, ch.z, ch.w};
                            int q[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const uint32_t w = word_of(xr[r][i], e >> 1);
                                const float x = __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
                                const float y = NORM ? __fmul_rn(__fmul_rn(x, ir[r]), cf[e]) : (has_vec ? __fmul_rn(x, cf[e]) : x);
                                q[e] = code_of_clamped(y, sinv);
                            }
                            if (SQ_CHECK(r0 + r < p.rows, p.status))
                                qrow[v] = make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
                        }
                    }
                }
                if (gtid == 0) {
#pragma unroll
                    for (int r = 0; r < R; ++r)
                        if (r < nr && SQ_CHECK(r0 + r < p.rows, p.status)) p.scale[r0 + r] = sdelta;
                }
            } else {
                // ---- pass B: y = (x * inv_rms) * c  (or x * c, or x; LayerNorm: its own form), row maxima.
                // Binary32 scalars: each value is rounded exactly as the definition orders it.
                float yv[R][VPL][8];
                float m[R];
#pragma unroll
                for (int r = 0; r < R; ++r) m[r] = 0.0f;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int v = i * GT + gtid;
                    const bool in = SQ_COL_IN(v);
                    float4 cl = make_float4(1.f, 1.f, 1.f, 1.f), ch = cl;
                    if (has_vec && in) { cl = c_lo[v]; ch = c_hi[v]; }
                    const float cf[8] = {cl.x, cl.y, cl.z, cl.w, ch.x, ch.y, ch.z, ch.w};
                    uint64_t g2[4], b2[4];                      // LayerNorm: gamma and beta pairs
                    if (LN && in) ln_params<BTAB>(c_lo, c_hi, p.vec2, v, g2, b2);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t w = word_of(xr[r][i], k);
                            float yl, yh;
                            if (LN) {
                                // an absent vector must not reach the row maximum (its y is not 0)
                                uint32_t l = 0u, h = 0u;
                                if (in) unpack2(ln_y2(w, pack2(-mu[r], -mu[r]), pack2(ir[r], ir[r]), g2[k], b2[k]), l, h);
                                yl = __uint_as_float(l);
                                yh = __uint_as_float(h);
                            } else {
                                const float xl = __uint_as_float(w << 16), xh = __uint_as_float(w & 0xFFFF0000u);
                                yl = NORM ? __fmul_rn(__fmul_rn(xl, ir[r]), cf[2 * k]) : (has_vec ? __fmul_rn(xl, cf[2 * k]) : xl);
                                yh = NORM ? __fmul_rn(__fmul_rn(xh, ir[r]), cf[2 * k + 1]) : (has_vec ? __fmul_rn(xh, cf[2 * k + 1]) : xh);
                            }
                            yv[r][i][2 * k] = yl;
                            yv[r][i][2 * k + 1] = yh;
                            m[r] = max3f(m[r], fabsf(yl), fabsf(yh));
                        }
                    }
                }
                float mrow = rows_max<R>(m, lane);               // maximum of row lane / SUB
                if (WPR > 1) {
                    if (lane % SUB == 0) s_mx[j & 1][warp][lane / SUB] = mrow;
                    named_sync(1 + group, GT);
                    mrow = 0.0f;
#pragma unroll
                    for (int w = 0; w < WPR; ++w) mrow = fmaxf(mrow, s_mx[j & 1][group * WPR + w][lane / SUB]);
                }
                // step and reciprocal of the row this lane holds; one lane per row stores the step
                constexpr float qmax = MODE == MODE_QF8 ? kF8Max : kQmax;
                const float delta = mrow > 0.0f ? __fdiv_rn(mrow, qmax) : 0.0f;
                float inv_m = mrow > 0.0f ? __fdiv_rn(qmax, mrow) : 0.0f;
                // A row maximum below qmax / FLT_MAX (about 3.7e-37 for INT8): qmax / m overflows binary32.
                // Such a row is scaled by 2^64 first (exact: its values are far below the top of the
                // range) and coded with fl(qmax / fl(m * 2^64)); the step stays m / qmax.
                const bool tiny = isinf(inv_m);
                if (tiny) inv_m = __fdiv_rn(qmax, __fmul_rn(mrow, 0x1p64f));
                if (wig == 0 && (lane % SUB) == 0 && lane / SUB < nr && SQ_CHECK(r0 + lane / SUB < p.rows, p.status))
                    p.scale[r0 + lane / SUB] = delta;
                // ---- pass C: codes (INT8: round half away from zero of y * 127/m, exact product;
                // FP8: e4m3 of fl(y * 448/m))
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float iv = __shfl_sync(kAll, inv_m, r * SUB);
                    if (__shfl_sync(kAll, tiny ? 1 : 0, r * SUB) != 0) {      // uniform across the row's lanes
#pragma unroll
                        for (int i = 0; i < VPL; ++i)
#pragma unroll
                            for (int e = 0; e < 8; ++e) yv[r][i][e] = __fmul_rn(yv[r][i][e], 0x1p64f);
                    }
                    if (r < nr) {
                        uint2 *qrow = reinterpret_cast<uint2 *>(p.q + (r0 + r) * static_cast<int64_t>(K));
#pragma unroll
                        for (int i = 0; i < VPL; ++i) {
                            const int v = i * GT + gtid;
                            if (SQ_COL_IN(v)) {
                                uint2 out;
                                if (MODE == MODE_QF8) {
                                    uint32_t c[4];
#pragma unroll
                                    for (int k = 0; k < 4; ++k)
                                        c[k] = f8codes2(__fmul_rn(yv[r][i][2 * k], iv), __fmul_rn(yv[r][i][2 * k + 1], iv));
                                    out = make_uint2(__byte_perm(c[0], c[1], 0x5410), __byte_perm(c[2], c[3], 0x5410));
                                    if (iv == 0.0f) out = make_uint2(0u, 0u);   // a zero row: codes +0
                                } else {
                                    int q[8];
#pragma unroll
                                    for (int e = 0; e < 8; ++e) q[e] = code_of(yv[r][i][e], iv);
                                    out = make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
                                }
                                if (SQ_CHECK(r0 + r < p.rows, p.status)) qrow[v] = out;
                            }
                        }
                    }
                }
            }
            consumed = j + 1;
            if (++st == stages) { st = 0; phase ^= 1u; }
        }
    }

    if (failed) atomicCAS(p.status, 0u, static_cast<unsigned int>(SQ_ERR_TIMEOUT));
    // Copies issued but never consumed (only after a failed wait) must land before the CTA exits.
    if (leader) {
        if (LAST_REFILLS) issued = s_issued[group];   // refills of the group's other warps included
        for (int64_t j = consumed; j < issued; ++j)
            if (!mbar_wait(full_bar(static_cast<int>(j % stages)), static_cast<uint32_t>((j / stages) & 1), p.limit_ns, nullptr))
                atomicCAS(p.status, 0u, static_cast<unsigned int>(SQ_ERR_TIMEOUT));
    }
    __syncthreads();

    if (ABS) {
        __syncthreads();                                   // the ring is idle: reuse it
        float *red = reinterpret_cast<float *>(smem);      // [G][K]
        {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int v = i * GT + gtid;
                if (SQ_COL_IN(v)) {
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
            if (NORM && !LN) m = __fmul_rn(m, fabsf(__ldg(p.vec + c)));
            red[c] = m;
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        if (p.early) pdl_wait();                           // the zero-fill of amax is complete
        const int csize = static_cast<int>(cluster.num_blocks());
        const int share = (K + csize - 1) / csize;
        const int c0 = static_cast<int>(cluster.block_rank()) * share;
        const int c1 = min(K, c0 + share);
        for (int c = c0 + tid; c < c1; c += kThreads) {
            float m = 0.0f;
            for (int q = 0; q < csize; ++q) m = fmaxf(m, cluster.map_shared_rank(red, q)[c]);
            // abs-maxima are non-negative, where IEEE order equals unsigned integer order
            if (m > 0.0f && SQ_CHECK(c >= 0 && c < K, p.status))
                atomicMax(reinterpret_cast<unsigned int *>(p.amax + c), __float_as_uint(m));
        }
        cluster.sync();
    }
}

template <int WPR, int VPL, int R, int MODE, bool NORM, bool FULL>
__global__ void __launch_bounds__(kThreads, 1) k_rows(const RowArgs p)
{
    rows_body<WPR, VPL, R, MODE, NORM, FULL>(p, blockIdx.x, gridDim.x);
}

// Column abs-maxima of two inputs with the same row length in one launch: CTAs [0, ctas_a) reduce the
// rows of pa (their RMSNorm output when NORM_A), the others the plain rows of pw (a weight). The split
// lies on a cluster boundary, so the cross-CTA reduction of every cluster stays within one input.
template <int WPR, int VPL, int R, bool NORM_A, bool FULL>
__global__ void __launch_bounds__(kThreads, 1) k_absmax_pair(const RowArgs pa, const RowArgs pw, unsigned ctas_a)
{
    if (blockIdx.x < ctas_a) rows_body<WPR, VPL, R, MODE_ABSMAX, NORM_A, FULL>(pa, blockIdx.x, ctas_a);
    else rows_body<WPR, VPL, R, MODE_ABSMAX, false, FULL>(pw, blockIdx.x - ctas_a, gridDim.x - ctas_a);
}

// Zero-fill of two arrays in one launch (the running maxima of k_absmax_pair); waits for the
// previous work of the stream, then lets the next kernel start.
__global__ void k_fill_zero2(float *__restrict__ p, int64_t n, float *__restrict__ q, int64_t m) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n + m;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (i < n) p[i] = 0.0f;
        else q[i - n] = 0.0f;
    }
}

__global__ void k_fill_zero(float *__restrict__ p, int64_t n) {
    pdl_wait();          // earlier grids complete before the next kernel may start (it reads early)
    pdl_trigger();
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = 0.0f;
}

// ---------------------------------------------------------------------------------------------
// Static per-tensor activation scale, [W8A8] "One layer, measured" (one scale per tensor from the
// calibration tokens' maximum): m = max_k fl(amax[k] * |f[k]|) (f null: max_k amax[k]); scale2 =
// {m / 127, 127 / m} (zeros when m == 0). One CTA: per-thread maxima, then warp and block maxima.
__global__ void k_static_scale(const float *__restrict__ amax, const float *__restrict__ f, int64_t K,
                               float *__restrict__ scale2)
{
    __shared__ float s_w[32];
    pdl_wait();
    pdl_trigger();
    float m = 0.0f;
    for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
        const float a = __ldg(amax + k);
        m = fmaxf(m, f != nullptr ? __fmul_rn(a, fabsf(__ldg(f + k))) : a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kAll, m, o));
    if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.0f;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t = fmaxf(t, s_w[w]);
        scale2[0] = t > 0.0f ? __fdiv_rn(t, kQmax) : 0.0f;
        scale2[1] = t > 0.0f ? __fdiv_rn(kQmax, t) : 0.0f;
    }
}

// Smoothing factors and fold, [MIGRATE] section 3 and [W8A8] "The trick: move the range into the
// weights": s = max|X|^alpha / max|W|^(1-alpha) in binary64, rounded once, floored at 1e-5;
// fold = gamma / s (or 1 / s).
__global__ void k_scales(const float *__restrict__ ax, const float *__restrict__ aw, int64_t K,
                         double ea, double eb, const float *__restrict__ gamma,
                         float *__restrict__ s, float *__restrict__ fold)
{
    pdl_wait();
    pdl_trigger();
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
    int wpr, vpl, rpu, groups;   // warps per row group, vectors per lane, rows per unit
};

// Dynamic shared memory of a launch with `stages` ring slots per group.
size_t rows_smem(int K, int mode, const Geo &g, int stages) {
    const size_t slotbytes = static_cast<size_t>(K) * 2 * g.rpu;
    // table of the per-column factor (quantisers, LayerNorm g); LayerNorm with groups of up to four warps
    // adds a table of its bias b (the kernel's BTAB)
    const bool btab = (mode == MODE_QLN || mode == MODE_ALN) && g.wpr <= 4;
    const size_t ctab = (mode != MODE_ABSMAX ? static_cast<size_t>(K) * 4 : 0) + (btab ? static_cast<size_t>(K) * 4 : 0);
    const size_t ring = static_cast<size_t>(g.groups) * stages * slotbytes;
    const size_t red = mode == MODE_ABSMAX || mode == MODE_ALN ? static_cast<size_t>(g.groups) * K * 4 : 0;
    return (ring > red ? ring : red) + ctab;
}

// A lane covers 8 vectors (64 elements) of a row, or of R rows of a narrow input.
Geo row_geo(int K) {
    const int nvec = K / 8;
    Geo g;
    // Rows of up to 2048 elements take one warp each (R = 8 / VPL rows per unit), wider rows a
    // group of 2, 4 or 8 warps with one row per unit. (Groups of 4 warps over 2-row units of
    // 4096-element rows gave larger copies but lost more to the wider group barrier.)
    g.wpr = nvec <= 256 ? 1 : nvec <= 512 ? 2 : nvec <= 1024 ? 4 : 8;
    const int per = (nvec + 32 * g.wpr - 1) / (32 * g.wpr);
    g.vpl = per <= 1 ? 1 : per <= 2 ? 2 : per <= 4 ? 4 : 8;
    g.rpu = 8 / g.vpl;
    g.groups = kWarps / g.wpr;
    return g;
}

template <int WPR, int VPL, int R, int MODE, bool NORM, bool FULL>
sq_status launch_rows_t(RowArgs a, const Geo &geo, int dev, cudaStream_t st) {
    auto kern = k_rows<WPR, VPL, R, MODE, NORM, FULL>;
    constexpr int G = kWarps / WPR;
    // The kernel's lanes cover exactly WPR * 32 * VPL vectors of a row (FULL: no per-vector bounds
    // checks), R rows per unit: the geometry must be the one it was compiled for.
    const int nvec = a.K / 8;
    if (geo.wpr != WPR || geo.vpl != VPL || geo.rpu != R || geo.groups != G || nvec > WPR * 32 * VPL ||
        (FULL && nvec != WPR * 32 * VPL))
        return sq::fail(SQ_ERR_UNSUPPORTED, "row kernel geometry mismatch (K=%d)", a.K);
    constexpr bool ABS = MODE == MODE_ABSMAX || MODE == MODE_ALN;   // column abs-max: cluster launch
    // Per-device launch configuration of this instantiation, set up on first use (guarded: calls may
    // come from several host threads).
    static std::mutex mu;
    static size_t configured_smem[64];
    static int per_sm[64];
    static int cluster_size[64], cluster_ctas[64];
    static size_t smem_cap[64];    // opt-in maximum minus this kernel's static shared memory
    std::unique_lock<std::mutex> lk(mu);
    if (smem_cap[dev] == 0) {
        int optin = 0;
        cudaFuncAttributes fa;
        cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return sq::cuda_status(e, "shared memory limits (rows)");
        smem_cap[dev] = static_cast<size_t>(optin) - fa.sharedSizeBytes;
    }
    // as many ring slots per group as fit (2 .. kMaxStages)
    int stages = kMaxStages;
    while (stages > 2 && rows_smem(a.K, MODE, geo, stages) > smem_cap[dev]) --stages;
    const size_t smem = rows_smem(a.K, MODE, geo, stages);
    if (smem > smem_cap[dev]) return sq::fail(SQ_ERR_UNSUPPORTED, "row kernel needs %zu bytes of shared memory", smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (configured_smem[dev] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaFuncSetAttribute(rows)");
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, smem);
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor(rows)");
        per_sm[dev] = nb > 0 ? nb : 1;
        if (ABS) {
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
        configured_smem[dev] = smem;
    }
    const int per_sm_d = per_sm[dev], csz = cluster_size[dev], cctas = cluster_ctas[dev];
    lk.unlock();
    const int64_t full = static_cast<int64_t>(sq::sm_count(dev)) * per_sm_d;
    a.stages = stages;
    a.inv_k = (a.K & (a.K - 1)) == 0 ? 1.0 / static_cast<double>(a.K) : 0.0;
    a.status = sq::device_status_word(dev);
    a.limit_ns = sq::wait_timeout_ns(dev);
    a.stream_once = static_cast<double>(a.rows) * static_cast<double>(a.ld_bytes) > 0.5 * sq::l2_bytes(dev) ? 1 : 0;
    if (a.status == nullptr) return sq::fail(SQ_ERR_CUDA, "device status word unavailable");
    const int64_t units = (a.rows + R - 1) / R;
    if (!ABS) {
        // Up to 4 units per row group: units are numbered group by group across the CTAs, so every SM
        // gets an equal share (CTA by CTA, 4096 rows on 148 x 8 groups give 68 SMs 32 rows and the
        // other 80 SMs 24), and below one unit per SM each unit gets an SM of its own. Measured in CUDA
        // graphs of 8 calls: weight quantiser 4096 x 4096, 12.3 us per call against 13.1; activation
        // quantiser 4096 x 4096, 14.6 against 15.1; 8 / 64 tokens of 4096, 3.6 / 3.8 against 3.9 /
        // 4.1. With more units per group the CTA-by-CTA numbering measured up to 3 % faster.
        a.group_major = units <= 4 * G * full ? 1 : 0;
        int64_t ctas = a.group_major ? units : (units + G - 1) / G;
        if (ctas > full) ctas = full;
        return sq::cuda_status(sq::launch_pdl(kern, dim3(static_cast<unsigned>(ctas)), dim3(kThreads), smem, st, nullptr, a),
                               "launch(rowquant)");
    }
    // one wave of resident clusters at most, at least ~4 units per group
    int64_t ctas = (units + 4 * G - 1) / (4 * G);
    if (ctas > cctas) ctas = cctas;
    ctas = ((ctas + csz - 1) / csz) * csz;
    attr[0].val.clusterDim.x = csz;
    return sq::cuda_status(sq::launch_pdl(kern, dim3(static_cast<unsigned>(ctas)), dim3(kThreads), smem, st, &attr[0], a),
                           "launch(absmax)");
}

template <int MODE, bool NORM, bool FULL>
sq_status dispatch_rows_f(const RowArgs &a, const Geo &g, int dev, cudaStream_t st) {
    if constexpr (MODE == MODE_ABSMAX || MODE == MODE_ALN) {
        if (g.wpr == 4 && g.vpl == 4) return launch_rows_t<4, 4, 1, MODE, NORM, FULL>(a, g, dev, st);
    } else {
        if (g.wpr == 8 && g.vpl == 2) return launch_rows_t<8, 2, 1, MODE, NORM, FULL>(a, g, dev, st);
        if (g.wpr == 8 && g.vpl == 4) return launch_rows_t<8, 4, 1, MODE, NORM, FULL>(a, g, dev, st);
    }
    if (g.wpr == 2) return launch_rows_t<2, 8, 1, MODE, NORM, FULL>(a, g, dev, st);
    if (g.wpr == 4) return launch_rows_t<4, 8, 1, MODE, NORM, FULL>(a, g, dev, st);
    if (g.wpr == 8) return launch_rows_t<8, 8, 1, MODE, NORM, FULL>(a, g, dev, st);
    switch (g.vpl) {
        case 1: return launch_rows_t<1, 1, 8, MODE, NORM, FULL>(a, g, dev, st);
        case 2: return launch_rows_t<1, 2, 4, MODE, NORM, FULL>(a, g, dev, st);
        case 4: return launch_rows_t<1, 4, 2, MODE, NORM, FULL>(a, g, dev, st);
        default: return launch_rows_t<1, 8, 1, MODE, NORM, FULL>(a, g, dev, st);
    }
}

// FULL: the row is exactly VPL vectors per lane of the group (no bounds checks per vector).
template <int MODE, bool NORM>
sq_status dispatch_rows(const RowArgs &a, int dev, cudaStream_t st) {
    Geo g = row_geo(a.K);
    // Column abs-max over few rows (e.g. a weight): with fewer than 16 rows per two-warp group, four-warp
    // groups (half the groups, each row over 128 lanes) finish sooner (measured on a 4096 x 4096 weight:
    // 17.4 us against 21.5 us).
    if ((MODE == MODE_ABSMAX || MODE == MODE_ALN) && g.wpr == 2 && a.rows < 16LL * 8 * sq::sm_count(dev)) {
        g.wpr = 4;
        g.vpl = g.vpl / 2 < 1 ? 1 : g.vpl / 2;
        g.rpu = 1;
        g.groups = kWarps / g.wpr;
    }
    // Quantisers over few rows (decode-sized token counts): one row per group of eight warps. A row's
    // serial work (binary64 sums, group reductions, codes) is spread over 256 lanes instead of 64 or
    // 128, and with at most 4 rows per SM the shorter chains win. Measured at K = 4096 in CUDA graphs
    // of 8 calls: 3.84 us per call against 5.64 us at 8 to 128 tokens, 5.64 against 6.13 at 512; from
    // about 1024 rows the two-warp groups win (6.40 against 8.72 us).
    if (MODE != MODE_ABSMAX && MODE != MODE_ALN && (g.wpr == 2 || g.wpr == 4) && a.rows <= 4LL * sq::sm_count(dev)) {
        const int nvec = a.K / 8;
        g.wpr = 8;
        g.vpl = nvec <= 512 ? 2 : 4;
        g.rpu = 1;
        g.groups = kWarps / g.wpr;
    }
    const bool full = (a.K / 8) == g.vpl * 32 * g.wpr;
    return full ? dispatch_rows_f<MODE, NORM, true>(a, g, dev, st) : dispatch_rows_f<MODE, NORM, false>(a, g, dev, st);
}

// Relative cost of a row of the plain abs-max against a row of the RMSNorm-fed one (same length): the
// plain rows only stream through the ring, the norm-fed ones are bound by their per-element work. On a
// B200, 4096-element rows: a CTA streams plain rows at ~82 GB/s and RMSNorm-fed rows at ~32 GB/s; a
// 65536 + 4096 row pair ran in 205.7 / 117.9 / 121.9 / 128.3 us with 2 / 4 / 8 / 16 weight CTAs, and
// 262144 + 28672 rows of 8192 elements took 910 us with 6 weight CTAs (the weight side the slower).
constexpr double kPlainRowCost = 0.4;

template <int WPR, int VPL, int R, bool NORM_A, bool FULL>
sq_status launch_pair_t(RowArgs a, RowArgs w, const Geo &geo, int dev, cudaStream_t st) {
    auto kern = k_absmax_pair<WPR, VPL, R, NORM_A, FULL>;
    constexpr int G = kWarps / WPR;
    const int nvec = a.K / 8;
    if (geo.wpr != WPR || geo.vpl != VPL || geo.rpu != R || geo.groups != G || nvec > WPR * 32 * VPL ||
        (FULL && nvec != WPR * 32 * VPL))
        return sq::fail(SQ_ERR_UNSUPPORTED, "row kernel geometry mismatch (K=%d)", a.K);
    static std::mutex mu;
    static size_t configured_smem[64];
    static int cluster_size[64], cluster_ctas[64];
    static size_t smem_cap[64];
    std::unique_lock<std::mutex> lk(mu);
    if (smem_cap[dev] == 0) {
        int optin = 0;
        cudaFuncAttributes fa;
        cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return sq::cuda_status(e, "shared memory limits (absmax pair)");
        smem_cap[dev] = static_cast<size_t>(optin) - fa.sharedSizeBytes;
    }
    int stages = kMaxStages;
    while (stages > 2 && rows_smem(a.K, MODE_ABSMAX, geo, stages) > smem_cap[dev]) --stages;
    const size_t smem = rows_smem(a.K, MODE_ABSMAX, geo, stages);
    if (smem > smem_cap[dev]) return sq::fail(SQ_ERR_UNSUPPORTED, "row kernel needs %zu bytes of shared memory", smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    if (configured_smem[dev] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaFuncSetAttribute(absmax pair)");
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // the cluster size that keeps the most CTAs resident at once (ties: the larger cluster)
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
        configured_smem[dev] = smem;
    }
    const int csz = cluster_size[dev], cctas = cluster_ctas[dev];
    lk.unlock();
    if (cctas < 2 * csz) return sq::fail(SQ_ERR_UNSUPPORTED, "fewer than two clusters fit for the abs-max pair");
    for (RowArgs *r : {&a, &w}) {
        r->stages = stages;
        r->inv_k = (r->K & (r->K - 1)) == 0 ? 1.0 / static_cast<double>(r->K) : 0.0;
        r->status = sq::device_status_word(dev);
        r->limit_ns = sq::wait_timeout_ns(dev);
        r->stream_once = static_cast<double>(r->rows) * static_cast<double>(r->ld_bytes) > 0.5 * sq::l2_bytes(dev) ? 1 : 0;
    }
    if (a.status == nullptr) return sq::fail(SQ_ERR_CUDA, "device status word unavailable");
    // CTAs per input: at most one per ~4 units per group, whole clusters, one wave in total; when both
    // do not fit, the wave is divided by the inputs' costs.
    auto want = [&](int64_t rows) {
        const int64_t units = (rows + R - 1) / R;
        const int64_t c = (units + 4 * G - 1) / (4 * G);
        return ((c + csz - 1) / csz) * csz;
    };
    const int64_t wa = want(a.rows), ww = want(w.rows);
    const int64_t wave = (cctas / csz) * csz;
    int64_t ca = wa, cw = ww;
    if (ca + cw > wave) {
        const double cost_a = static_cast<double>(a.rows);
        const double cost_w = (NORM_A ? kPlainRowCost : 1.0) * static_cast<double>(w.rows);
        // rounded up to whole clusters: a weight CTA too few slows the whole launch by the weight's
        // share of its rows, a CTA too many takes one of the many calibration CTAs
        int64_t share_w = static_cast<int64_t>(std::ceil(static_cast<double>(wave) * cost_w / (cost_a + cost_w) / csz)) * csz;
        share_w = share_w < csz ? csz : share_w > wave - csz ? wave - csz : share_w;
        cw = ww < share_w ? ww : share_w;
        ca = wa < wave - cw ? wa : wave - cw;
        cw = ww < wave - ca ? ww : wave - ca;      // CTAs the other input leaves unused
    }
    attr[0].val.clusterDim.x = csz;
    return sq::cuda_status(sq::launch_pdl(kern, dim3(static_cast<unsigned>(ca + cw)), dim3(kThreads), smem, st, &attr[0], a, w,
                                          static_cast<unsigned>(ca)),
                           "launch(absmax pair)");
}

// The one-launch form covers rows of more than 2048 elements (one row per unit); false when the
// geometry has none, and the caller then launches the two reductions one after the other.
template <bool NORM_A>
bool dispatch_pair(const RowArgs &a, const RowArgs &w, int dev, cudaStream_t st, sq_status *out) {
    const Geo g = row_geo(a.K);
    if (g.wpr < 2) return false;
    const bool full = (a.K / 8) == g.vpl * 32 * g.wpr;
    switch (g.wpr) {
        case 2: *out = full ? launch_pair_t<2, 8, 1, NORM_A, true>(a, w, g, dev, st) : launch_pair_t<2, 8, 1, NORM_A, false>(a, w, g, dev, st); break;
        case 4: *out = full ? launch_pair_t<4, 8, 1, NORM_A, true>(a, w, g, dev, st) : launch_pair_t<4, 8, 1, NORM_A, false>(a, w, g, dev, st); break;
        default: *out = full ? launch_pair_t<8, 8, 1, NORM_A, true>(a, w, g, dev, st) : launch_pair_t<8, 8, 1, NORM_A, false>(a, w, g, dev, st); break;
    }
    return true;
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
        sq_status s0 = sq::cuda_status(
            sq::launch_pdl(k_fill_zero, dim3(static_cast<unsigned>((cols + 255) / 256)), dim3(256), 0, st, nullptr, amax, cols),
            "launch(fill)");
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
    ra.early = accumulate ? 0 : 1;   // the zero-fill above was the stream's last kernel
    return norm_gamma ? dispatch_rows<MODE_ABSMAX, true>(ra, dev, st) : dispatch_rows<MODE_ABSMAX, false>(ra, dev, st);
}

// Arguments of one input of sq_calibrate_absmax_pair, checked as sq_calibrate_absmax checks them.
static sq_status check_absmax_input(const char *fn, const char *name, const void *a, int64_t rows, int64_t cols,
                                    int64_t ld, const float *amax) {
    using sq::fail;
    if (!amax) return fail(SQ_ERR_INVALID_ARG, "%s: the maxima of %s are NULL", fn, name);
    if (rows < 0 || cols < 8 || ld < cols)
        return fail(SQ_ERR_INVALID_ARG, "%s: need rows >= 0, cols >= 8, ld >= cols for %s (rows=%lld cols=%lld ld=%lld)",
                    fn, name, (long long)rows, (long long)cols, (long long)ld);
    if (rows > 0 && !a) return fail(SQ_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);
    if (cols % 8 != 0 || ld % 8 != 0) return fail(SQ_ERR_MISALIGNED, "%s: cols and the ld of %s must be multiples of 8", fn, name);
    if ((a && !sq::aligned(a, 16)) || !sq::aligned(amax, 4))
        return fail(SQ_ERR_MISALIGNED, "%s: %s must be 16-byte aligned and its maxima 4-byte aligned", fn, name);
    if (cols > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "%s: cols must be <= %d", fn, kMaxK);
    return SQ_OK;
}

// The activation and weight maxima of one smoothing group (the two per-channel maxima that the
// smoothing factor of [MIGRATE] section 3 combines) in one launch. The two reductions are
// independent; sharing the launch saves the second one's start-up and end phase.
sq_status sq_calibrate_absmax_pair(const void *a, int64_t rows, int64_t cols, int64_t ld, const float *norm_gamma,
                                   float eps, float *amax, const void *w, int64_t w_rows, int64_t w_ld, float *amax_w,
                                   int accumulate, void *stream)
{
    using sq::fail;
    const char *fn = "sq_calibrate_absmax_pair";
    sq_status c = check_absmax_input(fn, "a", a, rows, cols, ld, amax);
    if (c == SQ_OK) c = check_absmax_input(fn, "w", w, w_rows, cols, w_ld, amax_w);
    if (c != SQ_OK) return c;
    if (norm_gamma && !sq::aligned(norm_gamma, 16)) return fail(SQ_ERR_MISALIGNED, "%s: norm_gamma must be 16-byte aligned", fn);
    if (amax < amax_w + cols && amax_w < amax + cols)
        return fail(SQ_ERR_INVALID_ARG, "%s: amax and amax_w must not overlap", fn);
    int dev = 0;
    SQ_TRY_ARCH(dev);
    cudaStream_t st = sq::as_stream(stream);
    if (!accumulate) {
        const int64_t n = 2 * cols;
        sq_status s0 = sq::cuda_status(sq::launch_pdl(k_fill_zero2, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0,
                                                      st, nullptr, amax, cols, amax_w, cols),
                                       "launch(fill)");
        if (s0 != SQ_OK) return s0;
    }
    RowArgs ra = {};
    ra.src = static_cast<const uint8_t *>(a);
    ra.rows = rows;
    ra.ld_bytes = ld * 2;
    ra.K = static_cast<int>(cols);
    ra.vec = norm_gamma;
    ra.eps = eps;
    ra.amax = amax;
    ra.early = accumulate ? 0 : 1;   // the zero-fill above was the stream's last kernel
    RowArgs rw = ra;
    rw.src = static_cast<const uint8_t *>(w);
    rw.rows = w_rows;
    rw.ld_bytes = w_ld * 2;
    rw.vec = nullptr;
    rw.amax = amax_w;
    if (rows > 0 && w_rows > 0) {
        sq_status out = SQ_OK;
        if (norm_gamma ? dispatch_pair<true>(ra, rw, dev, st, &out) : dispatch_pair<false>(ra, rw, dev, st, &out)) return out;
    }
    // one input empty, or rows of at most 2048 elements: the two reductions one after the other (the
    // second reads its rows only after the first has finished)
    if (rows > 0) {
        const sq_status s1 = norm_gamma ? dispatch_rows<MODE_ABSMAX, true>(ra, dev, st) : dispatch_rows<MODE_ABSMAX, false>(ra, dev, st);
        if (s1 != SQ_OK) return s1;
        rw.early = 0;
    }
    if (w_rows > 0) return dispatch_rows<MODE_ABSMAX, false>(rw, dev, st);
    return SQ_OK;
}

// LayerNorm-fed layers ([WOVS] "SmoothQuant: Weight-Only vs W8A8", "Integration with
// Transformers": S^-1 folded into the LayerNorm's gamma and beta). LayerNorm in the standard form,
// each step rounded as listed: m = fl32(sum x / K) and ms = fl32(sum c^2 / K) with binary64 sums,
// c = fl32(x - m), ir = fl32(1 / fl32(sqrt(fl32(ms + eps)))), y = fl32(fl32(fl32(c * ir) * g) + b).
// The sum of x is exact unless a row's nonzero magnitudes span more than about 2^31; both binary64
// sums are taken in a tree order, which can differ from another order only by binary64 roundings.
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
    if (cols > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_calibrate_absmax_layernorm: cols must be <= %d", kMaxK);
    int dev = 0;
    SQ_TRY_ARCH(dev);
    cudaStream_t st = sq::as_stream(stream);
    if (!accumulate) {
        sq_status s0 = sq::cuda_status(
            sq::launch_pdl(k_fill_zero, dim3(static_cast<unsigned>((cols + 255) / 256)), dim3(256), 0, st, nullptr, amax, cols),
            "launch(fill)");
        if (s0 != SQ_OK) return s0;
    }
    if (rows == 0) return SQ_OK;
    RowArgs ra = {};
    ra.src = static_cast<const uint8_t *>(a);
    ra.rows = rows;
    ra.ld_bytes = ld * 2;
    ra.K = static_cast<int>(cols);
    ra.vec = gamma;
    ra.vec2 = beta;
    ra.eps = eps;
    ra.amax = amax;
    ra.early = accumulate ? 0 : 1;   // the zero-fill above was the stream's last kernel
    return dispatch_rows<MODE_ALN, true>(ra, dev, st);
}

sq_status sq_layernorm_smooth_quant(const void *x, int64_t T, int64_t K, const float *fold, const float *beta_fold,
                                    float eps, int8_t *xq, float *x_scale, void *stream)
{
    using sq::fail;
    if (T < 0 || K < 8) return fail(SQ_ERR_INVALID_ARG, "sq_layernorm_smooth_quant: need T >= 0 and K >= 8");
    if (!fold) return fail(SQ_ERR_INVALID_ARG, "sq_layernorm_smooth_quant: fold is required");
    if (T > 0 && (!x || !xq || !x_scale)) return fail(SQ_ERR_INVALID_ARG, "sq_layernorm_smooth_quant: x, xq and x_scale are required");
    if (K % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_layernorm_smooth_quant: K must be a multiple of 8");
    if (K > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_layernorm_smooth_quant: K must be <= %d", kMaxK);
    if ((x && !sq::aligned(x, 16)) || (xq && !sq::aligned(xq, 8)) || !sq::aligned(fold, 16) ||
        (beta_fold && !sq::aligned(beta_fold, 16)) || (x_scale && !sq::aligned(x_scale, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_layernorm_smooth_quant: x, fold and beta_fold 16-byte, xq 8-byte, x_scale 4-byte alignment required");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    if (T == 0) return SQ_OK;
    RowArgs ra = {};
    ra.src = static_cast<const uint8_t *>(x);
    ra.rows = T;
    ra.ld_bytes = K * 2;
    ra.K = static_cast<int>(K);
    ra.vec = fold;
    ra.vec2 = beta_fold;
    ra.eps = eps;
    ra.q = xq;
    ra.scale = x_scale;
    return dispatch_rows<MODE_QLN, true>(ra, dev, sq::as_stream(stream));
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
    return sq::cuda_status(sq::launch_pdl(k_scales, dim3(static_cast<unsigned>((K + 255) / 256)), dim3(256), 0,
                                          sq::as_stream(stream), nullptr, amax_x, amax_w, K, ea, eb, gamma, s, fold),
                           "launch(scales)");
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

sq_status sq_smooth_quantize_weight_fp8(const void *w, int64_t N, int64_t K, const float *s, uint8_t *wq,
                                        float *w_scale, void *stream)
{
    using sq::fail;
    if (N < 0 || K < 8) return fail(SQ_ERR_INVALID_ARG, "sq_smooth_quantize_weight_fp8: need N >= 0 and K >= 8");
    if (N > 0 && (!w || !wq || !w_scale)) return fail(SQ_ERR_INVALID_ARG, "sq_smooth_quantize_weight_fp8: w, wq and w_scale are required");
    if (K % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_smooth_quantize_weight_fp8: K must be a multiple of 8");
    if (K > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_smooth_quantize_weight_fp8: K must be <= %d", kMaxK);
    if ((w && !sq::aligned(w, 16)) || (wq && !sq::aligned(wq, 8)) || (s && !sq::aligned(s, 16)) ||
        (w_scale && !sq::aligned(w_scale, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_smooth_quantize_weight_fp8: w and s 16-byte, wq 8-byte, w_scale 4-byte alignment required");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    if (N == 0) return SQ_OK;
    RowArgs ra = {};
    ra.src = static_cast<const uint8_t *>(w);
    ra.rows = N;
    ra.ld_bytes = K * 2;
    ra.K = static_cast<int>(K);
    ra.vec = s;
    ra.q = reinterpret_cast<int8_t *>(wq);
    ra.scale = w_scale;
    return dispatch_rows<MODE_QF8, false>(ra, dev, sq::as_stream(stream));
}

sq_status sq_rmsnorm_smooth_quant_fp8(const void *x, int64_t T, int64_t K, const float *fold, float eps,
                                      int apply_norm, uint8_t *xq, float *x_scale, void *stream)
{
    using sq::fail;
    if (T < 0 || K < 8) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant_fp8: need T >= 0 and K >= 8");
    if (!fold) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant_fp8: fold is required");
    if (T > 0 && (!x || !xq || !x_scale)) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant_fp8: x, xq and x_scale are required");
    if (K % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_rmsnorm_smooth_quant_fp8: K must be a multiple of 8");
    if (K > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_rmsnorm_smooth_quant_fp8: K must be <= %d", kMaxK);
    if ((x && !sq::aligned(x, 16)) || (xq && !sq::aligned(xq, 8)) || !sq::aligned(fold, 16) ||
        (x_scale && !sq::aligned(x_scale, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_rmsnorm_smooth_quant_fp8: x and fold 16-byte, xq 8-byte, x_scale 4-byte alignment required");
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
    ra.q = reinterpret_cast<int8_t *>(xq);
    ra.scale = x_scale;
    cudaStream_t st = sq::as_stream(stream);
    return apply_norm ? dispatch_rows<MODE_QF8, true>(ra, dev, st) : dispatch_rows<MODE_QF8, false>(ra, dev, st);
}

sq_status sq_static_scale(const float *amax, const float *factor, int64_t K, float *scale2, void *stream)
{
    using sq::fail;
    if (!amax || !scale2) return fail(SQ_ERR_INVALID_ARG, "sq_static_scale: amax and scale2 are required");
    if (K < 1) return fail(SQ_ERR_INVALID_ARG, "sq_static_scale: K must be >= 1");
    if (!sq::aligned(amax, 4) || !sq::aligned(scale2, 4) || (factor && !sq::aligned(factor, 4)))
        return fail(SQ_ERR_MISALIGNED, "sq_static_scale: fp32 arrays must be 4-byte aligned");
    int dev = 0;
    SQ_TRY_ARCH(dev);
    return sq::cuda_status(
        sq::launch_pdl(k_static_scale, dim3(1), dim3(1024), 0, sq::as_stream(stream), nullptr, amax, factor, K, scale2),
        "launch(static_scale)");
}

sq_status sq_rmsnorm_smooth_quant_static(const void *x, int64_t T, int64_t K, const float *fold, float eps,
                                         int apply_norm, const float *scale2, int8_t *xq, float *x_scale,
                                         void *stream)
{
    using sq::fail;
    if (T < 0 || K < 8) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant_static: need T >= 0 and K >= 8");
    if (!fold || !scale2) return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant_static: fold and scale2 are required");
    if (T > 0 && (!x || !xq || !x_scale))
        return fail(SQ_ERR_INVALID_ARG, "sq_rmsnorm_smooth_quant_static: x, xq and x_scale are required");
    if (K % 8 != 0) return fail(SQ_ERR_MISALIGNED, "sq_rmsnorm_smooth_quant_static: K must be a multiple of 8");
    if (K > kMaxK) return fail(SQ_ERR_UNSUPPORTED, "sq_rmsnorm_smooth_quant_static: K must be <= %d", kMaxK);
    if ((x && !sq::aligned(x, 16)) || (xq && !sq::aligned(xq, 8)) || !sq::aligned(fold, 16) || !sq::aligned(scale2, 4) ||
        (x_scale && !sq::aligned(x_scale, 4)))
        return fail(SQ_ERR_MISALIGNED,
                    "sq_rmsnorm_smooth_quant_static: x and fold 16-byte, xq 8-byte, scale2 and x_scale 4-byte alignment required");
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
    ra.scale2 = scale2;
    cudaStream_t st = sq::as_stream(stream);
    return apply_norm ? dispatch_rows<MODE_QSTATIC, true>(ra, dev, st) : dispatch_rows<MODE_QSTATIC, false>(ra, dev, st);
}

}  // extern "C"
