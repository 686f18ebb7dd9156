// sq_gemm.cu -- W8A8 linear on the sm_100a tensor cores: INT8 x INT8 -> INT32 with the
// dequantisation (per-token scale x per-output-channel scale, plus bias) fused into the epilogue.
//
// Pages cited (title, then section / equation / figure):
//   [MIGRATE] "06 -- SmoothQuant: Migrating Difficulty from Activations to Weights", section 7
//             ("Bit-level and kernel-level realities": INT8 x INT8 -> INT32 followed by
//             Y = scale_x * scale_w * Y_int32)
//   [TAMING]  "Taming the Outliers: A Deep Dive into SmoothQuant for LLM Quantization",
//             "System Architecture" (the flowchart's GEMM node and its bias-and-dequantise node)
//
// The pages name the operation, not a kernel design (their INT8 kernels target earlier tensor-core
// generations). This kernel is written for B200:
//   * persistent: one CTA per SM (the shared-memory footprint admits exactly one), tiles
//     128 tokens x 256 output channels handed out round-robin in bands of 16 or 32 M tiles for L2 reuse;
//   * warp 0 (one lane) streams 128-byte K slices of both operands into a 4-stage shared-memory
//     ring with TMA (128-byte swizzle), completion tracked by mbarrier transaction counts;
//   * warp 1 (one lane) issues tcgen05.mma.kind::i8 (M=128, N=256, K=32, signed x signed -> s32)
//     into a tensor-memory accumulator; two accumulators of 256 columns alternate so the epilogue
//     of one tile overlaps the main loop of the next;
//   * warps 2..5 read the accumulator with tcgen05.ld (each warp its own 32-lane quarter), apply
//     y = bf16(float(acc) * (x_scale * w_scale) + bias) in binary32 with explicit rounding, stage
//     32 x 32 boxes in 64-byte-swizzled shared memory and write them with TMA stores (the TMA clips
//     rows beyond T and columns beyond N).
// Other forms of the same kernel: 64-channel tiles when 256-wide tiles would leave SMs idle; for at
// most 128 tokens the decode form, where the weight is the 128-row MMA operand and the tokens the
// narrow one; an opt-in CTA-pair form (tcgen05 cta_group::2, 256 x 256 tiles); and FP8 E4M3 operands
// (kind::f8f6f4, binary32 accumulators) with the same epilogue. Every launch is a programmatic
// dependent launch: barrier and tensor-memory set-up overlap the previous kernel of the stream, and
// griddepcontrol.wait precedes the first global-memory access.
// Every mbarrier wait is bounded by a wall-clock limit (%globaltimer). When one runs out, the
// kernel records SQ_ERR_TIMEOUT in a device status word, every role leaves its loop, in-flight
// copies and MMAs are waited for (again with a limit), tensor memory is released and the kernel
// returns. No wait can hang the GPU.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "sq_device.cuh"
#include "sq_internal.h"

using namespace sqdev;

namespace {

// Device-side status word: 0 or the first sq_status a kernel recorded.
__device__ unsigned int g_sq_status;
// The status word's value at the moment sq_device_status read and cleared it.
__device__ unsigned int g_sq_status_read;

// Host-side choice of the GEMM form (sq_set_gemm_cta_pair).
std::atomic<int> g_cta_pair{0};

constexpr int BM = 128;            // tokens per tile (MMA M)
constexpr int BN = 256;            // output channels per tile of the wide forms (MMA N)
constexpr int BK = 128;            // K bytes per pipeline stage (one 128-byte swizzle row)
constexpr int UMMA_K = 32;         // K per tcgen05.mma.kind::i8
constexpr int A_STAGE = BM * BK;   // 16 KB
constexpr int EPI_WARPS = 4;
constexpr int OUT_COLS = 32;       // bf16 columns per TMA store box (64 bytes, 64-byte swizzle)
constexpr int OUT_ROWS = 32;       // rows per box: one warp's TMEM lane quarter
constexpr int OUT_BOX = OUT_COLS * 2 * OUT_ROWS;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
// M tiles per raster band, chosen per call (band_for below). Every band streams the whole weight,
// so when the weight does not fit the L2 wider bands read less from DRAM (the 70B-shaped MLP
// up-projection, T 16384, K 8192, N 28672: 2.02 GB read per call with bands of 16, 1.16 GB with 32).
// The GEMM runs at the power limit, and the DRAM power saved raised the sustained clock and rate
// (1440 -> 1466 MHz, 2674 -> 2733 TOPS; gate+up N 28672, K 4096: 2494 -> 2567 TOPS). With a weight that
// the L2 holds, 16 is slightly better (query projection N = K = 4096: 2450 against 2427 TOPS). Bands of
// 64 token tiles (67 MB of tokens at K = 8192) no longer stay in the L2 and read 6.6 GB.
constexpr int BAND_SMALL = 16;
constexpr int BAND_LARGE = 32;
int band_for(int64_t N, int64_t K) { return N * K > (int64_t(64) << 20) ? BAND_LARGE : BAND_SMALL; }
constexpr int COL_TAB = 2 * BN * 4;   // w_scale and bias (binary32) of up to 256 columns

// Instruction descriptor of tcgen05.mma.kind::i8: D = s32, A and B signed 8-bit, both K-major,
// N >> 3 at bits 17..22, M >> 4 at bits 24..28.
constexpr uint32_t make_idesc(int M, int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
// kind::f8f6f4 with A and B E4M3 (format 0), D = f32 (format 1 at bits 4..5), both K-major.
constexpr uint32_t make_idesc_f8(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
// Binary32 value of an accumulator word: the integer converted (INT8 form) or the f32 bits (FP8).
template <bool F8>
__device__ __forceinline__ float acc_value(uint32_t r) {
    if (F8) return __uint_as_float(r);
    return __int2float_rn(static_cast<int>(r));
}

// Shared-memory plan of the single-SM kernel for tiles of TN output channels. The 256-wide form
// serves token counts that fill the SMs with tiles; the 64-wide form serves few tokens (decode),
// where the weight stream dominates: four times as many tiles, and a deeper ring (8 stages of
// 24 KB) keeps more weight bytes in flight per SM.
//
// SWAP: the decode form for at most 128 tokens. The operands trade places: the weight is the MMA's
// 128-row A operand and the tokens its TN-column (16 .. 128) B operand, so every ring slot carries 16 KB
// of weight rows and the ring (6 .. 11 stages) keeps up to ~180 KB of the weight stream in flight per
// SM; the accumulator lanes are output channels and its columns tokens.
constexpr int DECODE_KS = 2;       // 128-byte K slices per stage of the decode form

template <int TN, bool SWAP = false>
struct Tile {
    // K slices per stage: the decode form reads DECODE_KS consecutive 128-byte pieces of every weight
    // row per stage (longer contiguous DRAM reads); the other forms one.
    static constexpr int KS = SWAP ? DECODE_KS : 1;
    static constexpr int A_SLOT = KS * A_STAGE;
    static constexpr int B_SLICE = TN * BK;
    static constexpr int B_SLOT = KS * B_SLICE;
    static constexpr int SPARE = 232448 - 1024 - EPI_WARPS * 2 * OUT_BOX - 2 * COL_TAB - 512;
    static constexpr int STAGES = SWAP ? (SPARE / (A_SLOT + B_SLOT) > 11 ? 11 : SPARE / (A_SLOT + B_SLOT))
                                       : (SPARE / (A_SLOT + B_SLOT) > 8 ? 8 : SPARE / (A_SLOT + B_SLOT));   // 256: 4, 64: 8
    // two accumulators ACC_STRIDE columns apart; the allocation is a power of two >= 32 columns
    static constexpr uint32_t TMEM_COLS = 2u * TN;
    static constexpr uint32_t ACC_STRIDE = TMEM_COLS / 2;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_SLOT;
    static constexpr int OFF_OUT = OFF_B + STAGES * B_SLOT;
    static constexpr int OFF_COL = OFF_OUT + EPI_WARPS * 2 * OUT_BOX;
    static constexpr int OFF_BAR = OFF_COL + 2 * COL_TAB;   // one column table per accumulator
    static constexpr int NBARS = 2 * STAGES + 5;            // full[S], empty[S], tfull[2], tempty[2], done
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM_TOTAL = OFF_MISC + 16 + 1024; // slack to align the base to 1024 bytes
    static constexpr uint32_t IDESC = make_idesc(BM, TN);
    static constexpr uint32_t IDESC_F8 = make_idesc_f8(BM, TN);
    static_assert(SMEM_TOTAL <= 232448, "shared memory budget of one sm_100 CTA");
    static_assert(SWAP ? (TN >= 16 && TN <= 128 && (TN & (TN - 1)) == 0)
                       : (TN % OUT_COLS == 0 && TN >= 32 && TN <= 256 && (TN & (TN - 1)) == 0), "tile width");
};

// ------------------------------------------------------------------------------------------------
// PTX wrappers.

__device__ __forceinline__ void record_status(unsigned int code) { atomicCAS(&g_sq_status, 0u, code); }

__device__ __forceinline__ void give_up(volatile int *abort_flag) {
    record_status(SQ_ERR_TIMEOUT);
    *abort_flag = 1;
}

// The tensor maps loaded here hold 8-bit operands: the innermost coordinate c0 must be a multiple of
// 16 elements (16 bytes). Stores write bf16: c0 a multiple of 8, and no coordinate negative.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1) {
    if (!SQ_CHECK(c0 >= 0 && (c0 & 15) == 0, &g_sq_status)) return;
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int c0, int c1) {
    if (!SQ_CHECK(c0 >= 0 && c1 >= 0 && (c0 & 7) == 0, &g_sq_status)) return;
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// L2 prefetch of one 8-bit tensor box (a hint: no shared memory is written and nothing completes on a
// barrier). The innermost coordinate c0 must be a multiple of 16 elements, as for the loads.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int c0, int c1) {
    if (!SQ_CHECK(c0 >= 0 && (c0 & 15) == 0, &g_sq_status)) return;
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// FP8 form: A and B both E4M3, binary32 accumulators (tcgen05.mma.kind::f8f6f4, K = 32 per instruction).
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory descriptor of a K-major operand tile written by TMA with the 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), leading byte offset 1
// (unused for swizzled K-major layouts), descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1u) << 16) |
           (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
           (static_cast<uint64_t>(2u) << 61);
}

__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int BAND, int &m, int &n) {
    const int per_band = BAND * n_tiles;
    const int band = t / per_band;
    const int within = t - band * per_band;
    const int bs = min(BAND, m_tiles - band * BAND);
    n = within / bs;
    m = band * BAND + (within - n * bs);
}

// 2-SM (CTA pair) forms.
__device__ __forceinline__ uint32_t mapa_rank(uint32_t addr, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
    return d;
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on `bar_cluster`, a barrier of
// either CTA of the pair (shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, uint32_t bar_cluster, int c0, int c1) {
    if (!SQ_CHECK(c0 >= 0 && (c0 & 15) == 0, &g_sq_status)) return;   // 8-bit operands, as above
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Lowers the pending transaction count of the current phase of `bar` by `bytes` (bytes that were
// expected but will never arrive).
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// 64-bit load from shared memory of a CTA of the cluster (a shared::cluster address).
__device__ __forceinline__ long long ld_cluster_s64(uint32_t addr) {
    long long v;
    asm volatile("ld.shared::cluster.b64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
    return v;
}
// Bounded wait with cluster-scope acquire (the barrier is completed from the peer CTA).
__device__ __noinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                               const volatile int *abort_flag) {
    if (mbar_try_cluster(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_cluster(bar, parity)) return true;
        if ((i & 127u) == 0u) {
            if (abort_flag && *abort_flag) return false;
            if (global_ns() - t0 > limit_ns) return false;
        }
    }
}
__device__ __forceinline__ void tmem_alloc2(uint32_t slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_commit2(uint32_t bar_cluster) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// Column table of one tile: w_scale and bias (widened to binary32) of its 256 output channels, read
// by every epilogue lane with broadcast shared-memory loads. The 128 epilogue threads each fetch two
// columns from global memory one tile ahead and write them when the tile starts; there is one table
// per accumulator buffer.
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr uint32_t EPI_BAR = 1;     // named barrier of the epilogue warps

struct ColShare {
    float2 w;
    uint32_t b;
};

// The tile's TN columns: thread ep fetches columns n0 + 2 ep and n0 + 2 ep + 1 (threads beyond
// TN / 2 fetch nothing).
template <int TN>
__device__ __forceinline__ void cols_fetch(ColShare &p, int n0, int ep, const float *__restrict__ w_scale,
                                           const __nv_bfloat16 *__restrict__ bias, int N) {
    const int col = n0 + 2 * ep;
    p.w = make_float2(0.f, 0.f);
    p.b = 0u;
    if (2 * ep < TN && col < N) {      // N is even: both columns are in range or both beyond it
        p.w = __ldg(reinterpret_cast<const float2 *>(w_scale + col));
        if (bias != nullptr) p.b = __ldg(reinterpret_cast<const unsigned int *>(bias + col));
    }
}

template <int TN>
__device__ __forceinline__ void cols_store(const ColShare &p, float *tab, int ep) {
    if (2 * ep >= TN) return;
    *reinterpret_cast<float2 *>(tab + 2 * ep) = p.w;
    *reinterpret_cast<float2 *>(tab + TN + 2 * ep) = make_float2(__uint_as_float(p.b << 16), __uint_as_float(p.b & 0xFFFF0000u));
}

// Two packed pairs (four consecutive binary32 values) from shared memory, same address in every lane.
__device__ __forceinline__ void lds_pairs(const float *p, uint64_t &a, uint64_t &b) {
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(smem_u32(p)));
}

__device__ __forceinline__ uint32_t bf16x2_rn(uint64_t v) {
    uint32_t lo, hi, d;
    unpack2(v, lo, hi);
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(__uint_as_float(hi)), "f"(__uint_as_float(lo)));
    return d;
}

// 32 columns of this warp's TMEM lane quarter into r[0..31] (asynchronous until tmem_ld_wait).
__device__ __forceinline__ void tmem_ld32p(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// Orders every later use of r[0..31] after the preceding tcgen05.wait::ld.
__device__ __forceinline__ void regs_after_wait(uint32_t *r) {
#pragma unroll
    for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// Epilogue of one warp for one output tile: reads its 32 TMEM lanes (token rows row0 .. row0+31) for
// columns n0 .. n0+TN-1 of accumulator buffer `tcol` (TMEM column offset), applies
// y = bf16(float(acc) * (x_scale * w_scale) + bias) in binary32 (each operation rounded once, two
// columns per packed instruction), stages 32 x 32 boxes in 64-byte-swizzled shared memory and writes
// them with TMA stores; optionally writes the raw accumulators. `tab` is the tile's column table,
// `xs` the x_scale of this lane's row. The TMEM read of the next 32 columns is in flight while the
// current 32 are converted. `stage_buf` holds two boxes that alternate; `nstores` counts this warp's
// stores.
template <int TN, bool F8>
__device__ __forceinline__ void epilogue_rows(uint32_t tmem_base, int quad, int lane, uint32_t tcol, int row0, int n0,
                                              float xs, const float *tab, bool has_bias, int32_t *__restrict__ acc_out,
                                              int T, int N, const CUtensorMap *tmY, uint8_t *stage_buf, int &nstores)
{
    if (row0 >= T) return;
    const int row = row0 + lane;
    const uint64_t xs2 = pack2(xs, xs);
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + tcol;
    uint32_t ra[32], rb[32];
    tmem_ld32p(tl, ra);
#pragma unroll
    for (int c = 0; c < TN / OUT_COLS; ++c) {
        uint32_t *cur = (c & 1) ? rb : ra;
        uint32_t *nxt = (c & 1) ? ra : rb;
        tmem_ld_wait();
        regs_after_wait(cur);
        if (c + 1 < TN / OUT_COLS) tmem_ld32p(tl + (c + 1) * OUT_COLS, nxt);
        const int col0 = n0 + c * OUT_COLS;
        if (col0 >= N) continue;
        if (acc_out != nullptr && row < T) {
            int4 *dst = reinterpret_cast<int4 *>(acc_out + static_cast<int64_t>(row) * N + col0);
#pragma unroll
            for (int g = 0; g < OUT_COLS / 4; ++g) {
                if (col0 + 4 * g < N && SQ_CHECK(row >= 0 && col0 + 4 * g + 4 <= N, &g_sq_status))
                    dst[g] = make_int4(static_cast<int>(cur[4 * g]), static_cast<int>(cur[4 * g + 1]),
                                       static_cast<int>(cur[4 * g + 2]), static_cast<int>(cur[4 * g + 3]));
            }
        }
        uint32_t packed[OUT_COLS / 2];
#pragma unroll
        for (int g = 0; g < OUT_COLS / 4; ++g) {
            uint64_t w01, w23;
            lds_pairs(tab + c * OUT_COLS + 4 * g, w01, w23);
            const uint64_t a01 = pack2(acc_value<F8>(cur[4 * g]), acc_value<F8>(cur[4 * g + 1]));
            const uint64_t a23 = pack2(acc_value<F8>(cur[4 * g + 2]), acc_value<F8>(cur[4 * g + 3]));
            uint64_t v01 = mul2_rn(a01, mul2_rn(xs2, w01));
            uint64_t v23 = mul2_rn(a23, mul2_rn(xs2, w23));
            if (has_bias) {
                // scalar round-to-nearest adds: never contracted with the multiply before them into
                // a fused multiply-add (a packed add after a packed multiply can be)
                uint64_t b01, b23;
                lds_pairs(tab + TN + c * OUT_COLS + 4 * g, b01, b23);
                v01 = add2_scalar(v01, b01);
                v23 = add2_scalar(v23, b23);
            }
            packed[2 * g] = bf16x2_rn(v01);
            packed[2 * g + 1] = bf16x2_rn(v23);
        }
        // stage the 32 x 32 box (64-byte rows, 64-byte swizzle: the 16-byte chunk index is XORed
        // with bits 1..2 of the row), then one TMA store
        uint8_t *sb = stage_buf + (nstores & 1) * OUT_BOX;
        if (lane == 0) bulk_wait_read_1();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int pos = q ^ ((lane >> 1) & 3);
            *reinterpret_cast<uint4 *>(sb + lane * 64 + pos * 16) =
                make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmY, smem_u32(sb), col0, row0);
            bulk_commit();
        }
        ++nstores;
    }
    tmem_ld_wait();     // nothing of this tile's accumulator is still being read
}

// 16 columns of this warp's TMEM lane quarter into r[0..15] (asynchronous until tmem_ld_wait).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Per-channel constants of the swapped (decode) form's epilogue for output channel n (w_scale and the
// bias widened to binary32; zeros beyond N). Fetched before the tile's accumulator is ready, so their
// memory latency overlaps the weight stream instead of following it.
struct SwapCol {
    float ws, b;
};
__device__ __forceinline__ SwapCol swap_col(int n, int N, const float *__restrict__ w_scale,
                                            const __nv_bfloat16 *__restrict__ bias) {
    SwapCol c = {0.0f, 0.0f};
    if (n < N) {
        c.ws = __ldg(w_scale + n);
        if (bias != nullptr) c.b = __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short *>(bias) + n)) << 16);
    }
    return c;
}

// Epilogue of the swapped (decode) form for one tile: thread (quad, lane) owns output channel
// n = n_base + 32 quad + lane (constants `col`, fetched ahead) and writes
// y[t][n] = bf16(float(acc) * (x_scale[t] * w_scale[n]) + bias[n]) (each operation rounded once, the same
// steps as the other forms) for the tile's tokens t < T, with x_scale read from the shared-memory copy
// `xs` (all T <= 128 tokens); a warp writes 32 consecutive channels of a token per store. Optionally
// writes the raw accumulators.
template <int TN, bool F8>
__device__ __forceinline__ void epilogue_swap(uint32_t tmem_base, int quad, int lane, uint32_t tcol, int n_base, int t0,
                                              const float *xs, SwapCol col, bool has_bias, __nv_bfloat16 *__restrict__ y,
                                              int32_t *__restrict__ acc_out, int T, int N)
{
    const int nq = n_base + quad * 32;
    if (nq >= N) return;                    // the whole quarter lies beyond N
    const int n = nq + lane;
    const bool okn = n < N;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + tcol;
#pragma unroll
    for (int c = 0; c < TN; c += 16) {
        if (t0 + c >= T) break;             // uniform in the warp
        uint32_t r[16];
        tmem_ld16(tl + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) asm volatile("" : "+r"(r[i]));
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int t = t0 + c + j;
            if (t < T && okn) {
                const int acc = static_cast<int>(r[j]);
                const int64_t o = static_cast<int64_t>(t) * N + n;
                if (!SQ_CHECK(t >= 0 && t < BM && n >= 0 && o < static_cast<int64_t>(T) * N, &g_sq_status)) continue;
                if (acc_out != nullptr) acc_out[o] = acc;
                float v = __fmul_rn(acc_value<F8>(r[j]), __fmul_rn(xs[t], col.ws));
                if (has_bias) v = __fadd_rn(v, col.b);
                y[o] = __float2bfloat16_rn(v);
            }
        }
    }
}

// ------------------------------------------------------------------------------------------------

template <int TN, bool SWAP, bool F8>
__global__ void __launch_bounds__(THREADS, 1)
k_w8a8_linear(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmY, const float *__restrict__ x_scale,
              const float *__restrict__ w_scale, const __nv_bfloat16 *__restrict__ bias,
              int32_t *__restrict__ acc_out, __nv_bfloat16 *__restrict__ y, int T, int N, int K, int m_tiles,
              int n_tiles, int band, uint64_t limit_ns)
{
    using L = Tile<TN, SWAP>;
    constexpr int STAGES = L::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + L::OFF_A;
    uint8_t *sB = smem + L::OFF_B;
    uint8_t *sOut = smem + L::OFF_OUT;
    float *sCol = reinterpret_cast<float *>(smem + L::OFF_COL);
    const uint32_t bar0 = smem_u32(smem + L::OFF_BAR);
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(full(s), 1); mbar_init(empty(s), 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(tfull(b), 1); mbar_init(tempty(b), 32 * EPI_WARPS); }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        mbar_init_fence();
        fence_async_smem();
    }
    if (warp == 0 && lane == 0) {
        prefetch_map(&tmA); prefetch_map(&tmB); prefetch_map(&tmY);
        if (SWAP && static_cast<int>(blockIdx.x) < m_tiles * n_tiles) {
            // Decode form: the first two stages of this CTA's weight rows (64 KB) are requested into
            // the L2 while the previous kernel of the stream finishes, so the first loads after the
            // dependency wait find them there (a whole ring's worth, most of the weight, competed with
            // the previous call's own stream). Only a cache hint: the loads themselves still follow the wait, and
            // the L2 is where every writer's data meets, so a weight written by that kernel is still
            // read as written.
            int m, n;
            tile_coords(blockIdx.x, m_tiles, n_tiles, band, m, n);
            const int kbs = (K + L::KS * BK - 1) / (L::KS * BK);
            for (int kb = 0; kb < 2 && kb < kbs; ++kb)
                for (int ks = 0; ks < L::KS; ++ks) tma_prefetch_l2_2d(&tmA, (kb * L::KS + ks) * BK, m * BM);
        }
    }
    if (warp == 1) { tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // dependent launch: the set-up above touched shared and tensor memory only (and, in the decode
    // form, sent L2 prefetch hints)
    pdl_wait();
    pdl_trigger();

    constexpr int KS = L::KS;
    const int k_blocks = (K + KS * BK - 1) / (KS * BK);   // slices beyond K are zero-filled by the TMA
    const int num_tiles = m_tiles * n_tiles;
    constexpr uint32_t stage_tx = static_cast<uint32_t>(L::A_SLOT + L::B_SLOT);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long fills = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int m, n;
                tile_coords(t, m_tiles, n_tiles, band, m, n);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(empty(stage), phase ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
                    mbar_expect_tx(full(stage), stage_tx);
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        tma_load_2d(smem_u32(sA + stage * L::A_SLOT + ks * A_STAGE), &tmA, full(stage), (kb * KS + ks) * BK, m * BM);
                        tma_load_2d(smem_u32(sB + stage * L::B_SLOT + ks * L::B_SLICE), &tmB, full(stage), (kb * KS + ks) * BK, n * TN);
                    }
                    ++fills;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) give_up(abort_flag);
            // Wait for the last fill of every stage to land, so no copy is in flight at exit.
            for (int s = 0; s < STAGES; ++s) {
                if (fills <= s) break;
                const long long last = s + ((fills - 1 - s) / STAGES) * STAGES;
                if (!mbar_wait(full(s), static_cast<uint32_t>((last / STAGES) & 1), limit_ns, nullptr))
                    record_status(SQ_ERR_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            bool issued = false;
            int lt = 0;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                const uint32_t use = static_cast<uint32_t>(lt >> 1);
                if (!mbar_wait(tempty(buf), (use & 1u) ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf) * L::ACC_STRIDE;
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(full(stage), phase, limit_ns, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const uint32_t a0 = smem_u32(sA + stage * L::A_SLOT + ks * A_STAGE);
                        const uint32_t b0 = smem_u32(sB + stage * L::B_SLOT + ks * L::B_SLICE);
#pragma unroll
                        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                            if (F8)
                                mma_f8(d_tmem, kmajor_sw128_desc(a0 + kk * UMMA_K), kmajor_sw128_desc(b0 + kk * UMMA_K), L::IDESC_F8,
                                       (kb | ks | kk) != 0 ? 1u : 0u);
                            else
                                mma_i8(d_tmem, kmajor_sw128_desc(a0 + kk * UMMA_K), kmajor_sw128_desc(b0 + kk * UMMA_K), L::IDESC,
                                       (kb | ks | kk) != 0 ? 1u : 0u);
                        }
                    }
                    issued = true;
                    tc_commit(empty(stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(tfull(buf));
            }
            if (!ok) give_up(abort_flag);
            // Every MMA issued above has completed once this commit's barrier flips.
            if (issued) {
                tc_commit(done_bar);
                if (!mbar_wait(done_bar, 0, limit_ns, nullptr)) record_status(SQ_ERR_TIMEOUT);
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int quad = warp & 3;                  // TMEM lanes this warp may read: 32*quad .. +31
      if constexpr (SWAP) {
        // the tokens' x_scale (T <= 128) into shared memory (the column-table area, unused by this
        // form) while the weight streams; the first tile's channel constants likewise
        const int ep = threadIdx.x - 64;
        if (ep < T && SQ_CHECK(ep < BM, &g_sq_status)) sCol[ep] = __ldg(x_scale + ep);
        named_sync(EPI_BAR, EPI_THREADS);
        int lt = 0;
        SwapCol col = {0.0f, 0.0f};
        if (static_cast<int>(blockIdx.x) < num_tiles) {
            int m, n;
            tile_coords(blockIdx.x, m_tiles, n_tiles, band, m, n);
            col = swap_col(m * BM + quad * 32 + lane, N, w_scale, bias);
        }
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1);
            if (!mbar_wait(tfull(buf), use & 1u, limit_ns, abort_flag)) { give_up(abort_flag); break; }
            tc_fence_after();
            int m, n;
            tile_coords(t, m_tiles, n_tiles, band, m, n);
            const SwapCol cur = col;
            const int tn = t + static_cast<int>(gridDim.x);
            if (tn < num_tiles) {                   // the next tile's constants, ahead of its accumulator
                int m2, n2;
                tile_coords(tn, m_tiles, n_tiles, band, m2, n2);
                col = swap_col(m2 * BM + quad * 32 + lane, N, w_scale, bias);
            }
            epilogue_swap<TN, F8>(tmem_base, quad, lane, static_cast<uint32_t>(buf) * L::ACC_STRIDE, m * BM, n * TN, sCol, cur,
                                  bias != nullptr, y, acc_out, T, N);
            tc_fence_before();
            mbar_arrive(tempty(buf));
        }
      } else {
        uint8_t *stage_buf = sOut + (warp - 2) * 2 * OUT_BOX;
        const int ep = threadIdx.x - 64;            // 0 .. 127 among the epilogue threads
        int nstores = 0;
        int lt = 0;
        // this thread's share of the next tile's column table, and its row's x_scale, one tile ahead
        ColShare cols;
        float xs = 0.0f;
        auto prefetch = [&](int t) {
            if (t >= num_tiles) return;
            int m, n;
            tile_coords(t, m_tiles, n_tiles, band, m, n);
            cols_fetch<TN>(cols, n * TN, ep, w_scale, bias, N);
            const int row = m * BM + quad * 32 + lane;
            xs = row < T ? __ldg(x_scale + row) : 0.0f;
        };
        prefetch(blockIdx.x);
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1);
            const bool ok = mbar_wait(tfull(buf), use & 1u, limit_ns, abort_flag);
            float *tab = sCol + buf * (COL_TAB / 4);
            if (ok) cols_store<TN>(cols, tab, ep);
            // every epilogue thread arrives (its wait is bounded); the table is complete after it
            if (named_sync_or(EPI_BAR, EPI_THREADS, !ok)) { give_up(abort_flag); break; }
            tc_fence_after();
            int m, n;
            tile_coords(t, m_tiles, n_tiles, band, m, n);
            const float xs_t = xs;
            prefetch(t + gridDim.x);
            epilogue_rows<TN, F8>(tmem_base, quad, lane, static_cast<uint32_t>(buf) * L::ACC_STRIDE, m * BM + quad * 32, n * TN, xs_t, tab,
                          bias != nullptr, acc_out, T, N, &tmY, stage_buf, nstores);
            tc_fence_before();
            mbar_arrive(tempty(buf));
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
      }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, L::TMEM_COLS);
}

// ------------------------------------------------------------------------------------------------
// 2-SM variant: a cluster of two CTAs computes a 256 x 256 tile with tcgen05.mma.cta_group::2
// (M = 256, N = 256, K = 32). Each CTA loads its own 128 rows of A and 128 rows of B (the MMA reads
// the peer's B half through the pair link), so every SM moves half the B bytes of the single-SM
// kernel per MMA and a 6-stage ring fits in shared memory. Only the even CTA issues MMAs; every TMA
// load of both CTAs completes on the even CTA's full barrier; each MMA batch is committed to the
// empty barriers of both CTAs and each finished accumulator to both CTAs' tfull barriers; the odd
// CTA's epilogue warps arrive remotely on the even CTA's tempty barrier.
constexpr int P_STAGES = 6;
constexpr int P_A_STAGE = BM * BK;          // 16 KB: this CTA's 128 token rows
constexpr int P_B_STAGE = 128 * BK;         // 16 KB: this CTA's 128 of the tile's 256 channels
constexpr int P_OFF_A = 0;
constexpr int P_OFF_B = P_OFF_A + P_STAGES * P_A_STAGE;
constexpr int P_OFF_OUT = P_OFF_B + P_STAGES * P_B_STAGE;
constexpr int P_OFF_COL = P_OFF_OUT + EPI_WARPS * 2 * OUT_BOX;
constexpr int P_OFF_BAR = P_OFF_COL + 2 * COL_TAB;
constexpr int P_NBARS = 2 * P_STAGES + 5;
constexpr int P_OFF_MISC = P_OFF_BAR + P_NBARS * 8;
constexpr int P_SMEM_TOTAL = P_OFF_MISC + 16 + 1024;
static_assert(P_SMEM_TOTAL <= 232448, "shared memory budget of one sm_100 CTA");
constexpr uint32_t P_IDESC = make_idesc(2 * BM, BN);
constexpr uint32_t P_TMEM_COLS = 2 * BN;

__global__ void __launch_bounds__(THREADS, 1)
k_w8a8_linear_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const float *__restrict__ x_scale,
                   const float *__restrict__ w_scale, const __nv_bfloat16 *__restrict__ bias,
                   int32_t *__restrict__ acc_out, int T, int N, int K, int m_tiles, int n_tiles, int band,
                   uint64_t limit_ns)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + P_OFF_A;
    uint8_t *sB = smem + P_OFF_B;
    uint8_t *sOut = smem + P_OFF_OUT;
    float *sCol = reinterpret_cast<float *>(smem + P_OFF_COL);
    const uint32_t bar0 = smem_u32(smem + P_OFF_BAR);
    auto full = [&](int st) { return bar0 + 8u * st; };
    auto empty = [&](int st) { return bar0 + 8u * (P_STAGES + st); };
    auto tfull = [&](int b) { return bar0 + 8u * (2 * P_STAGES + b); };
    auto tempty = [&](int b) { return bar0 + 8u * (2 * P_STAGES + 2 + b); };
    const uint32_t done_bar = bar0 + 8u * (2 * P_STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + P_OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + P_OFF_MISC + 4);
    long long *s_fills = reinterpret_cast<long long *>(smem + P_OFF_MISC + 8);   // ring fills this CTA issued

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();             // 0: issues the MMAs; 1: its peer
    const int cid = blockIdx.x >> 1;
    const int ncl = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int st = 0; st < P_STAGES; ++st) { mbar_init(full(st), 1); mbar_init(empty(st), 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(tfull(b), 1); mbar_init(tempty(b), 2 * EPI_WARPS); }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        *s_fills = 0;
        mbar_init_fence();
        fence_async_smem();
    }
    if (warp == 0 && lane == 0) { prefetch_map(&tmA); prefetch_map(&tmB); prefetch_map(&tmY); }
    if (warp == 1) { tmem_alloc2(smem_u32(tmem_slot), P_TMEM_COLS); tmem_relinquish2(); }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                                 // both CTAs' barriers exist before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();                                         // dependent launch (set-up above is on-chip only)
    pdl_trigger();

    const int k_blocks = (K + BK - 1) / BK;
    const int num_tiles = m_tiles * n_tiles;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long fills = 0;
            bool ok = true;
            for (int t = cid; t < num_tiles && ok; t += ncl) {
                int m, n;
                tile_coords(t, m_tiles, n_tiles, band, m, n);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_cluster(empty(stage), phase ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
                    if (rank == 0) mbar_expect_tx(full(stage), 2u * (P_A_STAGE + P_B_STAGE));
                    const uint32_t fb = mapa_rank(full(stage), 0);
                    tma_load_2d_pair(smem_u32(sA + stage * P_A_STAGE), &tmA, fb, kb * BK, m * 2 * BM + static_cast<int>(rank) * BM);
                    tma_load_2d_pair(smem_u32(sB + stage * P_B_STAGE), &tmB, fb, kb * BK, n * BN + static_cast<int>(rank) * 128);
                    ++fills;
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) give_up(abort_flag);
            *s_fills = fills;     // the pair's copies are drained at the end, once both counts are known
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (even CTA only) ----------------
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            bool issued = false;
            int lt = 0;
            for (int t = cid; t < num_tiles && ok; t += ncl, ++lt) {
                const int buf = lt & 1;
                const uint32_t use = static_cast<uint32_t>(lt >> 1);
                if (!mbar_wait_cluster(tempty(buf), (use & 1u) ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(full(stage), phase, limit_ns, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * P_A_STAGE);
                    const uint32_t b0 = smem_u32(sB + stage * P_B_STAGE);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        mma_i8_pair(d_tmem, kmajor_sw128_desc(a0 + kk * UMMA_K), kmajor_sw128_desc(b0 + kk * UMMA_K), P_IDESC,
                                    (kb | kk) != 0 ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit2(mapa_rank(empty(stage), 0));
                    tc_commit2(mapa_rank(empty(stage), 1));
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit2(mapa_rank(tfull(buf), 0));
                tc_commit2(mapa_rank(tfull(buf), 1));
            }
            if (!ok) give_up(abort_flag);
            if (issued) {
                tc_commit2(mapa_rank(done_bar, 0));
                if (!mbar_wait(done_bar, 0, limit_ns, nullptr)) record_status(SQ_ERR_TIMEOUT);
            }
        }
    } else {
        // ---------------- epilogue (both CTAs, each its 128 rows of the tile) ----------------
        const int quad = warp & 3;
        uint8_t *stage_buf = sOut + (warp - 2) * 2 * OUT_BOX;
        const int ep = threadIdx.x - 64;
        int nstores = 0;
        int lt = 0;
        ColShare cols;
        float xs = 0.0f;
        auto prefetch = [&](int t) {
            if (t >= num_tiles) return;
            int m, n;
            tile_coords(t, m_tiles, n_tiles, band, m, n);
            cols_fetch<BN>(cols, n * BN, ep, w_scale, bias, N);
            const int row = m * 2 * BM + static_cast<int>(rank) * BM + quad * 32 + lane;
            xs = row < T ? __ldg(x_scale + row) : 0.0f;
        };
        prefetch(cid);
        for (int t = cid; t < num_tiles; t += ncl, ++lt) {
            const int buf = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1);
            const bool ok = mbar_wait_cluster(tfull(buf), use & 1u, limit_ns, abort_flag);
            float *tab = sCol + buf * (COL_TAB / 4);
            if (ok) cols_store<BN>(cols, tab, ep);
            if (named_sync_or(EPI_BAR, EPI_THREADS, !ok)) { give_up(abort_flag); break; }
            tc_fence_after();
            int m, n;
            tile_coords(t, m_tiles, n_tiles, band, m, n);
            const float xs_t = xs;
            prefetch(t + ncl);
            epilogue_rows<BN, false>(tmem_base, quad, lane, static_cast<uint32_t>(buf * BN),
                          m * 2 * BM + static_cast<int>(rank) * BM + quad * 32, n * BN, xs_t, tab, bias != nullptr, acc_out,
                          T, N, &tmY, stage_buf, nstores);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(mapa_rank(tempty(buf), 0));   // one arrival per warp, on the even CTA
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    // Drain: every TMA copy of either CTA completes on the even CTA's full barriers, so the pair may
    // leave once the last fill of every stage has completed there. Without a timeout both CTAs issued
    // the same fills. After one, their counts f0 (even) and f1 (odd) may differ by at most a ring's
    // depth (neither producer can run more than one ring ahead of the MMAs, which need both halves):
    // a fill only the odd CTA issued still lacks the even CTA's arrival, posted here with the odd
    // CTA's bytes; a fill only the even CTA issued expects bytes the odd CTA will never send, taken
    // off its count here. Every wait is bounded; one that runs out records SQ_ERR_TIMEOUT.
    cluster_sync_all();                                 // both fill counts are written
    if (rank == 0 && threadIdx.x == 0) {
        const long long f0 = *s_fills;
        const long long f1 = ld_cluster_s64(mapa_rank(smem_u32(s_fills), 1));
        const long long lo = f0 < f1 ? f0 : f1, hi = f0 < f1 ? f1 : f0;
        for (long long j = lo; j < hi; ++j) {
            const int st = static_cast<int>(j % P_STAGES);
            if (f1 > f0) mbar_expect_tx(full(st), static_cast<uint32_t>(P_A_STAGE + P_B_STAGE));
            else mbar_complete_tx(full(st), static_cast<uint32_t>(P_A_STAGE + P_B_STAGE));
        }
        for (int st = 0; st < P_STAGES; ++st) {
            if (hi <= st) break;
            const long long last = st + ((hi - 1 - st) / P_STAGES) * P_STAGES;
            if (!mbar_wait(full(st), static_cast<uint32_t>((last / P_STAGES) & 1), limit_ns, nullptr))
                record_status(SQ_ERR_TIMEOUT);
        }
    }
    cluster_sync_all();                                 // the odd CTA leaves only after the drain
    tc_fence_after();
    if (warp == 1) tmem_dealloc2(tmem_base, P_TMEM_COLS);
}

// Reads and clears the status word in one atomic exchange, ordered on the caller's stream.
__global__ void k_status_exchange() { g_sq_status_read = atomicExch(&g_sq_status, 0u); }

// One thread waits, with the same bounded wait as the GEMM, on a barrier nothing completes.
__global__ void k_selftest_wait(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        mbar_init_fence();
        if (!mbar_wait(smem_u32(&bar), 0, limit_ns, &abort_flag)) record_status(SQ_ERR_TIMEOUT);
    }
}

#ifdef SQ_DEVICE_CHECKS
// Self-test of the bounds checks: one thread stores to index `i` of an 8-word array under a check
// whose limit is 4. Called with i in [4, 8), the check fails, records SQ_ERR_BOUNDS and skips the
// store; were the check missing, the store would still land inside the array.
__device__ unsigned int g_selftest_words[8];
__global__ void k_selftest_bounds(int i) {
    if (threadIdx.x == 0 && i >= 0 && i < 8 && SQ_CHECK(i < 4, &g_sq_status)) g_selftest_words[i] = 1u;
}
#endif

// ------------------------------------------------------------------------------------------------
// Host side.

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

sq_status get_encoder(EncodeTiledFn *out) {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return sq::fail(SQ_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
        f = reinterpret_cast<EncodeTiledFn>(p);
        fn.store(f, std::memory_order_release);
    }
    *out = f;
    return SQ_OK;
}

sq_status encode_2d(EncodeTiledFn enc, CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz,
                    const char *what) {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return sq::fail(SQ_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with CUresult %d", what, (int)r);
    return SQ_OK;
}

// Single-SM forms: one persistent CTA per SM at most. Plain: tiles of 128 tokens x TN channels (A =
// tokens, B = weight). SWAP: tiles of 128 channels x TN tokens (A = weight, B = tokens).
template <int TN, bool SWAP, bool F8>
sq_status launch_single(const CUtensorMap &mA, const CUtensorMap &mB, const CUtensorMap &mY, const float *x_scale,
                        const float *w_scale, const void *bias, int32_t *acc_out, void *y, int64_t T, int64_t N, int64_t K,
                        int dev, void *stream) {
    using L = Tile<TN, SWAP>;
    static std::atomic<int> configured[64];
    if (!configured[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(k_w8a8_linear<TN, SWAP, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_TOTAL);
        if (e != cudaSuccess) return sq::cuda_status(e, "cudaFuncSetAttribute(w8a8_linear)");
        configured[dev].store(1, std::memory_order_release);
    }
    const int64_t rows = SWAP ? N : T, cols = SWAP ? T : N;
    const int m_tiles = static_cast<int>((rows + BM - 1) / BM);
    const int n_tiles = static_cast<int>((cols + TN - 1) / TN);
    const int64_t tiles = static_cast<int64_t>(m_tiles) * n_tiles;
    if (tiles > 0x7FFFFFFF) return sq::fail(SQ_ERR_UNSUPPORTED, "sq_w8a8_linear: too many tiles");
    const int grid = static_cast<int>(tiles < sq::sm_count(dev) ? tiles : sq::sm_count(dev));
    return sq::cuda_status(
        sq::launch_pdl(k_w8a8_linear<TN, SWAP, F8>, dim3(grid), dim3(THREADS), L::SMEM_TOTAL, sq::as_stream(stream), nullptr,
                       mA, mB, mY, x_scale, w_scale, reinterpret_cast<const __nv_bfloat16 *>(bias), acc_out,
                       static_cast<__nv_bfloat16 *>(y), static_cast<int>(T), static_cast<int>(N), static_cast<int>(K), m_tiles,
                       n_tiles, band_for(N, K), sq::wait_timeout_ns(dev)),
        "launch(w8a8_linear)");
}

template <bool F8>
sq_status linear_impl(const void *xq, const float *x_scale, int64_t T, const void *wq, const float *w_scale, int64_t N,
                      int64_t K, const void *bias, void *y, void *acc_out_v, void *stream, const char *fn)
{
    int32_t *acc_out = static_cast<int32_t *>(acc_out_v);   // raw accumulator words (s32, or f32 bits)
    using sq::fail;
    if (T < 0 || N < 8 || K < 16) return fail(SQ_ERR_INVALID_ARG, "%s: need T >= 0, N >= 8, K >= 16", fn);
    if (!wq || !w_scale) return fail(SQ_ERR_INVALID_ARG, "%s: wq and w_scale are required", fn);
    if (T > 0 && (!xq || !x_scale || !y)) return fail(SQ_ERR_INVALID_ARG, "%s: xq, x_scale and y are required", fn);
    if (N % 8 != 0 || K % 16 != 0) return fail(SQ_ERR_MISALIGNED, "%s: N must be a multiple of 8 and K of 16", fn);
    if (K > 131072 || N > 0x7FFFFFFF || T > 0x7FFFFFFF)
        return fail(SQ_ERR_UNSUPPORTED, "%s: K must be <= 131072 and T, N < 2^31", fn);
    if ((xq && !sq::aligned(xq, 16)) || !sq::aligned(wq, 16) || (y && !sq::aligned(y, 16)) ||
        (acc_out && !sq::aligned(acc_out, 16)) || !sq::aligned(w_scale, 16) || (x_scale && !sq::aligned(x_scale, 4)) ||
        (bias && !sq::aligned(bias, 8)))
        return fail(SQ_ERR_MISALIGNED, "%s: xq, wq, y, acc_out, w_scale need 16-byte, bias 8-byte, x_scale 4-byte alignment", fn);
    int dev = 0;
    SQ_TRY_ARCH(dev);
    if (T == 0) return SQ_OK;

    EncodeTiledFn enc = nullptr;
    sq_status st = get_encoder(&enc);
    if (st != SQ_OK) return st;
    const bool pair = !F8 && g_cta_pair.load(std::memory_order_relaxed) != 0 && T >= 2 * BM;   // 256-row tiles on CTA pairs
    // 64-channel tiles when 256-channel tiles would leave SMs idle (few tokens: the weight stream
    // then bounds the call, and more tiles spread it over more SMs)
    // (192-channel tiles, which would fill the last wave better for some shapes, were measured slower:
    // with 40 KB of operands per 128 x 192 x 128 block against 48 KB per 128 x 256 x 128 the main loop
    // does not shrink with the tile width, so 1024 tiles of 192 took 92.3 us where 768 tiles of 256
    // took 84.0 us for the N = 6144, T = 4096, K = 4096 query-key-value projection.)
    const int64_t wide_tiles = ((T + BM - 1) / BM) * ((N + BN - 1) / BN);
    const bool narrow = !pair && wide_tiles < sq::sm_count(dev);
    CUtensorMap mA, mB, mY;
    if (!pair && T <= BM) {
        // Decode form: the weight streams as the 128-row operand, the tokens (padded to 16 .. 128
        // with zeros by the TMA) are the narrow one.
        const int tn = T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128;
        st = encode_2d(enc, &mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, K, N, K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B, "wq");
        if (st == SQ_OK) st = encode_2d(enc, &mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, K, T, K, BK, tn, CU_TENSOR_MAP_SWIZZLE_128B, "xq");
        if (st != SQ_OK) return st;
        switch (tn) {
            case 16: return launch_single<16, true, F8>(mA, mB, mA, x_scale, w_scale, bias, acc_out, y, T, N, K, dev, stream);
            case 32: return launch_single<32, true, F8>(mA, mB, mA, x_scale, w_scale, bias, acc_out, y, T, N, K, dev, stream);
            case 64: return launch_single<64, true, F8>(mA, mB, mA, x_scale, w_scale, bias, acc_out, y, T, N, K, dev, stream);
            default: return launch_single<128, true, F8>(mA, mB, mA, x_scale, w_scale, bias, acc_out, y, T, N, K, dev, stream);
        }
    }
    st = encode_2d(enc, &mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, K, T, K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B, "xq");
    if (st == SQ_OK) st = encode_2d(enc, &mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, K, N, K, BK, pair ? 128 : narrow ? 64 : BN, CU_TENSOR_MAP_SWIZZLE_128B, "wq");
    if (st == SQ_OK) st = encode_2d(enc, &mY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, T, N * 2, OUT_COLS, OUT_ROWS, CU_TENSOR_MAP_SWIZZLE_64B, "y");
    if (st != SQ_OK) return st;
    if (pair) {
        static std::atomic<int> pclusters[64];   // 0: not configured yet on this device
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(THREADS, 1, 1);
        cfg.dynamicSmemBytes = P_SMEM_TOTAL;
        cfg.stream = sq::as_stream(stream);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int npair = pclusters[dev].load(std::memory_order_acquire);
        if (npair == 0) {
            cudaError_t e = cudaFuncSetAttribute(k_w8a8_linear_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_TOTAL);
            if (e != cudaSuccess) return sq::cuda_status(e, "cudaFuncSetAttribute(w8a8_linear_pair)");
            cfg.gridDim = dim3(2, 1, 1);
            int nc = 0;
            e = cudaOccupancyMaxActiveClusters(&nc, k_w8a8_linear_pair, &cfg);
            if (e != cudaSuccess) return sq::cuda_status(e, "cudaOccupancyMaxActiveClusters(w8a8_linear_pair)");
            if (nc < 1) return sq::fail(SQ_ERR_CUDA, "no CTA pair of the GEMM fits on this device");
            npair = nc;
            pclusters[dev].store(nc, std::memory_order_release);
        }
        const int m_tiles = static_cast<int>((T + 2 * BM - 1) / (2 * BM));
        const int n_tiles = static_cast<int>((N + BN - 1) / BN);
        const int64_t tiles = static_cast<int64_t>(m_tiles) * n_tiles;
        if (tiles > 0x7FFFFFFF) return fail(SQ_ERR_UNSUPPORTED, "%s: too many tiles", fn);
        const int clusters = static_cast<int>(tiles < npair ? tiles : npair);
        return sq::cuda_status(
            sq::launch_pdl(k_w8a8_linear_pair, dim3(2 * clusters), dim3(THREADS), P_SMEM_TOTAL, sq::as_stream(stream), &attr[0],
                           mA, mB, mY, x_scale, w_scale, reinterpret_cast<const __nv_bfloat16 *>(bias), acc_out,
                           static_cast<int>(T), static_cast<int>(N), static_cast<int>(K), m_tiles, n_tiles,
                           band_for(N, K), sq::wait_timeout_ns(dev)),
            "launch(w8a8_linear_pair)");
    }

    return narrow ? launch_single<64, false, F8>(mA, mB, mY, x_scale, w_scale, bias, acc_out, y, T, N, K, dev, stream)
                  : launch_single<BN, false, F8>(mA, mB, mY, x_scale, w_scale, bias, acc_out, y, T, N, K, dev, stream);
}


}  // namespace

namespace sq {

unsigned int *device_status_word(int device) {
    static std::atomic<unsigned int *> addr[64];
    if (device < 0 || device >= 64) return nullptr;
    unsigned int *a = addr[device].load(std::memory_order_acquire);
    if (!a) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_sq_status) != cudaSuccess) return nullptr;
        a = static_cast<unsigned int *>(p);
        addr[device].store(a, std::memory_order_release);
    }
    return a;
}

}  // namespace sq

extern "C" {

sq_status sq_w8a8_linear(const int8_t *xq, const float *x_scale, int64_t T, const int8_t *wq,
                         const float *w_scale, int64_t N, int64_t K, const void *bias, void *y,
                         int32_t *acc_out, void *workspace, size_t workspace_bytes, void *stream)
{
    (void)workspace;
    (void)workspace_bytes;
    return linear_impl<false>(xq, x_scale, T, wq, w_scale, N, K, bias, y, acc_out, stream, "sq_w8a8_linear");
}

sq_status sq_w8a8_linear_fp8(const uint8_t *xq, const float *x_scale, int64_t T, const uint8_t *wq,
                             const float *w_scale, int64_t N, int64_t K, const void *bias, void *y,
                             float *acc_out, void *workspace, size_t workspace_bytes, void *stream)
{
    (void)workspace;
    (void)workspace_bytes;
    return linear_impl<true>(xq, x_scale, T, wq, w_scale, N, K, bias, y, acc_out, stream, "sq_w8a8_linear_fp8");
}

sq_status sq_set_gemm_cta_pair(int enable) {
    if (enable != 0 && enable != 1) return sq::fail(SQ_ERR_INVALID_ARG, "sq_set_gemm_cta_pair: enable must be 0 or 1");
    g_cta_pair.store(enable, std::memory_order_relaxed);
    return SQ_OK;
}

size_t sq_w8a8_linear_workspace_size(int64_t T, int64_t N, int64_t K) {
    (void)T;
    (void)N;
    (void)K;
    return 0;
}

sq_status sq_device_status(void *stream) {
    int dev = 0;
    SQ_TRY_ARCH(dev);
    cudaStream_t st = sq::as_stream(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return sq::cuda_status(e, "cudaStreamSynchronize");
    // read and clear in one atomic exchange: an error a kernel on another stream records meanwhile is
    // either reported now or stays in the word for the next call, never lost
    k_status_exchange<<<1, 1, 0, st>>>();
    e = cudaGetLastError();
    if (e != cudaSuccess) return sq::cuda_status(e, "launch(status_exchange)");
    unsigned int word = 0;
    e = cudaMemcpyFromSymbolAsync(&word, g_sq_status_read, sizeof word, 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return sq::cuda_status(e, "reading the status word");
    if (word != 0)
        return sq::fail(static_cast<sq_status>(word), "device status word reported %s", sq_status_string(static_cast<int>(word)));
    return SQ_OK;
}

sq_status sq_selftest_wait_timeout(void *stream) {
    int dev = 0;
    SQ_TRY_ARCH(dev);
    k_selftest_wait<<<1, 32, 0, sq::as_stream(stream)>>>(sq::wait_timeout_ns(dev));
    return sq::cuda_status(cudaGetLastError(), "launch(selftest_wait)");
}

sq_status sq_selftest_bounds_check(void *stream) {
    int dev = 0;
    SQ_TRY_ARCH(dev);
#ifdef SQ_DEVICE_CHECKS
    k_selftest_bounds<<<1, 32, 0, sq::as_stream(stream)>>>(5);
    return sq::cuda_status(cudaGetLastError(), "launch(selftest_bounds)");
#else
    (void)stream;
    return sq::fail(SQ_ERR_UNSUPPORTED, "sq_selftest_bounds_check: the library was built without device checks");
#endif
}

}  // extern "C"
