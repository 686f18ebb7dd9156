// sq_device.cuh -- device-side building blocks shared by the libsq kernels (sm_100a):
// mbarriers with bounded waits, TMA bulk copies, named barriers, packed binary32 arithmetic.
#pragma once

#include <stdint.h>

#include "sq.h"

// Device-side bounds checks. A build with SQ_DEVICE_CHECKS defined (libsq_checked.so) evaluates
// each SQ_CHECK(ok, status): a false `ok` records SQ_ERR_BOUNDS in the device status word (the first
// error recorded is kept) and the caller skips the access the check guards, so a wrong index shows
// up as a status from sq_device_status instead of a fault. In the product build SQ_CHECK is the
// constant true and its arguments are not compiled at all.
#ifdef SQ_DEVICE_CHECKS
static __device__ __forceinline__ bool sq_check_record(bool ok, unsigned int *status) {
    if (!ok) atomicCAS(status, 0u, static_cast<unsigned int>(SQ_ERR_BOUNDS));
    return ok;
}
#define SQ_CHECK(ok, status) sq_check_record((ok), (status))
#else
#define SQ_CHECK(ok, status) true
#endif

// Every helper is `static` (internal linkage): each translation unit keeps its own copy.
namespace sqdev {

static __device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------- mbarriers
static __device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
static __device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
static __device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
static __device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
static __device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
static __device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the phase of `bar` with parity `parity` has completed. Returns false when `limit_ns`
// elapsed first or (when `abort_flag` is given) another role of the CTA gave up. Never unbounded.
static __device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                       const volatile int *abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 127u) == 0u) {
            if (abort_flag && *abort_flag) return false;
            if (global_ns() - t0 > limit_ns) return false;
        }
    }
}

// mbar_wait with the common case (phase already complete) inlined.
static __device__ __forceinline__ bool mbar_ready(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                                  const volatile int *abort_flag) {
    return mbar_try(bar, parity) || mbar_wait(bar, parity, limit_ns, abort_flag);
}

// ---------------------------------------------------------------------------------- TMA bulk copy
// Global -> shared copy of `bytes` (multiple of 16; both addresses 16-byte aligned), completion
// counted on the mbarrier's transaction count. Destination is this CTA's own shared memory.
static __device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Orders this thread's earlier shared-memory accesses (generic proxy) before its later TMA
// (async proxy) accesses to shared memory.
static __device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// bulk_g2s with an L2 cache-policy hint (a policy made by createpolicy).
static __device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar, uint64_t policy) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(policy)
                 : "memory");
}
// L2 policy that marks the lines it touches first in line for eviction (data read once).
static __device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// ---------------------------------------------------------------------------------- dependent launch
// Programmatic dependent launch: every libsq kernel is launched so that it may start while the
// kernel before it in the stream is finishing. pdl_wait() returns once every earlier grid of the
// stream has completed and its memory is visible; a kernel touches no global memory it shares with
// earlier work before it (only shared memory, tensor memory and its parameters). pdl_trigger() lets
// the next kernel of the stream start; every libsq grid fits in one wave (all its CTAs resident at
// once), so the next kernel's CTAs never hold SMs this grid still needs. Both are no-ops when the
// kernel was launched without the attribute.
static __device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
static __device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------------- barriers
static __device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Barrier over `nthreads` threads that also returns whether `pred` held in any of them.
static __device__ __forceinline__ bool named_sync_or(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %3, 0;\n\t"
        "bar.red.or.pred q, %1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(id), "r"(nthreads), "r"(pred ? 1u : 0u)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------------------------- packed binary32
// Two binary32 values in one 64-bit register: low half = first element.
// (register-pair moves, so that no 64-bit integer shift or or is emitted)
static __device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
static __device__ __forceinline__ uint64_t pack2u(uint32_t lo, uint32_t hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
    return d;
}
static __device__ __forceinline__ void unpack2(uint64_t v, uint32_t &lo, uint32_t &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
static __device__ __forceinline__ float lo2(uint64_t v) {
    uint32_t l, h;
    unpack2(v, l, h);
    return __uint_as_float(l);
}
static __device__ __forceinline__ float hi2(uint64_t v) {
    uint32_t l, h;
    unpack2(v, l, h);
    return __uint_as_float(h);
}
static __device__ __forceinline__ uint64_t mul2_rn(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
static __device__ __forceinline__ uint64_t add2_rn(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// fl(a + b) for both halves with scalar round-to-nearest adds, which the compiler never contracts
// with a preceding multiply into a fused multiply-add (a packed add after a packed multiply can be
// contracted, so a sum that must be rounded on its own uses this form).
static __device__ __forceinline__ uint64_t add2_scalar(uint64_t a, uint64_t b) {
    uint32_t al, ah, bl, bh;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(al), "=r"(ah) : "l"(a));
    asm("mov.b64 {%0, %1}, %2;" : "=r"(bl), "=r"(bh) : "l"(b));
    return pack2(__fadd_rn(__uint_as_float(al), __uint_as_float(bl)), __fadd_rn(__uint_as_float(ah), __uint_as_float(bh)));
}
static __device__ __forceinline__ uint64_t add2_rz(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
static __device__ __forceinline__ uint64_t fma2_rn(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// high 32 bits of a * b, plus c
static __device__ __forceinline__ uint32_t mad_hi(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

}  // namespace sqdev
