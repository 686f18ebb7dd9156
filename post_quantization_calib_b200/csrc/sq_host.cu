// sq_host.cu -- status codes, error messages, device checks of libsq.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "sq_internal.h"

namespace sq {

namespace {
thread_local char g_last_error[512] = "";

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_arch_ok[kMaxDevices];    // 0 unknown, 1 ok, -1 wrong arch
int g_sms[kMaxDevices];
int g_l2[kMaxDevices];
uint64_t g_timeout_ns[kMaxDevices];
}  // namespace

sq_status fail(sq_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

sq_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return SQ_OK;
    return fail(SQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

sq_status check_arch(int *device_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(SQ_ERR_UNSUPPORTED, "device index %d out of range", dev);
    if (device_out) *device_out = dev;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_arch_ok[dev] == 1) return SQ_OK;
    }
    int major = 0, minor = 0, sms = 0, l2 = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaDeviceGetAttribute");
    std::lock_guard<std::mutex> lk(g_mu);
    if (major != 10 || minor != 0) {
        g_arch_ok[dev] = -1;
        return fail(SQ_ERR_ARCH, "device %d is compute capability %d.%d; libsq is built for 10.0 (sm_100a)",
                    dev, major, minor);
    }
    g_arch_ok[dev] = 1;
    g_sms[dev] = sms;
    g_l2[dev] = l2;
    if (g_timeout_ns[dev] == 0) g_timeout_ns[dev] = 2000000000ull;
    return SQ_OK;
}

int sm_count(int device) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_sms[device] > 0 ? g_sms[device] : 148;
}

double l2_bytes(int device) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_l2[device] > 0 ? static_cast<double>(g_l2[device]) : 126.0 * 1024 * 1024;
}

uint64_t wait_timeout_ns(int device) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_timeout_ns[device] ? g_timeout_ns[device] : 2000000000ull;
}

void set_wait_timeout_ns(int device, uint64_t ns) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_timeout_ns[device] = ns < 1000 ? 1000 : ns;
}

}  // namespace sq

extern "C" {

const char *sq_status_string(int status) {
    switch (status) {
        case SQ_OK: return "SQ_OK";
        case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG";
        case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED";
        case SQ_ERR_MISALIGNED: return "SQ_ERR_MISALIGNED";
        case SQ_ERR_ARCH: return "SQ_ERR_ARCH";
        case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
        case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT";
        case SQ_ERR_BOUNDS: return "SQ_ERR_BOUNDS";
        default: return "SQ_ERR_UNKNOWN";
    }
}

const char *sq_last_error(void) { return sq::g_last_error; }

const char *sq_version(void) { return "libsq 0.1 (sm_100a)"; }

sq_status sq_set_wait_timeout_ns(uint64_t ns) {
    int dev = 0;
    SQ_TRY_ARCH(dev);
    sq::set_wait_timeout_ns(dev, ns);
    return SQ_OK;
}

}  // extern "C"
