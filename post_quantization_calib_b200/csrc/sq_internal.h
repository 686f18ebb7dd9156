// sq_internal.h -- host-side helpers shared by the libsq translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sq.h"

namespace sq {

// Records a one-line reason for `st` (thread-local) and returns st.
sq_status fail(sq_status st, const char *fmt, ...);

// Checks that the current device is compute capability 10.0; caches per device.
sq_status check_arch(int *device_out = nullptr);

// SM count of the current device (cached).
int sm_count(int device);

// L2 cache size in bytes of the current device (cached).
double l2_bytes(int device);

// cudaError_t -> SQ_OK / SQ_ERR_CUDA with the CUDA error text recorded.
sq_status cuda_status(cudaError_t e, const char *what);

// Device address of the status word (SQ_OK or the first error a kernel recorded) on `device`,
// which must be the current device. NULL if it cannot be resolved.
unsigned int *device_status_word(int device);

// Per-device limit of bounded device-side waits, in ns.
uint64_t wait_timeout_ns(int device);
void set_wait_timeout_ns(int device, uint64_t ns);

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Launch with programmatic stream serialisation (the kernel may start while the previous kernel of the
// stream finishes; it calls pdl_wait() before touching global memory shared with earlier work).
// `extra` (nullable) adds one more launch attribute, e.g. a cluster shape.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       const cudaLaunchAttribute *extra, Args... args) {
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    unsigned n = 1;
    if (extra != nullptr) attr[n++] = *extra;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace sq

#define SQ_TRY_ARCH(dev)                        \
    do {                                        \
        sq_status _st = sq::check_arch(&(dev)); \
        if (_st != SQ_OK) return _st;           \
    } while (0)
