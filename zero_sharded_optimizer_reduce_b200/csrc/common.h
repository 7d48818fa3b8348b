// Shared host-side helpers of the libzero C ABI: error reporting and
// argument checks.  No arithmetic of the method lives here.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <string>

#include "zero.h"

namespace zero {

// Record `msg` as the calling thread's last error and return `code`.
int fail(int code, const char* fmt, ...);

// Clear the calling thread's last error and return ZERO_OK.
int ok();

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int dtype_size(zero_dtype_t d) {
    switch (d) {
        case ZERO_F16:
        case ZERO_BF16: return 2;
        case ZERO_F32: return 4;
        default: return 0;
    }
}

// True when byte ranges [a, a+na) and [b, b+nb) share at least one byte.
inline bool overlaps(const void* a, int64_t na, const void* b, int64_t nb) {
    if (na <= 0 || nb <= 0) return false;
    auto x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + static_cast<uintptr_t>(nb) && y < x + static_cast<uintptr_t>(na);
}

// Step-kernel override of zero_test_force_step_kernel (-1: the automatic
// choice), shared by every translation unit that prepares a step launch.
int step_kernel_override();

// True when `p` is device memory of device `dev` (not another GPU's memory
// mapped into this process, not host memory).  Kernels that stage their
// inputs with bulk copies take only such sources; other sources go to the
// kernels that read with plain loads.  A failed query counts as "not local"
// and its error is cleared, so that a launch check that follows is not
// misled.
inline bool local_device_memory(const void* p, int dev) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice && a.device == dev;
}

// True when every one of the n pointers is device memory of the current device.
inline bool all_local_device_memory(const void* const* ptrs, int n) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    for (int i = 0; i < n; ++i)
        if (!local_device_memory(ptrs[i], dev)) return false;
    return true;
}

}  // namespace zero
