// Shared host-side helpers of the libzero C ABI: error reporting and
// argument checks.  No arithmetic of the method lives here.
#pragma once

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

}  // namespace zero
