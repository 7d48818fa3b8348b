// Self-test of the pipeline kernel's bounded waits.
//
// The shared-memory pipeline waits on mbarriers that its own bulk copies
// complete.  If a wait never ends (a device fault), the kernel must give up
// after a time limit, report it through the flag word and return, leaving
// the context usable.  This entry point runs that exact wait routine on an
// mbarrier that nothing arrives at, so the give-up path can be tested
// without making anything fail.
#include "step_launch.h"

using zero::fail;

extern "C" int zero_test_wait_timeout(int32_t* status, int64_t limit_ns, zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_test_wait_timeout";
    if (!status) return fail(ZERO_ERR_ARG, "%s: NULL status", fn);
    if (!zero::aligned(status, 4)) return fail(ZERO_ERR_ALIGN, "%s: status misaligned", fn);
    if (limit_ns < 0 || limit_ns > 10000000000LL) return fail(ZERO_ERR_ARG, "%s: limit_ns outside 0..1e10", fn);
    wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, static_cast<uint64_t>(limit_ns));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    return zero::ok();
}
