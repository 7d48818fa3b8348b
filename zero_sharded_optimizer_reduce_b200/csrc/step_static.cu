// zero_reduce_scatter_adam_step_noalloc: the fused step for callers that
// cannot allocate device memory.
//
// The only scratch the fused step needs is for the optional gradient
// square-norm: a ticket word and one partial sum per block.  The regular entry
// point takes it from a caller-provided workspace.  Some callers have no way
// to provide one: code running under an allocator that owns all device memory
// and forbids direct cudaMalloc calls, a latency-critical host thread that
// must not take cudaMalloc's implicit device synchronization, or a plain C
// caller that has no device allocator at hand.  For them this entry point
// keeps the scratch in a fixed array inside the library's own device image
// and allocates nothing.
//
// Limits and rules:
//  - the array holds the ticket and kStaticMaxBlocks (4096) fp64 partial
//    sums, 33,024 bytes; every GPU that loads the library holds it until exit;
//  - the fused kernels' grids are at most 16 blocks per SM (2368 blocks on a
//    B200), so any input size fits; a call whose grid would need more than
//    4096 blocks is rejected with ZERO_ERR_RANGE;
//  - every call on a device shares the array: calls that overlap on the GPU
//    (different streams, or several host threads) race on it;
//  - the first call on a device that asks for the norm looks up the array's
//    device address with cudaGetSymbolAddress (once per device, with that
//    device current); make that first call before any stream capture;
//  - no cudaMalloc, cudaFree or other allocating call is made.
#include "step_launch.h"

namespace zero {
namespace {

constexpr int64_t kStaticMaxBlocks = 4096;
constexpr size_t kStaticScratchBytes = fused::kWsPartialsOffset + sizeof(double) * kStaticMaxBlocks;

// Ticket word at offset 0, per-block partial sums from kWsPartialsOffset,
// the same layout as the caller-provided workspace.
static __device__ __align__(256) unsigned char g_step_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_step_scratch on the current device.  In host code the
// array's name is only a host-side handle, so the address is looked up once
// per device with that device current.
int scratch_address(const char* fn, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: cudaGetDevice failed: %s", fn, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(ZERO_ERR_CUDA, "%s: device %d beyond %d", fn, dev, kMaxDevices);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_step_scratch);
        if (e != cudaSuccess || !p)
            return fail(ZERO_ERR_CUDA, "%s: cudaGetSymbolAddress failed: %s", fn, cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return ZERO_OK;
}

}  // namespace
}  // namespace zero

using zero::fail;

extern "C" size_t zero_step_static_scratch_bytes(void) { return zero::kStaticScratchBytes; }

extern "C" int zero_reduce_scatter_adam_step_noalloc(
    const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
    zero_dtype_t grad_dtype, const float* master_in, const float* m_in, const float* v_in,
    float* master_out, float* m_out, float* v_out, void* param_out, zero_dtype_t param_dtype,
    const zero_adam_hparams_t* hp, float loss_scale, int32_t* overflow_flag, double* grad_sqnorm,
    zero_stream_t stream) {
    using namespace zero;
    using namespace zero::fused;
    const char* fn = "zero_reduce_scatter_adam_step_noalloc";
    // Validate with a placeholder workspace (aligned, never dereferenced): the
    // real scratch address is looked up only once the arguments are known good.
    void* const placeholder = reinterpret_cast<void*>(static_cast<uintptr_t>(256));
    StepParams prm{};
    int64_t blocks = 0;
    if (int rc = prepare_step(fn, grad_bufs, world, padded_numel, partition, grad_dtype, master_in, m_in, v_in,
                              master_out, m_out, v_out, param_out, param_dtype, hp, loss_scale, overflow_flag,
                              grad_sqnorm, grad_sqnorm ? placeholder : nullptr, &prm, &blocks))
        return rc;
    if (blocks == 0) return ok();
    if (grad_sqnorm) {
        if (blocks > kStaticMaxBlocks)
            return fail(ZERO_ERR_RANGE, "%s: the launch needs %lld partial sums, the static scratch holds %lld", fn,
                        (long long)blocks, (long long)kStaticMaxBlocks);
        void* scratch = nullptr;
        if (int rc = scratch_address(fn, &scratch)) return rc;
        // the ticket must start at zero; the partial sums need no clearing
        cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(unsigned int), reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: clearing the ticket failed: %s", fn, cudaGetErrorString(e));
        prm.ticket = static_cast<unsigned int*>(scratch);
        prm.partials = reinterpret_cast<double*>(static_cast<char*>(scratch) + kWsPartialsOffset);
    }
    return launch_step(fn, prm, blocks, grad_dtype, param_dtype, stream);
}
