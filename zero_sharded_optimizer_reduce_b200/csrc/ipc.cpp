// CUDA IPC plumbing for the multi-process ZeRO step: export a device buffer
// to the other ranks of a node and map theirs.  Each rank's fused kernel then
// reads its partition of every peer's gradient buffer directly (NVLink P2P
// loads between GPUs, plain loads within one GPU), in rank order, so the
// reduction keeps the fixed fp32 order of the single-GPU path.
//
// Host only.  cudaIpcGetMemHandle needs the base of an allocation; buffers
// from a caching allocator sit inside larger blocks, so the export records
// the offset from the base, found with the driver's address-range query
// (obtained through cudaGetDriverEntryPoint: the library needs no link
// against the driver library and still loads on a machine without a GPU).
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "common.h"

namespace zero {
namespace {

using CUdeviceptr_t = unsigned long long;
using GetAddressRangeFn = int (*)(CUdeviceptr_t* base, size_t* size, CUdeviceptr_t dptr);

std::mutex g_ipc_mu;
GetAddressRangeFn g_get_range = nullptr;

int address_range(const char* fn, const void* ptr, CUdeviceptr_t* base, size_t* size) {
    std::lock_guard<std::mutex> lk(g_ipc_mu);
    if (!g_get_range) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        cudaError_t e = cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q);
        if (e != cudaSuccess || !f || q != cudaDriverEntryPointSuccess)
            return fail(ZERO_ERR_CUDA, "%s: cuMemGetAddressRange unavailable: %s", fn, cudaGetErrorString(e));
        g_get_range = reinterpret_cast<GetAddressRangeFn>(f);
    }
    int rc = g_get_range(base, size, reinterpret_cast<CUdeviceptr_t>(ptr));
    if (rc != 0) return fail(ZERO_ERR_CUDA, "%s: address-range query failed (driver error %d)", fn, rc);
    return ZERO_OK;
}

}  // namespace
}  // namespace zero

using zero::fail;

extern "C" int zero_ipc_export(const void* ptr, zero_ipc_handle_t* handle, int64_t* offset) {
    const char* fn = "zero_ipc_export";
    if (!ptr || !handle || !offset) return fail(ZERO_ERR_ARG, "%s: NULL argument", fn);
    zero::CUdeviceptr_t base = 0;
    size_t size = 0;
    if (int rc = zero::address_range(fn, ptr, &base, &size)) return rc;
    cudaIpcMemHandle_t h;
    cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: cudaIpcGetMemHandle failed: %s", fn, cudaGetErrorString(e));
    static_assert(sizeof(h) == sizeof(handle->bytes), "IPC handle size");
    std::memcpy(handle->bytes, &h, sizeof h);
    *offset = static_cast<int64_t>(reinterpret_cast<zero::CUdeviceptr_t>(ptr) - base);
    return zero::ok();
}

extern "C" int zero_ipc_import(const zero_ipc_handle_t* handle, int64_t offset, void** ptr, void** base) {
    const char* fn = "zero_ipc_import";
    if (!handle || !ptr || !base || offset < 0) return fail(ZERO_ERR_ARG, "%s: bad argument", fn);
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle->bytes, sizeof h);
    void* b = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: cudaIpcOpenMemHandle failed: %s", fn, cudaGetErrorString(e));
    *base = b;
    *ptr = static_cast<char*>(b) + offset;
    return zero::ok();
}

extern "C" int zero_ipc_close(void* base) {
    const char* fn = "zero_ipc_close";
    if (!base) return fail(ZERO_ERR_ARG, "%s: NULL base", fn);
    cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: cudaIpcCloseMemHandle failed: %s", fn, cudaGetErrorString(e));
    return zero::ok();
}
