// Host side of the staged step's update: validation, kernel choice and
// launch of the kernels in staged.cuh.  Included by every translation unit
// that launches them (the staged entry points and the step runner).
#pragma once

#include "staged.cuh"
#include "step_launch.h"

namespace zero {
namespace fused {
namespace {

// Tile of the pipeline kernel: 4 fp32 arrays x 4096 elements per stage
// (64 KB), 2 rounds of one 4-element chunk per consumer thread.  Measured on
// B200 (GPT-2 1.5B buckets): 6305 GB/s; 6144-element tiles 6092 GB/s.
constexpr int kReducedTile = 4096;

inline uint32_t reduced_pipe_smem_bytes(int tile) {
    return static_cast<uint32_t>(kReducedStages) * 16u * static_cast<uint32_t>(tile);
}

using ReducedKernelFn = void (*)(StepParams, ParamDsts);

inline ReducedKernelFn pick_reduced_kernel(zero_dtype_t pd, bool bcast) {
    if (bcast) return pd == ZERO_F16 ? adam_reduced_kernel<__half, true> : adam_reduced_kernel<__nv_bfloat16, true>;
    return pd == ZERO_F16 ? adam_reduced_kernel<__half, false> : adam_reduced_kernel<__nv_bfloat16, false>;
}

inline ReducedKernelFn pick_reduced_pipe_kernel(zero_dtype_t pd, bool bcast) {
    if (bcast)
        return pd == ZERO_F16 ? adam_reduced_pipe_kernel<__half, true> : adam_reduced_pipe_kernel<__nv_bfloat16, true>;
    return pd == ZERO_F16 ? adam_reduced_pipe_kernel<__half, false> : adam_reduced_pipe_kernel<__nv_bfloat16, false>;
}

struct ReducedDevice {
    int sms = 0;
    int blocks_per_sm[4] = {0, 0, 0, 0};        // [dtype * 2 + bcast]
    bool pipe_ready[4] = {false, false, false, false};
};

std::mutex g_red_mu;
ReducedDevice g_red[64];

// SM count, resident blocks of the register kernel, and the pipeline
// kernel's shared-memory limit, queried or set once per device, dtype and
// store mode.
inline int reduced_device(zero_dtype_t pd, bool bcast, ReducedDevice** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(ZERO_ERR_CUDA, "cudaGetDevice failed");
    std::lock_guard<std::mutex> lk(g_red_mu);
    ReducedDevice& d = g_red[dev];
    const int w = (pd == ZERO_F16 ? 0 : 2) + (bcast ? 1 : 0);
    if (d.sms == 0 && cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        d.sms = 0;
        return fail(ZERO_ERR_CUDA, "cannot query the SM count");
    }
    if (d.blocks_per_sm[w] == 0) {
        int n = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, pick_reduced_kernel(pd, bcast), kThreads, 0);
        if (e != cudaSuccess || n < 1) return fail(ZERO_ERR_CUDA, "occupancy query failed: %s", cudaGetErrorString(e));
        d.blocks_per_sm[w] = n;
    }
    if (!d.pipe_ready[w]) {
        cudaError_t e = cudaFuncSetAttribute(pick_reduced_pipe_kernel(pd, bcast),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(reduced_pipe_smem_bytes(kReducedTile)));
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "cannot raise the shared-memory limit: %s", cudaGetErrorString(e));
        d.pipe_ready[w] = true;
    }
    *out = &d;
    return ZERO_OK;
}

// Validate an update-from-reduced call and build its parameters;
// *work_out is the number of vector (or, with none, scalar) work items.
inline int prepare_reduced(const char* fn, const float* reduced, int64_t count, const float* master_in,
                           const float* m_in, const float* v_in, float* master_out, float* m_out, float* v_out,
                           void* param_out, zero_dtype_t param_dtype, const zero_adam_hparams_t* hp,
                           StepParams* prm_out, int64_t* work_out) {
    if (!hp) return fail(ZERO_ERR_ARG, "%s: NULL hp", fn);
    if (count < 0) return fail(ZERO_ERR_ARG, "%s: negative count", fn);
    if (param_dtype != ZERO_F16 && param_dtype != ZERO_BF16)
        return fail(ZERO_ERR_DTYPE, "%s: parameters must be ZERO_F16 or ZERO_BF16", fn);
    if (int rc = check_hparams(fn, hp)) return rc;
    if (count == 0) {
        *work_out = 0;
        return ZERO_OK;
    }
    const float* f_in[] = {master_in, m_in, v_in, reduced};
    float* f_out[] = {master_out, m_out, v_out};
    for (const float* a : f_in) {
        if (!a) return fail(ZERO_ERR_ARG, "%s: NULL input array", fn);
        if (!aligned(a, 4)) return fail(ZERO_ERR_ALIGN, "%s: fp32 input not 4-byte aligned", fn);
    }
    for (float* a : f_out) {
        if (!a) return fail(ZERO_ERR_ARG, "%s: NULL output array", fn);
        if (!aligned(a, 4)) return fail(ZERO_ERR_ALIGN, "%s: fp32 output not 4-byte aligned", fn);
    }
    if (!param_out) return fail(ZERO_ERR_ARG, "%s: NULL param_out", fn);
    if (!aligned(param_out, 2)) return fail(ZERO_ERR_ALIGN, "%s: param_out not 2-byte aligned", fn);
    // each output is its own input (in place) or overlaps nothing else
    const int64_t fb = count * 4;
    const void* outs[] = {master_out, m_out, v_out, param_out};
    const int64_t out_bytes[] = {fb, fb, fb, count * 2};
    for (int i = 0; i < 4; ++i) {
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(outs[i], out_bytes[i], outs[j], out_bytes[j]))
                return fail(ZERO_ERR_ARG, "%s: output arrays overlap", fn);
        for (int j = 0; j < 4; ++j)
            if (!(i == j && j < 3 && outs[i] == f_in[j]) && overlaps(outs[i], out_bytes[i], f_in[j], fb))
                return fail(ZERO_ERR_ARG, "%s: an output overlaps an input it does not replace", fn);
    }

    StepParams prm{};
    prm.world = 1;
    prm.grads[0] = reduced;
    prm.count = count;
    prm.master_in = master_in;
    prm.m_in = m_in;
    prm.v_in = v_in;
    prm.master_out = master_out;
    prm.m_out = m_out;
    prm.v_out = v_out;
    prm.param_out = param_out;
    prm.c = adam_consts(hp, 1.0f);
    // the first element at which every array sits on a 16-byte boundary
    int64_t h = -1;
    for (int64_t c = 0; c < kVec && h < 0; ++c) {
        bool good = ((reinterpret_cast<uintptr_t>(param_out) + 2 * c) % 16) == 0;
        const void* f32s[] = {reduced, master_in, m_in, v_in, master_out, m_out, v_out};
        for (const void* a : f32s) good = good && ((reinterpret_cast<uintptr_t>(a) + 4 * c) % 16) == 0;
        if (good) h = c;
    }
    if (h < 0 || h >= count) {
        prm.head = count;
        prm.nvec = 0;
    } else {
        prm.head = h;
        prm.nvec = (count - h) / kVec;
    }
    // 32-byte state stores when the fp32 outputs are 32-byte aligned at head
    prm.st32 = 0;
    if (prm.nvec > 0) {
        bool al = true;
        for (const float* a : {master_out, m_out, v_out})
            al = al && ((reinterpret_cast<uintptr_t>(a) + 4 * static_cast<uintptr_t>(h)) % 32) == 0;
        prm.st32 = al ? 1 : 0;
    }
    prm.tile = 0;
    *prm_out = prm;
    *work_out = prm.nvec > 0 ? prm.nvec : count;
    return ZERO_OK;
}

// Enqueue the update prepared by prepare_reduced: the register kernel (plain
// loads, 32-byte state stores where the outputs allow them, a grid of
// kRegWaves waves); the pipeline kernel only when zero_test_force_step_kernel
// asks for it.  Measured on B200 (fp32 reduced gradients in, 30 bytes per
// element, against a measured copy rate of 6.43 TB/s): 16M elements 0.93-0.96
// register against 0.87 pipeline, 64M 0.99 against 0.95, 256M-492M
// 0.99 against 0.98.  `work` as returned by prepare_reduced (> 0).
inline int launch_reduced(const char* fn, StepParams prm, const ParamDsts& d, int64_t work, zero_dtype_t pd,
                          bool bcast, zero_stream_t stream) {
    ReducedDevice* dev = nullptr;
    if (int rc = reduced_device(pd, bcast, &dev)) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t ntiles = prm.nvec > 0 ? (prm.count - prm.head) / kReducedTile : 0;
    const int force = step_kernel_override();
    const bool pipe = force == kKindPipe && ntiles >= 1;
    if (pipe) {
        // the pipeline kernel takes the whole tiles; the rest goes through
        // its scalar path
        prm.tile = kReducedTile;
        prm.nvec = ntiles * kReducedTile / kVec;
        pick_reduced_pipe_kernel(pd, bcast)<<<static_cast<unsigned int>(dev->sms), kPipeThreads,
                                             reduced_pipe_smem_bytes(kReducedTile), s>>>(prm, d);
    } else {
        const int w = (pd == ZERO_F16 ? 0 : 2) + (bcast ? 1 : 0);
        const int64_t limit = static_cast<int64_t>(kRegWaves) * dev->sms * dev->blocks_per_sm[w];
        int64_t blocks = (work + kThreads - 1) / kThreads;
        if (blocks > limit) blocks = limit;
        if (blocks > kMaxBlocks) blocks = kMaxBlocks;
        pick_reduced_kernel(pd, bcast)<<<static_cast<unsigned int>(blocks), kThreads, 0, s>>>(prm, d);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    return ZERO_OK;
}

}  // namespace
}  // namespace fused
}  // namespace zero
