// Host side of the fused step: argument validation, kernel choice, grid
// sizing and launch.  Included by every translation unit that launches the
// kernels of fused_step.cuh.
#pragma once

#include <mutex>

#include "fused_step.cuh"
#include "grad_stats.cuh"

namespace zero {
namespace fused {
namespace {

constexpr uint32_t kPipeSmemTarget = 180u * 1024u;  // shared memory of both stages, at most
constexpr uint32_t kPipeMinTile = 1536;             // elements: 3/4 of 4 x consumer threads
constexpr uint32_t kPipeSmemMax = 220u * 1024u;     // dynamic shared memory cap
constexpr int kPipeMaxWorld = 20;                   // largest N measured to gain from the pipeline
constexpr int64_t kPipeMinTilesPerSm = 128;         // calls with fewer tiles per SM take the oct / quad kernel
constexpr int kRegMaxWorldLarge = 5;                // large calls with 3 <= N <= this take the register kernel
constexpr int64_t kStatsPipeMinTilesPerSm = 128;    // the same for the staged reduce-scatter
constexpr int kStatsPipeMaxWorldWrite = 8;          // largest N whose reduce-scatter takes that pipeline

using KernelFn = void (*)(StepParams);
using StatsKernelFn = void (*)(StepParams, float*);

inline KernelFn pick_kernel(zero_dtype_t g, zero_dtype_t pd) {
    if (g == ZERO_F16 && pd == ZERO_F16) return fused_step_kernel<__half, __half>;
    if (g == ZERO_F16 && pd == ZERO_BF16) return fused_step_kernel<__half, __nv_bfloat16>;
    if (g == ZERO_BF16 && pd == ZERO_F16) return fused_step_kernel<__nv_bfloat16, __half>;
    return fused_step_kernel<__nv_bfloat16, __nv_bfloat16>;
}

// write: the staged reduce-scatter variant that also stores the unscaled
// gradients
inline StatsKernelFn pick_stats_kernel(zero_dtype_t g, bool write) {
    if (write) return g == ZERO_F16 ? grad_stats_kernel<__half, true> : grad_stats_kernel<__nv_bfloat16, true>;
    return g == ZERO_F16 ? grad_stats_kernel<__half, false> : grad_stats_kernel<__nv_bfloat16, false>;
}

inline StatsKernelFn pick_stats_pipe_kernel(zero_dtype_t g, bool write) {
    if (write)
        return g == ZERO_F16 ? grad_stats_pipe_kernel<__half, true> : grad_stats_pipe_kernel<__nv_bfloat16, true>;
    return g == ZERO_F16 ? grad_stats_pipe_kernel<__half, false> : grad_stats_pipe_kernel<__nv_bfloat16, false>;
}

template <int B>
inline KernelFn pick_quad_b(zero_dtype_t g, zero_dtype_t pd) {
    constexpr int U = QuadShape<B>::U, NT = QuadShape<B>::NT;
    if (g == ZERO_F16 && pd == ZERO_F16) return fused_step_quad_kernel<__half, __half, B, U, NT>;
    if (g == ZERO_F16 && pd == ZERO_BF16) return fused_step_quad_kernel<__half, __nv_bfloat16, B, U, NT>;
    if (g == ZERO_BF16 && pd == ZERO_F16) return fused_step_quad_kernel<__nv_bfloat16, __half, B, U, NT>;
    return fused_step_quad_kernel<__nv_bfloat16, __nv_bfloat16, B, U, NT>;
}

// The quad-kernel instance for N replicas (N <= kQuadMaxWorld), its threads
// per block and quads per thread and iteration.
inline KernelFn pick_quad_kernel(zero_dtype_t g, zero_dtype_t pd, int world, int* nt, int* u) {
    if (world <= 2) { *nt = QuadShape<2>::NT; *u = QuadShape<2>::U; return pick_quad_b<2>(g, pd); }
    if (world <= 4) { *nt = QuadShape<4>::NT; *u = QuadShape<4>::U; return pick_quad_b<4>(g, pd); }
    if (world <= 8) { *nt = QuadShape<8>::NT; *u = QuadShape<8>::U; return pick_quad_b<8>(g, pd); }
    *nt = QuadShape<16>::NT;
    *u = QuadShape<16>::U;
    return pick_quad_b<16>(g, pd);
}

template <int B>
inline StatsKernelFn pick_stats_quad_b(zero_dtype_t g, bool write) {
    constexpr int U = StatsQuadShape<B>::U, NT = StatsQuadShape<B>::NT;
    if (write)
        return g == ZERO_F16 ? grad_stats_quad_kernel<__half, true, B, U, NT>
                             : grad_stats_quad_kernel<__nv_bfloat16, true, B, U, NT>;
    return g == ZERO_F16 ? grad_stats_quad_kernel<__half, false, B, U, NT>
                         : grad_stats_quad_kernel<__nv_bfloat16, false, B, U, NT>;
}

// The quad statistics kernel for N replicas (N <= kQuadMaxWorld), its threads
// per block and quads per thread and iteration.
inline StatsKernelFn pick_stats_quad_kernel(zero_dtype_t g, bool write, int world, int* nt, int* u) {
    if (world <= 1) { *nt = StatsQuadShape<1>::NT; *u = StatsQuadShape<1>::U; return pick_stats_quad_b<1>(g, write); }
    if (world <= 2) { *nt = StatsQuadShape<2>::NT; *u = StatsQuadShape<2>::U; return pick_stats_quad_b<2>(g, write); }
    if (world <= 4) { *nt = StatsQuadShape<4>::NT; *u = StatsQuadShape<4>::U; return pick_stats_quad_b<4>(g, write); }
    if (world <= 8) { *nt = StatsQuadShape<8>::NT; *u = StatsQuadShape<8>::U; return pick_stats_quad_b<8>(g, write); }
    *nt = StatsQuadShape<16>::NT;
    *u = StatsQuadShape<16>::U;
    return pick_stats_quad_b<16>(g, write);
}

template <int B>
inline KernelFn pick_oct_b(zero_dtype_t g, zero_dtype_t pd) {
    constexpr int NT = OctShape<B>::NT, M = OctShape<B>::MINB;
    if (g == ZERO_F16 && pd == ZERO_F16) return fused_step_oct_kernel<__half, __half, B, NT, M>;
    if (g == ZERO_F16 && pd == ZERO_BF16) return fused_step_oct_kernel<__half, __nv_bfloat16, B, NT, M>;
    if (g == ZERO_BF16 && pd == ZERO_F16) return fused_step_oct_kernel<__nv_bfloat16, __half, B, NT, M>;
    return fused_step_oct_kernel<__nv_bfloat16, __nv_bfloat16, B, NT, M>;
}

// The oct-kernel instance for N replicas (N <= kQuadMaxWorld), its threads
// per block and the blocks per SM of its grid.
inline KernelFn pick_oct_kernel(zero_dtype_t g, zero_dtype_t pd, int world, int* nt, int* bps) {
    if (world <= 2) { *nt = OctShape<2>::NT; *bps = OctShape<2>::BPS; return pick_oct_b<2>(g, pd); }
    if (world <= 4) { *nt = OctShape<4>::NT; *bps = OctShape<4>::BPS; return pick_oct_b<4>(g, pd); }
    if (world <= 8) { *nt = OctShape<8>::NT; *bps = OctShape<8>::BPS; return pick_oct_b<8>(g, pd); }
    *nt = OctShape<16>::NT;
    *bps = OctShape<16>::BPS;
    return pick_oct_b<16>(g, pd);
}

// The oct reduce-scatter for N <= 2, its threads per block and octs per
// thread and iteration.
inline StatsKernelFn pick_rs_oct_kernel(zero_dtype_t g, int world, int* nt, int* u) {
    if (world <= 1) {
        *nt = RsOctShape<1>::NT;
        *u = RsOctShape<1>::U;
        return g == ZERO_F16 ? grad_rs_oct_kernel<__half, 1, RsOctShape<1>::U, RsOctShape<1>::NT>
                             : grad_rs_oct_kernel<__nv_bfloat16, 1, RsOctShape<1>::U, RsOctShape<1>::NT>;
    }
    *nt = RsOctShape<2>::NT;
    *u = RsOctShape<2>::U;
    return g == ZERO_F16 ? grad_rs_oct_kernel<__half, 2, RsOctShape<2>::U, RsOctShape<2>::NT>
                         : grad_rs_oct_kernel<__nv_bfloat16, 2, RsOctShape<2>::U, RsOctShape<2>::NT>;
}

inline KernelFn pick_pipe_kernel(zero_dtype_t g, zero_dtype_t pd) {
    if (g == ZERO_F16 && pd == ZERO_F16) return fused_step_pipe_kernel<__half, __half>;
    if (g == ZERO_F16 && pd == ZERO_BF16) return fused_step_pipe_kernel<__half, __nv_bfloat16>;
    if (g == ZERO_BF16 && pd == ZERO_F16) return fused_step_pipe_kernel<__nv_bfloat16, __half>;
    return fused_step_pipe_kernel<__nv_bfloat16, __nv_bfloat16>;
}

// Pipeline tile for N replicas: the largest multiple of 512 elements whose
// two stages fit in kPipeSmemTarget, for N <= kPipeMaxWorld; 0 (the
// register kernel runs) otherwise.  Measured on B200: large stages and tiles
// that split evenly into rounds of 4 elements per consumer thread run
// fastest (N = 8: T = 3072, 6.96 TB/s; T = 2304, 6.07 TB/s); above N = 20
// the register kernel is faster than the small tiles that would fit.
inline int pipe_tile(int world) {
    if (world > kPipeMaxWorld) return 0;
    const uint32_t per_elem = 2u * static_cast<uint32_t>(world) + 12u;
    uint32_t t = kPipeSmemTarget / (static_cast<uint32_t>(kPipeStages) * per_elem) / 512u * 512u;
    if (t > 8192u) t = 8192u;
    if (t < kPipeMinTile) return 0;
    if (static_cast<uint64_t>(kPipeStages) * t * per_elem > kPipeSmemMax) return 0;
    return static_cast<int>(t);
}

// Tile of the statistics pipeline (stages hold gradients only, 2N bytes per
// element): the same rule as pipe_tile.
inline int stats_pipe_tile(int world) {
    if (world > kPipeMaxWorld) return 0;
    const uint32_t per_elem = 2u * static_cast<uint32_t>(world);
    uint32_t t = kPipeSmemTarget / (static_cast<uint32_t>(kPipeStages) * per_elem) / 512u * 512u;
    if (t > 8192u) t = 8192u;
    if (t < kPipeMinTile) return 0;
    return static_cast<int>(t);
}

inline uint32_t stats_pipe_smem_bytes(int world, int tile) {
    return static_cast<uint32_t>(kPipeStages) * static_cast<uint32_t>(tile) * 2u * static_cast<uint32_t>(world);
}

inline uint32_t pipe_smem_bytes(int world, int tile) {
    return static_cast<uint32_t>(kPipeStages) * static_cast<uint32_t>(tile) * (2u * static_cast<uint32_t>(world) + 12u);
}

struct DeviceInfo {
    int sms = 0;
    int blocks_per_sm[4] = {0, 0, 0, 0};
    int stats_blocks_per_sm[4] = {0, 0, 0, 0};   // [dtype * 2 + write]
    bool pipe_ready[4] = {false, false, false, false};
    bool stats_pipe_ready[4] = {false, false, false, false};
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

inline int device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return fail(ZERO_ERR_CUDA, "cudaGetDevice failed");
    DeviceInfo& d = g_dev[dev];
    if (d.sms == 0) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return fail(ZERO_ERR_CUDA, "cannot query the SM count");
    }
    *out = &d;
    return ZERO_OK;
}

inline int grid_limit(zero_dtype_t g, zero_dtype_t pd, int* out) {
    const int which = static_cast<int>(g) * 2 + static_cast<int>(pd);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo* d = nullptr;
    if (int rc = device_info(&d)) return rc;
    if (d->blocks_per_sm[which] == 0) {
        int n = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, pick_kernel(g, pd), kThreads, 0);
        if (e != cudaSuccess || n < 1) return fail(ZERO_ERR_CUDA, "occupancy query failed: %s", cudaGetErrorString(e));
        d->blocks_per_sm[which] = n;
    }
    int lim = kRegWaves * d->sms * d->blocks_per_sm[which];
    *out = lim < kMaxBlocks ? lim : kMaxBlocks;
    return ZERO_OK;
}

inline int stats_grid_limit(zero_dtype_t g, bool write, int* out) {
    const int which = static_cast<int>(g) * 2 + (write ? 1 : 0);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo* d = nullptr;
    if (int rc = device_info(&d)) return rc;
    if (d->stats_blocks_per_sm[which] == 0) {
        int n = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, pick_stats_kernel(g, write), kThreads, 0);
        if (e != cudaSuccess || n < 1) return fail(ZERO_ERR_CUDA, "occupancy query failed: %s", cudaGetErrorString(e));
        d->stats_blocks_per_sm[which] = n;
    }
    int lim = kRegWaves * d->sms * d->stats_blocks_per_sm[which];
    *out = lim < kMaxBlocks ? lim : kMaxBlocks;
    return ZERO_OK;
}

// SM count, and the pipeline kernel's shared-memory limit raised once per
// device and dtype pair.
inline int pipe_setup(zero_dtype_t g, zero_dtype_t pd, int* sms) {
    const int which = static_cast<int>(g) * 2 + static_cast<int>(pd);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo* d = nullptr;
    if (int rc = device_info(&d)) return rc;
    if (!d->pipe_ready[which]) {
        cudaError_t e = cudaFuncSetAttribute(pick_pipe_kernel(g, pd), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kPipeSmemMax));
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "cannot raise the shared-memory limit: %s", cudaGetErrorString(e));
        d->pipe_ready[which] = true;
    }
    *sms = d->sms;
    return ZERO_OK;
}

// Smallest h in [0, kVec) at which every array sits on a 16-byte boundary,
// or -1 if their phases never coincide.
inline int64_t common_phase(const StepParams& p) {
    for (int64_t h = 0; h < kVec; ++h) {
        bool good = true;
        for (int k = 0; k < p.world && good; ++k)
            good = ((reinterpret_cast<uintptr_t>(p.grads[k]) + 2 * h) % 16) == 0;
        const void* f32s[] = {p.master_in, p.m_in, p.v_in, p.master_out, p.m_out, p.v_out};
        for (const void* a : f32s) good = good && ((reinterpret_cast<uintptr_t>(a) + 4 * h) % 16) == 0;
        good = good && ((reinterpret_cast<uintptr_t>(p.param_out) + 2 * h) % 16) == 0;
        if (good) return h;
    }
    return -1;
}


// Range checks of the Adam hyper-parameters shared by every update call.
inline int check_hparams(const char* fn, const zero_adam_hparams_t* hp) {
    if (!(hp->step >= 1)) return fail(ZERO_ERR_ARG, "%s: hp->step must be >= 1", fn);
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay) ||
        !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) ||
        !(hp->grad_divisor >= 0.0f) || !std::isfinite(hp->grad_divisor))
        return fail(ZERO_ERR_ARG, "%s: hyper-parameters out of range", fn);
    return ZERO_OK;
}

// The update's constants for step hp->step: each computed in double and
// rounded once to float; `inv` multiplies the incoming gradient.
inline Consts adam_consts(const zero_adam_hparams_t* hp, float inv) {
    const double t = static_cast<double>(hp->step);
    Consts c{};
    c.lr = hp->lr;
    c.b1 = hp->beta1;
    c.b2 = hp->beta2;
    c.eps = hp->eps;
    c.inv = inv;
    c.omb1 = static_cast<float>(1.0 - static_cast<double>(hp->beta1));
    c.omb2 = static_cast<float>(1.0 - static_cast<double>(hp->beta2));
    c.rbc1 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(hp->beta1), t)));
    c.rsbc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(hp->beta2), t)));
    c.decay = static_cast<float>(1.0 - static_cast<double>(hp->lr) * static_cast<double>(hp->weight_decay));
    c.clip = 1.0f;
    return c;
}

// Validate the arguments of a fused-step call and build its kernel
// parameters and grid size.  `workspace` is the scratch used for the
// gradient norm (ticket + per-block partials).  On success *blocks_out is the
// number of blocks to launch (0: nothing to do).
inline int prepare_step(const char* fn, const void* const* grad_bufs, int32_t world, int64_t padded_numel,
                        int32_t partition, zero_dtype_t grad_dtype, const float* master_in, const float* m_in,
                        const float* v_in, float* master_out, float* m_out, float* v_out, void* param_out,
                        zero_dtype_t param_dtype, const zero_adam_hparams_t* hp, float loss_scale,
                        int32_t* overflow_flag, double* grad_sqnorm, void* workspace, StepParams* prm_out,
                        int64_t* blocks_out) {
    if (!grad_bufs || !hp || !overflow_flag) return fail(ZERO_ERR_ARG, "%s: NULL grad_bufs, hp or overflow_flag", fn);
    if (world < 1 || world > ZERO_MAX_WORLD)
        return fail(ZERO_ERR_ARG, "%s: world %d outside 1..%d", fn, world, ZERO_MAX_WORLD);
    if (padded_numel < 0 || padded_numel % world != 0)
        return fail(ZERO_ERR_ARG, "%s: padded_numel %lld is not a non-negative multiple of world %d", fn,
                    (long long)padded_numel, world);
    if (partition != ZERO_ALL_PARTITIONS && (partition < 0 || partition >= world))
        return fail(ZERO_ERR_RANGE, "%s: partition %d outside 0..%d", fn, partition, world - 1);
    if ((grad_dtype != ZERO_F16 && grad_dtype != ZERO_BF16) || (param_dtype != ZERO_F16 && param_dtype != ZERO_BF16))
        return fail(ZERO_ERR_DTYPE, "%s: gradients and parameters must be ZERO_F16 or ZERO_BF16", fn);
    if (int rc = check_hparams(fn, hp)) return rc;
    if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale))
        return fail(ZERO_ERR_ARG, "%s: loss_scale must be positive and finite", fn);
    if (grad_sqnorm && !workspace) return fail(ZERO_ERR_ARG, "%s: grad_sqnorm needs a workspace", fn);
    if (!aligned(overflow_flag, 4) || (grad_sqnorm && !aligned(grad_sqnorm, 8)) ||
        (workspace && !aligned(workspace, 16)))
        return fail(ZERO_ERR_ALIGN, "%s: flag, norm or workspace misaligned", fn);

    const int64_t P = padded_numel / world;
    const int64_t begin = partition == ZERO_ALL_PARTITIONS ? 0 : static_cast<int64_t>(partition) * P;
    const int64_t count = partition == ZERO_ALL_PARTITIONS ? padded_numel : P;
    if (count == 0) {
        *blocks_out = 0;
        return ZERO_OK;
    }

    const float* f_in[] = {master_in, m_in, v_in};
    float* f_out[] = {master_out, m_out, v_out};
    for (int i = 0; i < 3; ++i) {
        if (!f_in[i] || !f_out[i]) return fail(ZERO_ERR_ARG, "%s: NULL state pointer", fn);
        if (!aligned(f_in[i], 4) || !aligned(f_out[i], 4)) return fail(ZERO_ERR_ALIGN, "%s: fp32 state not 4-byte aligned", fn);
    }
    if (!param_out) return fail(ZERO_ERR_ARG, "%s: NULL param_out", fn);
    if (!aligned(param_out, 2)) return fail(ZERO_ERR_ALIGN, "%s: param_out not 2-byte aligned", fn);
    for (int k = 0; k < world; ++k) {
        if (!grad_bufs[k]) return fail(ZERO_ERR_ARG, "%s: grad_bufs[%d] is NULL", fn, k);
        if (!aligned(grad_bufs[k], 2)) return fail(ZERO_ERR_ALIGN, "%s: grad_bufs[%d] not 2-byte aligned", fn, k);
    }
    // outputs: each output either is its own input (in place) or overlaps
    // nothing else; outputs never overlap each other or a gradient buffer
    const int64_t fb = count * 4, pb = count * 2, gb = padded_numel * 2;
    const void* outs[] = {master_out, m_out, v_out, param_out};
    const int64_t out_bytes[] = {fb, fb, fb, pb};
    for (int i = 0; i < 4; ++i) {
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(outs[i], out_bytes[i], outs[j], out_bytes[j]))
                return fail(ZERO_ERR_ARG, "%s: output arrays overlap", fn);
        for (int j = 0; j < 3; ++j)
            if (!(i == j && outs[i] == f_in[j]) && overlaps(outs[i], out_bytes[i], f_in[j], fb))
                return fail(ZERO_ERR_ARG, "%s: an output overlaps an input it does not replace", fn);
        for (int k = 0; k < world; ++k)
            if (overlaps(outs[i], out_bytes[i], grad_bufs[k], gb))
                return fail(ZERO_ERR_ARG, "%s: an output overlaps grad_bufs[%d]", fn, k);
    }

    StepParams prm{};
    prm.world = world;
    for (int k = 0; k < world; ++k) prm.grads[k] = static_cast<const uint16_t*>(grad_bufs[k]) + begin;
    prm.count = count;
    prm.master_in = master_in;
    prm.m_in = m_in;
    prm.v_in = v_in;
    prm.master_out = master_out;
    prm.m_out = m_out;
    prm.v_out = v_out;
    prm.param_out = param_out;
    prm.overflow = overflow_flag;
    prm.sqnorm = grad_sqnorm;
    if (grad_sqnorm) {
        prm.ticket = static_cast<unsigned int*>(workspace);
        prm.partials = reinterpret_cast<double*>(static_cast<char*>(workspace) + kWsPartialsOffset);
    }
    const double divisor = hp->grad_divisor > 0.0f ? static_cast<double>(hp->grad_divisor) : static_cast<double>(world);
    prm.c = adam_consts(hp, static_cast<float>(1.0 / (divisor * static_cast<double>(loss_scale))));
    prm.gate = nullptr;
    prm.clip_sqnorm = nullptr;
    prm.max_norm = 0.0;

    const int64_t h = common_phase(prm);
    if (h < 0 || h >= count) {
        prm.head = count;
        prm.nvec = 0;
    } else {
        prm.head = h;
        prm.nvec = (count - h) / kVec;
    }
    prm.tile = 0;
    prm.kind = kKindRegister;
    // 32-byte state stores need the fp32 outputs 32-byte aligned where the
    // vector region starts
    prm.st32 = 0;
    if (prm.nvec > 0) {
        bool al = true;
        for (const float* a : {master_out, m_out, v_out})
            al = al && ((reinterpret_cast<uintptr_t>(a) + 4 * static_cast<uintptr_t>(h)) % 32) == 0;
        prm.st32 = al ? 1 : 0;
    }

    // Kernel choice (measured on B200 against a measured copy rate of
    // 6.43 TB/s, L2 cold, each call alone, each kernel forced in turn):
    //  - arrays whose 16-byte phases never coincide, or N > kPipeMaxWorld: the
    //    register kernel (its scalar path when unaligned; at N = 64 it runs at
    //    the copy rate);
    //  - 3 <= N <= kRegMaxWorldLarge with at least kPipeMinTilesPerSm tiles
    //    per SM: the register kernel (256M-1B elements, N = 3 / 4 / 5:
    //    1.01-1.02 / 1.03 / 1.02 against 1.00-1.01 for the oct kernel and
    //    0.96-1.02 for the pipeline; the cause was not isolated: the oct
    //    kernel with the register kernel's grid, store width, load form or
    //    load order measured the same);
    //  - N <= 16 streams otherwise: the oct kernel when the fp32 outputs are
    //    32-byte aligned at the vector region (its 32-byte stores: N = 1 / 2 at
    //    256M and 1B elements 1.00-1.02 against 0.98-0.99 for the quad kernel
    //    and 0.96-0.99 for the register kernel), else the quad kernel; they
    //    take N <= 2 at every size, calls below kPipeMinTilesPerSm tiles per
    //    SM (no pipeline to fill and drain: 16M elements at N = 1..16,
    //    0.96-1.04 against 0.82-1.04) and gradients in another GPU's memory;
    //  - otherwise, with every gradient buffer in this GPU's memory, the
    //    pipeline kernel (its bulk copies never read another GPU's memory;
    //    N = 8 / 16 at 256M-1B: 1.04-1.08 / 1.09-1.10 against 1.03-1.04 /
    //    1.08 for the oct kernel);
    //  - 17 <= N <= 20 calls below the pipeline threshold: the pipeline kernel
    //    when the gradients are local and every SM gets two tiles, else the
    //    register kernel.
    // zero_test_force_step_kernel overrides the choice where the forced
    // kernel can run the call.
    int64_t blocks = 0;
    int sms = 0;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DeviceInfo* d = nullptr;
        if (int rc = device_info(&d)) return rc;
        sms = d->sms;
    }
    const int force = step_kernel_override();
    const int tile = h >= 0 ? pipe_tile(world) : 0;
    const int64_t ntiles = tile > 0 ? (count - h) / tile : 0;
    int kind = kKindRegister;
    if (h >= 0 && world <= kPipeMaxWorld) {
        const bool quad_ok = world <= kQuadMaxWorld;
        const bool big = ntiles >= kPipeMinTilesPerSm * static_cast<int64_t>(sms);
        const int stream_kind = prm.st32 ? kKindOct : kKindQuad;
        if (big && world >= 3 && world <= kRegMaxWorldLarge) {
            kind = kKindRegister;
        } else if (quad_ok && (world <= 2 || !big)) {
            kind = stream_kind;
        } else if (all_local_device_memory(grad_bufs, world)) {   // queried only where it decides
            if (big || ntiles >= 2 * static_cast<int64_t>(sms)) kind = kKindPipe;
        } else if (quad_ok) {
            kind = stream_kind;
        }
    }
    if (force == kKindRegister) kind = kKindRegister;
    if (force == kKindQuad && h >= 0 && world <= kQuadMaxWorld) kind = kKindQuad;
    if (force == kKindPipe && tile > 0 && ntiles >= 1 && all_local_device_memory(grad_bufs, world)) kind = kKindPipe;
    if (force == kKindOct && h >= 0 && world <= kQuadMaxWorld && prm.st32) kind = kKindOct;
    if (kind == kKindOct) {
        prm.kind = kKindOct;
        int nt = 0, bps = 0;
        (void)pick_oct_kernel(grad_dtype, param_dtype, world, &nt, &bps);
        blocks = (prm.nvec + nt - 1) / nt;
        int64_t cap = static_cast<int64_t>(sms) * bps;
        if (cap > kMaxBlocks) cap = kMaxBlocks;   // one norm partial per block in the workspace
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
    } else if (kind == kKindPipe) {
        if (int rc = pipe_setup(grad_dtype, param_dtype, &sms)) return rc;
        prm.tile = tile;
        prm.nvec = ntiles * tile / kVec;
        prm.kind = kKindPipe;
        blocks = sms;
    } else if (kind == kKindQuad) {
        prm.kind = kKindQuad;
        int nt = 0, u = 0;
        (void)pick_quad_kernel(grad_dtype, param_dtype, world, &nt, &u);
        const int64_t per_block = static_cast<int64_t>(nt) * u;
        const int64_t work = prm.nvec > 0 ? 2 * prm.nvec : count;
        blocks = (work + per_block - 1) / per_block;
        int64_t cap = static_cast<int64_t>(sms) * kQuadBlocksPerSm;
        if (cap > kMaxBlocks) cap = kMaxBlocks;   // one norm partial per block in the workspace
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
    } else {
        int limit = 0;
        if (int rc = grid_limit(grad_dtype, param_dtype, &limit)) return rc;
        if (h < 0 || h >= count) {
            prm.head = count;
            prm.nvec = 0;
        }
        const int64_t work = prm.nvec > 0 ? prm.nvec : count;
        blocks = (work + kThreads - 1) / kThreads;
        if (blocks > limit) blocks = limit;
        if (blocks < 1) blocks = 1;
    }
    *prm_out = prm;
    *blocks_out = blocks;
    return ZERO_OK;
}

// SM count, and the statistics pipeline kernel's shared-memory limit.
inline int stats_pipe_setup(zero_dtype_t g, bool write, int* sms) {
    const int which = static_cast<int>(g) * 2 + (write ? 1 : 0);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo* d = nullptr;
    if (int rc = device_info(&d)) return rc;
    if (!d->stats_pipe_ready[which]) {
        cudaError_t e = cudaFuncSetAttribute(pick_stats_pipe_kernel(g, write), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kPipeSmemMax));
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "cannot raise the shared-memory limit: %s", cudaGetErrorString(e));
        d->stats_pipe_ready[which] = true;
    }
    *sms = d->sms;
    return ZERO_OK;
}

// Validate a statistics call and build its kernel parameters (the state
// pointers stay NULL: the statistics kernel reads gradients only).
inline int prepare_stats(const char* fn, const void* const* grad_bufs, int32_t world, int64_t padded_numel,
                         int32_t partition, zero_dtype_t grad_dtype, float loss_scale, float grad_divisor,
                         const float* reduced, int32_t* overflow_flag, double* grad_sqnorm, void* workspace,
                         StepParams* prm_out, int64_t* blocks_out) {
    if (!grad_bufs || !overflow_flag) return fail(ZERO_ERR_ARG, "%s: NULL grad_bufs or overflow_flag", fn);
    if (world < 1 || world > ZERO_MAX_WORLD)
        return fail(ZERO_ERR_ARG, "%s: world %d outside 1..%d", fn, world, ZERO_MAX_WORLD);
    if (padded_numel < 0 || padded_numel % world != 0)
        return fail(ZERO_ERR_ARG, "%s: padded_numel %lld is not a non-negative multiple of world %d", fn,
                    (long long)padded_numel, world);
    if (partition != ZERO_ALL_PARTITIONS && (partition < 0 || partition >= world))
        return fail(ZERO_ERR_RANGE, "%s: partition %d outside 0..%d", fn, partition, world - 1);
    if (grad_dtype != ZERO_F16 && grad_dtype != ZERO_BF16)
        return fail(ZERO_ERR_DTYPE, "%s: gradients must be ZERO_F16 or ZERO_BF16", fn);
    if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale))
        return fail(ZERO_ERR_ARG, "%s: loss_scale must be positive and finite", fn);
    if (!(grad_divisor >= 0.0f) || !std::isfinite(grad_divisor))
        return fail(ZERO_ERR_ARG, "%s: grad_divisor must be >= 0 and finite", fn);
    if (grad_sqnorm && !workspace) return fail(ZERO_ERR_ARG, "%s: grad_sqnorm needs a workspace", fn);
    if (!aligned(overflow_flag, 4) || (grad_sqnorm && !aligned(grad_sqnorm, 8)) ||
        (workspace && !aligned(workspace, 16)))
        return fail(ZERO_ERR_ALIGN, "%s: flag, norm or workspace misaligned", fn);
    for (int k = 0; k < world; ++k) {
        if (!grad_bufs[k]) return fail(ZERO_ERR_ARG, "%s: grad_bufs[%d] is NULL", fn, k);
        if (!aligned(grad_bufs[k], 2)) return fail(ZERO_ERR_ALIGN, "%s: grad_bufs[%d] not 2-byte aligned", fn, k);
    }
    const int64_t P = padded_numel / world;
    const int64_t begin = partition == ZERO_ALL_PARTITIONS ? 0 : static_cast<int64_t>(partition) * P;
    const int64_t count = partition == ZERO_ALL_PARTITIONS ? padded_numel : P;
    if (reduced) {
        if (!aligned(reduced, 4)) return fail(ZERO_ERR_ALIGN, "%s: reduced_out not 4-byte aligned", fn);
        for (int k = 0; k < world; ++k)
            if (overlaps(reduced, count * 4, grad_bufs[k], padded_numel * 2))
                return fail(ZERO_ERR_ARG, "%s: reduced_out overlaps grad_bufs[%d]", fn, k);
    }
    if (count == 0) {
        *blocks_out = 0;
        return ZERO_OK;
    }
    StepParams prm{};
    prm.world = world;
    for (int k = 0; k < world; ++k) prm.grads[k] = static_cast<const uint16_t*>(grad_bufs[k]) + begin;
    prm.count = count;
    prm.overflow = overflow_flag;
    prm.sqnorm = grad_sqnorm;
    if (grad_sqnorm) {
        prm.ticket = static_cast<unsigned int*>(workspace);
        prm.partials = reinterpret_cast<double*>(static_cast<char*>(workspace) + kWsPartialsOffset);
    }
    const double divisor = grad_divisor > 0.0f ? static_cast<double>(grad_divisor) : static_cast<double>(world);
    prm.c.inv = static_cast<float>(1.0 / (divisor * static_cast<double>(loss_scale)));
    prm.c.clip = 1.0f;
    // the first element at which every replica (and the reduced output) is
    // 16-byte aligned
    int64_t h = -1;
    for (int64_t c = 0; c < kVec && h < 0; ++c) {
        bool good = !reduced || ((reinterpret_cast<uintptr_t>(reduced) + 4 * c) % 16) == 0;
        for (int k = 0; k < world && good; ++k)
            good = ((reinterpret_cast<uintptr_t>(prm.grads[k]) + 2 * c) % 16) == 0;
        if (good) h = c;
    }
    if (h < 0 || h >= count) {
        prm.head = count;
        prm.nvec = 0;
    } else {
        prm.head = h;
        prm.nvec = (count - h) / kVec;
    }
    prm.tile = 0;
    prm.kind = kKindRegister;
    // Kernel choice (measured on B200 against a measured copy rate of
    // 6.43 TB/s, inputs larger than 4x L2):
    //  - statistics only (2N bytes per element, all reads): the quad kernel
    //    for N <= 16 (256M elements, N = 2..16: 0.90-1.14 against 0.64-1.10
    //    for the pipeline kernel);
    //  - with the fp32 store of the staged reduce-scatter: the pipeline
    //    kernel for 3 <= N <= 8 from kStatsPipeMinTilesPerSm tiles per SM when
    //    every gradient buffer is this GPU's memory (256M, N = 4 / 8: 1.04 /
    //    1.09 against 1.02 / 1.06), the quad kernel for the rest of N <= 16
    //    (256M, N = 16: 1.06 against 1.02; 64M, N = 2: 0.93 against 0.85);
    //  - 17 <= N <= 20: the pipeline kernel from two tiles per SM when the
    //    gradients are local, else the register kernel; unaligned calls and
    //    N > 20: the register kernel.
    // zero_test_force_step_kernel overrides the choice where the forced
    // kernel can run the call.
    int sms = 0;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DeviceInfo* d = nullptr;
        if (int rc = device_info(&d)) return rc;
        sms = d->sms;
    }
    const int force = step_kernel_override();
    const int tile = h >= 0 ? stats_pipe_tile(world) : 0;
    const int64_t ntiles = tile > 0 ? (count - h) / tile : 0;
    const bool vec = prm.nvec > 0;
    const bool quad_ok = vec && world <= kQuadMaxWorld;
    const bool pipe_big = reduced != nullptr && world >= 3 && world <= kStatsPipeMaxWorldWrite &&
                          ntiles >= kStatsPipeMinTilesPerSm * static_cast<int64_t>(sms);
    int kind = kKindRegister;
    if (quad_ok && !pipe_big) {
        kind = kKindQuad;
    } else if (tile > 0 && ntiles >= 2 * static_cast<int64_t>(sms) && all_local_device_memory(grad_bufs, world)) {
        kind = kKindPipe;
    } else if (quad_ok) {
        kind = kKindQuad;
    }
    // the write-heavy reduce-scatter at N <= 2: 32-byte stores of the reduced
    // gradients (the oct version) where `reduced` is 32-byte aligned at h
    const bool rs_oct_ok = quad_ok && reduced != nullptr && world <= 2 &&
                           ((reinterpret_cast<uintptr_t>(reduced) + 4 * static_cast<uintptr_t>(h)) % 32) == 0;
    if (kind == kKindQuad && rs_oct_ok) kind = kKindOct;
    if (force == kKindRegister) kind = kKindRegister;
    if (force == kKindQuad && quad_ok) kind = kKindQuad;
    if (force == kKindOct && rs_oct_ok) kind = kKindOct;
    if (force == kKindPipe && tile > 0 && ntiles >= 1 && all_local_device_memory(grad_bufs, world)) kind = kKindPipe;
    int64_t blocks = 0;
    if (kind == kKindOct) {
        prm.kind = kKindOct;
        int nt = 0, u = 0;
        (void)pick_rs_oct_kernel(grad_dtype, world, &nt, &u);
        const int64_t per_block = static_cast<int64_t>(nt) * u;
        blocks = (prm.nvec + per_block - 1) / per_block;
        int64_t cap = static_cast<int64_t>(sms) * kQuadBlocksPerSm;
        if (cap > kMaxBlocks) cap = kMaxBlocks;   // one norm partial per block in the workspace
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
    } else if (kind == kKindPipe) {
        if (int rc = stats_pipe_setup(grad_dtype, reduced != nullptr, &sms)) return rc;
        prm.tile = tile;
        prm.nvec = ntiles * tile / kVec;
        prm.kind = kKindPipe;
        blocks = sms;
    } else if (kind == kKindQuad) {
        prm.kind = kKindQuad;
        int nt = 0, u = 0;
        (void)pick_stats_quad_kernel(grad_dtype, reduced != nullptr, world, &nt, &u);
        const int64_t per_block = static_cast<int64_t>(nt) * u;
        blocks = (2 * prm.nvec + per_block - 1) / per_block;
        int64_t cap = static_cast<int64_t>(sms) * kQuadBlocksPerSm;
        if (cap > kMaxBlocks) cap = kMaxBlocks;   // one norm partial per block in the workspace
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
    } else {
        int limit = 0;
        if (int rc = stats_grid_limit(grad_dtype, reduced != nullptr, &limit)) return rc;
        const int64_t work = prm.nvec > 0 ? prm.nvec : count;
        blocks = (work + kThreads - 1) / kThreads;
        if (blocks > limit) blocks = limit;
        if (blocks < 1) blocks = 1;
    }
    *prm_out = prm;
    *blocks_out = blocks;
    return ZERO_OK;
}

// Enqueue the statistics kernel prepared by prepare_stats; `reduced` is the
// same pointer prepare_stats saw (NULL: statistics only).
inline int launch_stats(const char* fn, const StepParams& prm, int64_t blocks, zero_dtype_t grad_dtype,
                        float* reduced, zero_stream_t stream) {
    if (blocks == 0) return ok();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool write = reduced != nullptr;
    if (prm.kind == kKindPipe) {
        pick_stats_pipe_kernel(grad_dtype, write)<<<static_cast<unsigned int>(blocks), kPipeThreads,
                                                    stats_pipe_smem_bytes(prm.world, prm.tile), s>>>(prm, reduced);
    } else if (prm.kind == kKindQuad) {
        int nt = 0, u = 0;
        StatsKernelFn k = pick_stats_quad_kernel(grad_dtype, write, prm.world, &nt, &u);
        k<<<static_cast<unsigned int>(blocks), nt, 0, s>>>(prm, reduced);
    } else if (prm.kind == kKindOct) {
        int nt = 0, u = 0;
        StatsKernelFn k = pick_rs_oct_kernel(grad_dtype, prm.world, &nt, &u);
        k<<<static_cast<unsigned int>(blocks), nt, 0, s>>>(prm, reduced);
    } else {
        pick_stats_kernel(grad_dtype, write)<<<static_cast<unsigned int>(blocks), kThreads, 0, s>>>(prm, reduced);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    return ok();
}

// Add the gate and the clipping inputs to prepared step parameters.
inline int add_gate_and_clip(const char* fn, StepParams* prm, const int32_t* gate, const double* clip_sqnorm,
                             float max_norm) {
    if (gate && !aligned(gate, 4)) return fail(ZERO_ERR_ALIGN, "%s: gate misaligned", fn);
    if (gate && gate == prm->overflow)
        return fail(ZERO_ERR_ARG, "%s: gate must not be the call's own overflow_flag", fn);
    if (clip_sqnorm) {
        if (!aligned(clip_sqnorm, 8)) return fail(ZERO_ERR_ALIGN, "%s: clip_sqnorm misaligned", fn);
        if (!(max_norm > 0.0f) || !std::isfinite(max_norm))
            return fail(ZERO_ERR_ARG, "%s: max_norm must be positive and finite", fn);
    }
    prm->gate = gate;
    prm->clip_sqnorm = clip_sqnorm;
    prm->max_norm = static_cast<double>(max_norm);
    return ZERO_OK;
}

// Enqueue the fused kernel prepared by prepare_step.
inline int launch_step(const char* fn, const StepParams& prm, int64_t blocks, zero_dtype_t grad_dtype,
                       zero_dtype_t param_dtype, zero_stream_t stream) {
    if (blocks == 0) return ok();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (prm.kind == kKindPipe) {
        pick_pipe_kernel(grad_dtype, param_dtype)<<<static_cast<unsigned int>(blocks), kPipeThreads,
                                                     pipe_smem_bytes(prm.world, prm.tile), s>>>(prm);
    } else if (prm.kind == kKindQuad) {
        int nt = 0, u = 0;
        KernelFn k = pick_quad_kernel(grad_dtype, param_dtype, prm.world, &nt, &u);
        k<<<static_cast<unsigned int>(blocks), nt, 0, s>>>(prm);
    } else if (prm.kind == kKindOct) {
        int nt = 0, bps = 0;
        KernelFn k = pick_oct_kernel(grad_dtype, param_dtype, prm.world, &nt, &bps);
        k<<<static_cast<unsigned int>(blocks), nt, 0, s>>>(prm);
    } else {
        pick_kernel(grad_dtype, param_dtype)<<<static_cast<unsigned int>(blocks), kThreads, 0, s>>>(prm);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    return ok();
}

}  // namespace
}  // namespace fused
}  // namespace zero
