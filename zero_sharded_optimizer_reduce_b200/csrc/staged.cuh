// Device code of the staged ZeRO-2 step's second half: the Adam update of a
// partition from its reduced fp32 gradients (the output of the staged
// reduce-scatter, grad_stats.cuh with kWrite), as a register-streaming and a
// bulk-copy pipeline kernel.  Reads 16 bytes per element
// (gradient, master, m, v), writes 14 (master, m, v, parameter): 30 bytes,
// against the fused step's 2N + 26 read in one pass.
#pragma once

#include "fused_step.cuh"

namespace zero {
namespace fused {
namespace {

// Destinations of the updated parameters when they are broadcast: this
// rank's slot in every rank's parameter buffer (peers' buffers mapped into
// this process), i.e. the all-gather done by the update's own stores.
struct ParamDsts {
    void* dst[ZERO_MAX_WORLD];  // each already offset to the call's first element
    int32_t n;
};

// Parameter stores of 8, 4 or 1 element(s) at element e: to p.param_out, or
// (kBcast) to every destination in d.
template <bool kBcast>
__device__ __forceinline__ void store_params8(const StepParams& p, const ParamDsts& d, int64_t e, uint4 q) {
    if constexpr (kBcast) {
        for (int k = 0; k < d.n; ++k) st_u16x8(static_cast<uint16_t*>(d.dst[k]) + e, q);
    } else {
        st_u16x8(static_cast<uint16_t*>(p.param_out) + e, q);
    }
}

template <bool kBcast>
__device__ __forceinline__ void store_params4(const StepParams& p, const ParamDsts& d, int64_t e, uint2 q) {
    if constexpr (kBcast) {
        for (int k = 0; k < d.n; ++k) st_u16x4(static_cast<uint16_t*>(d.dst[k]) + e, q);
    } else {
        st_u16x4(static_cast<uint16_t*>(p.param_out) + e, q);
    }
}

template <bool kBcast>
__device__ __forceinline__ void store_param1(const StepParams& p, const ParamDsts& d, int64_t e, uint16_t q) {
    if constexpr (kBcast) {
        for (int k = 0; k < d.n; ++k) static_cast<uint16_t*>(d.dst[k])[e] = q;
    } else {
        static_cast<uint16_t*>(p.param_out)[e] = q;
    }
}

__device__ __forceinline__ float4 ld_once16(const float* p) {
    const uint4 r = ld_grad16(p);
    return make_float4(__uint_as_float(r.x), __uint_as_float(r.y), __uint_as_float(r.z), __uint_as_float(r.w));
}

// p.grads[0] holds the reduced fp32 gradients g (already unscaled), indexed
// like the state arrays; p.c.inv is 1, so adam() forms g * clip exactly as
// the fused step forms (s * inv) * clip.  Gate and clip as in the fused
// step; no flag or norm (the reduce-scatter produced them).  kBcast: the
// parameters go to every destination of d instead of p.param_out.
template <typename PT, bool kBcast>
__global__ void __launch_bounds__(kThreads) adam_reduced_kernel(const __grid_constant__ StepParams p,
                                                                const __grid_constant__ ParamDsts d) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    Consts c = p.c;
    if (!step_prologue(p, c)) return;
    const float* gin = static_cast<const float*>(p.grads[0]);

    for (int64_t vi = tid; vi < p.nvec; vi += nthreads) {
        const int64_t e0 = p.head + vi * kVec;
        if (out_of_bounds(e0 + kVec <= p.count, p.overflow)) continue;
        const float4 ga = ld_once16(gin + e0), gb = ld_once16(gin + e0 + 4);
        const float4 pa = ld_state16(p.master_in + e0), pb = ld_state16(p.master_in + e0 + 4);
        const float4 ma = ld_state16(p.m_in + e0), mb = ld_state16(p.m_in + e0 + 4);
        const float4 va = ld_state16(p.v_in + e0), vb = ld_state16(p.v_in + e0 + 4);
        const float g[kVec] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
        float pw[kVec] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
        float mw[kVec] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
        float vw[kVec] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int e = 0; e < kVec; ++e) adam(g[e], pw[e], mw[e], vw[e], c);
        if (p.st32) {   // uniform over the grid
            st_state32(p.master_out + e0, pw);
            st_state32(p.m_out + e0, mw);
            st_state32(p.v_out + e0, vw);
        } else {
            st_state16(p.master_out + e0, pw[0], pw[1], pw[2], pw[3]);
            st_state16(p.master_out + e0 + 4, pw[4], pw[5], pw[6], pw[7]);
            st_state16(p.m_out + e0, mw[0], mw[1], mw[2], mw[3]);
            st_state16(p.m_out + e0 + 4, mw[4], mw[5], mw[6], mw[7]);
            st_state16(p.v_out + e0, vw[0], vw[1], vw[2], vw[3]);
            st_state16(p.v_out + e0 + 4, vw[4], vw[5], vw[6], vw[7]);
        }
        uint4 q;
        q.x = Fmt<PT>::pack(pw[0], pw[1]);
        q.y = Fmt<PT>::pack(pw[2], pw[3]);
        q.z = Fmt<PT>::pack(pw[4], pw[5]);
        q.w = Fmt<PT>::pack(pw[6], pw[7]);
        store_params8<kBcast>(p, d, e0, q);
    }

    // head and tail, one element per thread and iteration
    const int64_t vec_end = p.head + p.nvec * kVec;
    const int64_t nscalar = p.head + (p.count - vec_end);
    for (int64_t q = tid; q < nscalar; q += nthreads) {
        const int64_t e = q < p.head ? q : vec_end + (q - p.head);
        if (out_of_bounds(e >= 0 && e < p.count, p.overflow)) continue;
        float pw = p.master_in[e], mw = p.m_in[e], vw = p.v_in[e];
        adam(gin[e], pw, mw, vw, c);
        p.master_out[e] = pw;
        p.m_out[e] = mw;
        p.v_out[e] = vw;
        store_param1<kBcast>(p, d, e, Fmt<PT>::round1(pw));
    }
}

// Pipeline version (calls whose arrays share a 16-byte phase and give every
// SM at least two tiles): one CTA per SM; the producer warp streams tiles of
// p.tile elements of the four fp32 inputs (g, master, m, v) into
// kReducedStages shared-memory stages with 1-D bulk copies into this CTA's own
// shared memory (no multicast) completing on an mbarrier; 16 consumer warps
// update 4 consecutive elements per thread and store straight to global
// memory.  Every wait is bounded (kFlagDeviceTimeout into *p.overflow on
// expiry, then the CTA drains its own copies and returns).
// Stages of the pipeline kernel's ring.
constexpr int kReducedStages = 2;

template <typename PT, bool kBcast>
__global__ void __launch_bounds__(kPipeThreads, 1) adam_reduced_pipe_kernel(const __grid_constant__ StepParams p,
                                                                            const __grid_constant__ ParamDsts d) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kReducedStages];
    __shared__ __align__(8) uint64_t empty[kReducedStages];
    __shared__ int abort_flag;
    const int T = p.tile;
    const uint32_t abytes = 4u * static_cast<uint32_t>(T);
    const uint32_t stage = 4u * abytes;
    const int64_t ntiles = p.nvec * kVec / T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Consts c = p.c;
    if (!step_prologue(p, c)) return;   // uniform over the grid: before any barrier is set up
    if (threadIdx.x == 0) {
        for (int s = 0; s < kReducedStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kPipeConsumerWarps);
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kPipeConsumerWarps) {
        // ---- producer warp: lane 0 arms the stage, lanes 0..3 issue the copies
        int64_t i = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
            const int s = static_cast<int>(i % kReducedStages);
            const uint32_t ph = static_cast<uint32_t>((i / kReducedStages) & 1);
            bool ok = true;
            if (i >= kReducedStages && lane == 0) ok = mbar_wait_bounded(&empty[s], ph ^ 1u);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) {
                    atomicOr(p.overflow, kFlagDeviceTimeout);
                    abort_flag = 1;
                }
                break;
            }
            if (__shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&abort_flag), 0)) break;
            unsigned char* st = smem + static_cast<size_t>(s) * stage;
            const int64_t e0 = p.head + tile * T;
            if (out_of_bounds(e0 + T <= p.count, p.overflow)) {   // uniform over the warp
                if (lane == 0) abort_flag = 1;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[s], stage);
            __syncwarp();
            if (lane < 4) {
                const float* src = lane == 0 ? static_cast<const float*>(p.grads[0])
                                             : (lane == 1 ? p.master_in : (lane == 2 ? p.m_in : p.v_in));
                bulk_load(st + static_cast<size_t>(lane) * abytes, src + e0, abytes, &full[s]);
            }
        }
        if (lane == 0) {
            const int64_t issued = i;
            for (int64_t j = issued > kReducedStages ? issued - kReducedStages : 0; j < issued; ++j)
                if (!mbar_wait_bounded(&full[j % kReducedStages], static_cast<uint32_t>((j / kReducedStages) & 1)))
                    atomicOr(p.overflow, kFlagDeviceTimeout);
        }
        __syncwarp();
    } else {
        // ---- consumer warps: thread t takes 4 consecutive elements per chunk
        constexpr int C = kPipeConsumerWarps * 32;
        const int t = threadIdx.x;
        int64_t i = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
            const int s = static_cast<int>(i % kReducedStages);
            const uint32_t ph = static_cast<uint32_t>((i / kReducedStages) & 1);
            bool ok = true;
            if (lane == 0) ok = !*reinterpret_cast<volatile int*>(&abort_flag) && mbar_wait_bounded(&full[s], ph);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) {
                    atomicOr(p.overflow, kFlagDeviceTimeout);
                    abort_flag = 1;
                }
                break;
            }
            const float* sg = reinterpret_cast<const float*>(smem + static_cast<size_t>(s) * stage);
            const float* sp = sg + T;
            const float* sm = sp + T;
            const float* sv = sm + T;
            const int64_t base = p.head + tile * T;
            for (int ch = t; ch < T / 4; ch += C) {
                const int j = 4 * ch;
                if (out_of_bounds(j + 4 <= T && base + j + 4 <= p.count, p.overflow)) continue;
                const float4 g4 = *reinterpret_cast<const float4*>(sg + j);
                const float4 p4 = *reinterpret_cast<const float4*>(sp + j);
                const float4 m4 = *reinterpret_cast<const float4*>(sm + j);
                const float4 v4 = *reinterpret_cast<const float4*>(sv + j);
                float pw[4] = {p4.x, p4.y, p4.z, p4.w};
                float mw[4] = {m4.x, m4.y, m4.z, m4.w};
                float vw[4] = {v4.x, v4.y, v4.z, v4.w};
                const float g[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) adam(g[e], pw[e], mw[e], vw[e], c);
                st_state16(p.master_out + base + j, pw[0], pw[1], pw[2], pw[3]);
                st_state16(p.m_out + base + j, mw[0], mw[1], mw[2], mw[3]);
                st_state16(p.v_out + base + j, vw[0], vw[1], vw[2], vw[3]);
                uint2 pk;
                pk.x = Fmt<PT>::pack(pw[0], pw[1]);
                pk.y = Fmt<PT>::pack(pw[2], pw[3]);
                store_params4<kBcast>(p, d, base + j, pk);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        // head and tail, spread over every consumer thread of the grid
        const float* gin = static_cast<const float*>(p.grads[0]);
        const int64_t vec_end = p.head + p.nvec * kVec;
        const int64_t nscalar = p.head + (p.count - vec_end);
        for (int64_t q = static_cast<int64_t>(blockIdx.x) * C + t; q < nscalar;
             q += static_cast<int64_t>(gridDim.x) * C) {
            const int64_t e = q < p.head ? q : vec_end + (q - p.head);
            if (out_of_bounds(e >= 0 && e < p.count, p.overflow)) continue;
            float pw = p.master_in[e], mw = p.m_in[e], vw = p.v_in[e];
            adam(gin[e], pw, mw, vw, c);
            p.master_out[e] = pw;
            p.m_out[e] = mw;
            p.v_out[e] = vw;
            store_param1<kBcast>(p, d, e, Fmt<PT>::round1(pw));
        }
    }
}

}  // namespace
}  // namespace fused
}  // namespace zero
