// Kernels of the statistics pass: the rank-order fp32 sums of the N
// replicas, the overflow OR and (optionally) the squared norm of the
// unscaled gradient, with no optimizer state read or written.  2N bytes per
// element.  Used before an in-place update (exact skip with one bank of
// states) and for global-norm clipping.  With kWrite they are also the
// staged reduce-scatter: each element's unscaled gradient g = s * inv is
// stored to `reduced` as fp32 (2N + 4 bytes per element).  Device helpers
// come from fused_step.cuh.
#pragma once

#include "fused_step.cuh"

namespace zero {
namespace fused {
namespace {

// Rank-order sum of element e over the N replicas (scalar path).
template <typename GT>
__device__ __forceinline__ float replica_sum(const StepParams& p, int64_t e) {
    float s = Fmt<GT>::one(static_cast<const uint16_t*>(p.grads[0])[e]);
    for (int k = 1; k < p.world; ++k) s = __fadd_rn(s, Fmt<GT>::one(static_cast<const uint16_t*>(p.grads[k])[e]));
    return s;
}

// Elements outside the vector (or tile) region.
template <typename GT, bool kWrite>
__device__ __forceinline__ void stats_scalar_elements(const StepParams& p, float* reduced, int64_t tid,
                                                      int64_t nthreads, bool& bad, double& sq) {
    const float inv = p.c.inv;
    const int64_t vec_end = p.head + p.nvec * kVec;
    const int64_t nscalar = p.head + (p.count - vec_end);
    for (int64_t q = tid; q < nscalar; q += nthreads) {
        const int64_t e = q < p.head ? q : vec_end + (q - p.head);
        if (out_of_bounds(e >= 0 && e < p.count, p.overflow)) continue;
        const float s = replica_sum<GT>(p, e);
        bad |= !isfinite(s);
        const float g = __fmul_rn(s, inv);
        if constexpr (kWrite) reduced[e] = g;
        if (p.sqnorm) sq = fma(static_cast<double>(g), static_cast<double>(g), sq);
    }
}

// Statistics pre-pass: the rank-order fp32 sum of the N replicas, the
// overflow test and, when p.sqnorm is set, the squared norm of the unscaled
// gradient g = s * inv, without reading or writing any optimizer state.
// 2N bytes per element.  Lets a caller decide skip and clipping for a whole
// step before any state is written (in-place update with an exact skip).
// kWrite: also store g to reduced[e] (16-byte stores).
template <typename GT, bool kWrite>
__global__ void __launch_bounds__(kThreads) grad_stats_kernel(const __grid_constant__ StepParams p,
                                                              float* __restrict__ reduced) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    const int world = p.world;
    const float inv = p.c.inv;
    const bool want_sq = p.sqnorm != nullptr;
    bool bad = false;
    double sq = 0.0;
    for (int64_t vi = tid; vi < p.nvec; vi += nthreads) {
        const int64_t e0 = p.head + vi * kVec;
        if (out_of_bounds(e0 + kVec <= p.count, p.overflow)) continue;
        float s[kVec];
        {
            uint4 r[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
                if (b < world) r[b] = ld_grad16(static_cast<const uint16_t*>(p.grads[b]) + e0);
            cvt8<GT>(r[0], s);
#pragma unroll
            for (int b = 1; b < kBatch; ++b)
                if (b < world) add8<GT>(r[b], s);
        }
        for (int k0 = kBatch; k0 < world; k0 += kBatch) {
            uint4 r[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
                if (k0 + b < world) r[b] = ld_grad16(static_cast<const uint16_t*>(p.grads[k0 + b]) + e0);
#pragma unroll
            for (int b = 0; b < kBatch; ++b)
                if (k0 + b < world) add8<GT>(r[b], s);
        }
        float g[kVec];
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            bad |= !isfinite(s[e]);
            g[e] = __fmul_rn(s[e], inv);
            if (want_sq) sq = fma(static_cast<double>(g[e]), static_cast<double>(g[e]), sq);
        }
        if constexpr (kWrite) {
            st_state16(reduced + e0, g[0], g[1], g[2], g[3]);
            st_state16(reduced + e0 + 4, g[4], g[5], g[6], g[7]);
        }
    }
    stats_scalar_elements<GT, kWrite>(p, reduced, tid, nthreads, bad, sq);
    finish_block<kThreads>(p, bad, sq);
}

// Quad-streaming statistics kernel for N <= B replicas: thread t sums quads
// (4 consecutive elements) t, t + T, ..., U of them per iteration, issuing
// every replica's 8-byte load of those U quads before the first add (plain
// loads, a grid of several waves), as the quad step kernel does for the
// fused step.  For calls too short for the pipeline kernel to fill and
// drain its stages.  kWrite: also store g = s * inv with one 16-byte store
// per quad.
template <typename GT, bool kWrite, int B, int U, int NT>
__global__ void __launch_bounds__(NT, 2) grad_stats_quad_kernel(const __grid_constant__ StepParams p,
                                                                  float* __restrict__ reduced) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * NT + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * NT;
    const int world = p.world;
    const float inv = p.c.inv;
    const bool want_sq = p.sqnorm != nullptr;
    bool bad = false;
    double sq = 0.0;
    const int64_t nq = 2 * p.nvec;
    for (int64_t q0 = tid; q0 < nq; q0 += U * nthreads) {
        uint2 r[U][B];
        bool live[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t e0 = p.head + 4 * (q0 + u * nthreads);
            live[u] = q0 + u * nthreads < nq && !out_of_bounds(e0 + 4 <= p.count, p.overflow);
            if (!live[u]) continue;
#pragma unroll
            for (int k = 0; k < B; ++k)
                if (k < world) r[u][k] = ld_u2(static_cast<const uint16_t*>(p.grads[k]) + e0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (!live[u]) continue;
            const int64_t e0 = p.head + 4 * (q0 + u * nthreads);
            // rank-order fp32 sum
            float s0 = Fmt<GT>::lo(r[u][0].x), s1 = Fmt<GT>::hi(r[u][0].x);
            float s2 = Fmt<GT>::lo(r[u][0].y), s3 = Fmt<GT>::hi(r[u][0].y);
#pragma unroll
            for (int k = 1; k < B; ++k) {
                if (k >= world) break;
                s0 = __fadd_rn(s0, Fmt<GT>::lo(r[u][k].x));
                s1 = __fadd_rn(s1, Fmt<GT>::hi(r[u][k].x));
                s2 = __fadd_rn(s2, Fmt<GT>::lo(r[u][k].y));
                s3 = __fadd_rn(s3, Fmt<GT>::hi(r[u][k].y));
            }
            bad |= !isfinite(s0) | !isfinite(s1) | !isfinite(s2) | !isfinite(s3);
            const float g0 = __fmul_rn(s0, inv), g1 = __fmul_rn(s1, inv);
            const float g2 = __fmul_rn(s2, inv), g3 = __fmul_rn(s3, inv);
            if (want_sq) {
                sq = fma(static_cast<double>(g0), static_cast<double>(g0), sq);
                sq = fma(static_cast<double>(g1), static_cast<double>(g1), sq);
                sq = fma(static_cast<double>(g2), static_cast<double>(g2), sq);
                sq = fma(static_cast<double>(g3), static_cast<double>(g3), sq);
            }
            if constexpr (kWrite) st_state16(reduced + e0, g0, g1, g2, g3);
        }
    }
    stats_scalar_elements<GT, kWrite>(p, reduced, tid, nthreads, bad, sq);
    finish_block<NT>(p, bad, sq);
}

// Shapes of the quad statistics kernel by replica count: U quads per thread
// per iteration (B x U 8-byte loads: 128 bytes in flight per thread at
// N = B >= 2, 64 at N = 1, where U = 16 would spill), NT threads per block.
template <int B> struct StatsQuadShape;
template <> struct StatsQuadShape<1> { static constexpr int U = 8, NT = 512; };
template <> struct StatsQuadShape<2> { static constexpr int U = 8, NT = 512; };
template <> struct StatsQuadShape<4> { static constexpr int U = 4, NT = 512; };
template <> struct StatsQuadShape<8> { static constexpr int U = 2, NT = 512; };
template <> struct StatsQuadShape<16> { static constexpr int U = 1, NT = 512; };

// Oct-streaming staged reduce-scatter for N <= B replicas (B = 1, 2: the
// write-heavy cases, 4 bytes written per 2N read): thread t reduces octs (8
// consecutive elements) t, t + T, ..., U of them per iteration, every
// replica's 16-byte load of those U octs issued before the first add, then
// one 32-byte store of the 8 unscaled gradients per oct.  Needs `reduced`
// 32-byte aligned at the vector region's start (the host checks).
template <typename GT, int B, int U, int NT>
__global__ void __launch_bounds__(NT, 2) grad_rs_oct_kernel(const __grid_constant__ StepParams p,
                                                           float* __restrict__ reduced) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * NT + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * NT;
    const int world = p.world;
    const float inv = p.c.inv;
    const bool want_sq = p.sqnorm != nullptr;
    bool bad = false;
    double sq = 0.0;
    for (int64_t v0 = tid; v0 < p.nvec; v0 += U * nthreads) {
        uint4 r[U][B];
        bool live[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t e0 = p.head + kVec * (v0 + u * nthreads);
            live[u] = v0 + u * nthreads < p.nvec && !out_of_bounds(e0 + kVec <= p.count, p.overflow);
            if (!live[u]) continue;
#pragma unroll
            for (int k = 0; k < B; ++k)
                if (k < world) r[u][k] = ld_grad16(static_cast<const uint16_t*>(p.grads[k]) + e0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (!live[u]) continue;
            const int64_t e0 = p.head + kVec * (v0 + u * nthreads);
            float g[kVec];
            cvt8<GT>(r[u][0], g);   // rank-order fp32 sum
#pragma unroll
            for (int k = 1; k < B; ++k)
                if (k < world) add8<GT>(r[u][k], g);
#pragma unroll
            for (int e = 0; e < kVec; ++e) {
                bad |= !isfinite(g[e]);
                g[e] = __fmul_rn(g[e], inv);
                if (want_sq) sq = fma(static_cast<double>(g[e]), static_cast<double>(g[e]), sq);
            }
            st_state32(reduced + e0, g);
        }
    }
    stats_scalar_elements<GT, true>(p, reduced, tid, nthreads, bad, sq);
    finish_block<NT>(p, bad, sq);
}

template <int B> struct RsOctShape;
template <> struct RsOctShape<1> { static constexpr int U = 4, NT = 512; };
template <> struct RsOctShape<2> { static constexpr int U = 4, NT = 512; };

// Pipeline statistics kernel: the producer warp streams tiles of the N
// gradient slices into two shared-memory stages with 1-D bulk copies (no
// multicast, this CTA's own shared memory); 16 consumer warps sum each
// 4-element chunk in rank order (kWrite: and store its 4 unscaled gradients
// with one 16-byte store).  Waits bounded as in the step's pipeline.
template <typename GT, bool kWrite>
__global__ void __launch_bounds__(kPipeThreads, 1) grad_stats_pipe_kernel(const __grid_constant__ StepParams p,
                                                                          float* __restrict__ reduced) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kPipeStages];
    __shared__ __align__(8) uint64_t empty[kPipeStages];
    __shared__ int abort_flag;
    const int world = p.world;
    const int T = p.tile;
    const uint32_t gbytes = 2u * static_cast<uint32_t>(T);
    const uint32_t stage = static_cast<uint32_t>(world) * gbytes;
    const int64_t ntiles = p.nvec * kVec / T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float inv = p.c.inv;
    const bool want_sq = p.sqnorm != nullptr;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPipeStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kPipeConsumerWarps);
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    bool bad = false;
    double sq = 0.0;
    if (warp == kPipeConsumerWarps) {
        int64_t i = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
            const int s = static_cast<int>(i % kPipeStages);
            const uint32_t ph = static_cast<uint32_t>((i / kPipeStages) & 1);
            bool ok = true;
            if (i >= kPipeStages && lane == 0) ok = mbar_wait_bounded(&empty[s], ph ^ 1u);
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
            for (int k = lane; k < world; k += 32)
                bulk_load(st + static_cast<size_t>(k) * gbytes, static_cast<const uint16_t*>(p.grads[k]) + e0, gbytes,
                          &full[s]);
        }
        if (lane == 0) {
            const int64_t issued = i;
            for (int64_t j = issued > kPipeStages ? issued - kPipeStages : 0; j < issued; ++j)
                if (!mbar_wait_bounded(&full[j % kPipeStages], static_cast<uint32_t>((j / kPipeStages) & 1)))
                    atomicOr(p.overflow, kFlagDeviceTimeout);
        }
        __syncwarp();
    } else {
        constexpr int C = kPipeConsumerWarps * 32;
        const int t = threadIdx.x;
        int64_t i = 0;
        for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
            const int s = static_cast<int>(i % kPipeStages);
            const uint32_t ph = static_cast<uint32_t>((i / kPipeStages) & 1);
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
            const unsigned char* st = smem + static_cast<size_t>(s) * stage;
            const int64_t base = p.head + tile * T;
            for (int ch = t; ch < T / 4; ch += C) {
                const int j = 4 * ch;
                if (out_of_bounds(j + 4 <= T && base + j + 4 <= p.count, p.overflow)) continue;
                const uint2 r0 = *reinterpret_cast<const uint2*>(st + 2 * j);
                float a0 = Fmt<GT>::lo(r0.x), a1 = Fmt<GT>::hi(r0.x), a2 = Fmt<GT>::lo(r0.y), a3 = Fmt<GT>::hi(r0.y);
#pragma unroll 4
                for (int k = 1; k < world; ++k) {
                    const uint2 r = *reinterpret_cast<const uint2*>(st + static_cast<size_t>(k) * gbytes + 2 * j);
                    a0 = __fadd_rn(a0, Fmt<GT>::lo(r.x));
                    a1 = __fadd_rn(a1, Fmt<GT>::hi(r.x));
                    a2 = __fadd_rn(a2, Fmt<GT>::lo(r.y));
                    a3 = __fadd_rn(a3, Fmt<GT>::hi(r.y));
                }
                bad |= !isfinite(a0) | !isfinite(a1) | !isfinite(a2) | !isfinite(a3);
                const float g0 = __fmul_rn(a0, inv), g1 = __fmul_rn(a1, inv);
                const float g2 = __fmul_rn(a2, inv), g3 = __fmul_rn(a3, inv);
                if constexpr (kWrite) st_state16(reduced + base + j, g0, g1, g2, g3);
                if (want_sq) {
                    sq = fma(static_cast<double>(g0), static_cast<double>(g0), sq);
                    sq = fma(static_cast<double>(g1), static_cast<double>(g1), sq);
                    sq = fma(static_cast<double>(g2), static_cast<double>(g2), sq);
                    sq = fma(static_cast<double>(g3), static_cast<double>(g3), sq);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        stats_scalar_elements<GT, kWrite>(p, reduced, static_cast<int64_t>(blockIdx.x) * C + t,
                                          static_cast<int64_t>(gridDim.x) * C, bad, sq);
    }
    finish_block<kPipeThreads>(p, bad, sq);
}

}  // namespace
}  // namespace fused
}  // namespace zero
