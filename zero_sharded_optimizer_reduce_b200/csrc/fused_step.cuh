// Device code of the fused ZeRO-2 step: the register-streaming and the
// shared-memory pipeline kernels, the device helpers they share with the
// statistics kernels, and the bounded-wait self-test kernel.  Host-side
// validation, kernel choice and launch live in step_launch.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "bulk.cuh"
#include "common.h"

namespace zero {
namespace fused {
// Internal linkage: every translation unit that includes this header gets
// its own instance of the kernel, registered with its own module.
namespace {

constexpr int kThreads = 256;
constexpr int kVec = 8;          // elements per vector
constexpr int kBatch = 8;        // replicas whose loads are issued together
constexpr int kMaxBlocks = 8192; // per-block partials held by the workspace
constexpr int kRegWaves = 4;     // register kernels: grid = kRegWaves x resident blocks per SM x SMs

// Workspace: [ticket:uint32][pad to 256 B][partials: double x kMaxBlocks]
constexpr size_t kWsPartialsOffset = 256;
constexpr size_t kWorkspaceBytes = kWsPartialsOffset + sizeof(double) * kMaxBlocks;

struct Consts {
    float lr, b1, b2, eps, inv, omb1, omb2, rbc1, rsbc2, decay;
    float clip;  // gradient multiplier of global-norm clipping; 1 when not clipping
};

// Step kernels the host can launch for a prepared call (StepParams::kind).
constexpr int32_t kKindRegister = 0;  // fused_step_kernel: 8 elements per thread
constexpr int32_t kKindPipe = 1;      // fused_step_pipe_kernel: bulk-copy tiles through shared memory
constexpr int32_t kKindQuad = 2;      // fused_step_quad_kernel: 4 elements per thread, plain loads (N <= 16)
constexpr int32_t kKindOct = 3;       // fused_step_oct_kernel: 8 elements per thread, 32-byte state stores

struct StepParams {
    const void* grads[ZERO_MAX_WORLD];  // already offset to the call's first element
    int32_t world;
    int64_t count;  // elements processed
    int64_t head;   // elements [0, head) take the scalar path
    int64_t nvec;   // vectors of kVec elements starting at `head`
    int32_t tile;   // elements per pipeline tile (pipeline kernels only)
    int32_t kind;   // which step kernel the host launches: kKindRegister / kKindPipe / kKindQuad / kKindOct
    int32_t st32;   // 1: the fp32 outputs are 32-byte aligned at `head` (32-byte state stores)
    const float* master_in;
    const float* m_in;
    const float* v_in;
    float* master_out;
    float* m_out;
    float* v_out;
    void* param_out;
    Consts c;
    int32_t* overflow;
    double* sqnorm;
    double* partials;
    unsigned int* ticket;
    const int32_t* gate;        // device; when not NULL and non-zero the kernel writes nothing
    const double* clip_sqnorm;  // device; when not NULL, clip gradients to norm max_norm
    double max_norm;
};

// ---------------------------------------------------------------- loads/stores

// Loads of the register kernels: the read-only path for gradients, plain
// loads for states (which may be written in place); no L1 no-allocate hint
// (measured on B200 it cost 2-3 % on these streams).
__device__ __forceinline__ uint4 ld_grad16(const void* p) {
    uint4 r;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ float4 ld_state16(const float* p) {
    float4 r;
    asm volatile("ld.global.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_state16(float* p, float a, float b, float c, float d) {
    asm volatile("st.global.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// One 32-byte store of 8 fp32 values (a 32-byte aligned address).  On B200
// the store width sets the rate of write-heavy streams: a 1:1 copy with
// 32-byte stores runs 3-4 % faster than with 16-byte stores.
__device__ __forceinline__ void st_state32(float* p, const float* w) {
    asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(w[0]), "f"(w[1]), "f"(w[2]),
                 "f"(w[3]), "f"(w[4]), "f"(w[5]), "f"(w[6]), "f"(w[7])
                 : "memory");
}

__device__ __forceinline__ void st_u16x4(void* p, uint2 v) {
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ void st_u16x8(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// -------------------------------------------------------------- conversions

template <typename T>
struct Fmt;

template <>
struct Fmt<__half> {
    static __device__ __forceinline__ float lo(uint32_t w) {
        return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu)));
    }
    static __device__ __forceinline__ float hi(uint32_t w) {
        return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
    }
    static __device__ __forceinline__ float one(uint16_t b) { return __half2float(__ushort_as_half(b)); }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);  // round to nearest even, a in the low half
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint16_t round1(float a) { return __half_as_ushort(__float2half_rn(a)); }
};

template <>
struct Fmt<__nv_bfloat16> {
    static __device__ __forceinline__ float lo(uint32_t w) { return __uint_as_float(w << 16); }
    static __device__ __forceinline__ float hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
    static __device__ __forceinline__ float one(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint16_t round1(float a) {
        return __bfloat16_as_ushort(__float2bfloat16_rn(a));
    }
};

template <typename GT>
__device__ __forceinline__ void cvt8(const uint4& r, float* s) {
    s[0] = Fmt<GT>::lo(r.x); s[1] = Fmt<GT>::hi(r.x);
    s[2] = Fmt<GT>::lo(r.y); s[3] = Fmt<GT>::hi(r.y);
    s[4] = Fmt<GT>::lo(r.z); s[5] = Fmt<GT>::hi(r.z);
    s[6] = Fmt<GT>::lo(r.w); s[7] = Fmt<GT>::hi(r.w);
}

template <typename GT>
__device__ __forceinline__ void add8(const uint4& r, float* s) {
    s[0] = __fadd_rn(s[0], Fmt<GT>::lo(r.x)); s[1] = __fadd_rn(s[1], Fmt<GT>::hi(r.x));
    s[2] = __fadd_rn(s[2], Fmt<GT>::lo(r.y)); s[3] = __fadd_rn(s[3], Fmt<GT>::hi(r.y));
    s[4] = __fadd_rn(s[4], Fmt<GT>::lo(r.z)); s[5] = __fadd_rn(s[5], Fmt<GT>::hi(r.z));
    s[6] = __fadd_rn(s[6], Fmt<GT>::lo(r.w)); s[7] = __fadd_rn(s[7], Fmt<GT>::hi(r.w));
}

// ------------------------------------------------------------------ the update

// Adam with bias correction, epsilon outside the square root, decoupled
// weight decay; every operation explicitly rounded so that no contraction
// changes the result.  Returns the unscaled gradient g for the norm.
__device__ __forceinline__ float adam(float s, float& p, float& m, float& v, const Consts& c) {
    const float g = __fmul_rn(__fmul_rn(s, c.inv), c.clip);
    const float mn = __fmaf_rn(c.b1, m, __fmul_rn(c.omb1, g));
    const float vn = __fmaf_rn(c.b2, v, __fmul_rn(__fmul_rn(c.omb2, g), g));
    const float den = __fmaf_rn(__fsqrt_rn(vn), c.rsbc2, c.eps);
    const float u = __fdiv_rn(__fmul_rn(mn, c.rbc1), den);
    p = __fmaf_rn(-c.lr, u, __fmul_rn(p, c.decay));
    m = mn;
    v = vn;
    return g;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Flag bit of debug builds (ZERO_DEBUG_BOUNDS): an index check failed.
constexpr int32_t kFlagBounds = 4;

// Index check of debug builds: when `ok` is false, record kFlagBounds in
// *flag and return true so that the caller skips the access.  In release
// builds it is the constant false and compiles away.
__device__ __forceinline__ bool out_of_bounds(bool ok, int32_t* flag) {
#ifdef ZERO_DEBUG_BOUNDS
    if (!ok) {
        atomicOr(flag, kFlagBounds);
        return true;
    }
#endif
    (void)ok;
    (void)flag;
    return false;
}

// Gate and clip, read once per thread from device memory: returns false
// (write nothing) when the gate is set; otherwise sets c.clip from the
// global squared norm, min(1, max_norm / (sqrt(sqnorm) + 1e-6)) computed in
// double and rounded once to float.  Every thread of the grid takes the
// same branch.
__device__ __forceinline__ bool step_prologue(const StepParams& p, Consts& c) {
    if (p.gate != nullptr && *reinterpret_cast<const volatile int32_t*>(p.gate) != 0) return false;
    if (p.clip_sqnorm != nullptr) {
        const double coef = p.max_norm / (sqrt(*p.clip_sqnorm) + 1e-6);
        c.clip = coef < 1.0 ? static_cast<float>(coef) : 1.0f;
    }
    return true;
}

// Elements outside the vector (or tile) region: [0, head) and
// [head + nvec*kVec, count), one element per thread and iteration.
template <typename GT, typename PT>
__device__ __forceinline__ void scalar_elements(const StepParams& p, const Consts& c, int64_t tid, int64_t nthreads,
                                                bool& bad, double& sq) {
    const int world = p.world;
    const int64_t vec_end = p.head + p.nvec * kVec;
    const int64_t nscalar = p.head + (p.count - vec_end);
    for (int64_t q = tid; q < nscalar; q += nthreads) {
        const int64_t e = q < p.head ? q : vec_end + (q - p.head);
        if (out_of_bounds(e >= 0 && e < p.count, p.overflow)) continue;
        float s = Fmt<GT>::one(static_cast<const uint16_t*>(p.grads[0])[e]);
        for (int k = 1; k < world; ++k)
            s = __fadd_rn(s, Fmt<GT>::one(static_cast<const uint16_t*>(p.grads[k])[e]));
        float pw = p.master_in[e], mw = p.m_in[e], vw = p.v_in[e];
        bad |= !isfinite(s);
        const float g = adam(s, pw, mw, vw, c);
        if (p.sqnorm) sq = fma(static_cast<double>(g), static_cast<double>(g), sq);
        p.master_out[e] = pw;
        p.m_out[e] = mw;
        p.v_out[e] = vw;
        static_cast<uint16_t*>(p.param_out)[e] = Fmt<PT>::round1(pw);
    }
}

// Overflow vote and the optional deterministic norm fold.  Every thread of
// the block must call it (it synchronizes the block).
template <int NT>
__device__ __forceinline__ void finish_block(const StepParams& p, bool bad, double sq) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // one atomic per warp that saw a non-finite sum
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.overflow, 1);
    if (p.sqnorm == nullptr) return;
    __shared__ double wsum[NT / 32];
    __shared__ bool last;
    sq = warp_sum_d(sq);
    if (lane == 0) wsum[warp] = sq;
    __syncthreads();
    if (warp == 0) {
        double x = lane < NT / 32 ? wsum[lane] : 0.0;
        x = warp_sum_d(x);
        if (lane == 0) {
            p.partials[blockIdx.x] = x;
            __threadfence();
            const unsigned int t = atomicAdd(p.ticket, 1u);
            last = (t == gridDim.x - 1);
        }
    }
    __syncthreads();
    if (last && warp == 0) {
        __threadfence();
        double acc = 0.0;
        for (unsigned int b = lane; b < gridDim.x; b += 32) acc += __ldcg(p.partials + b);
        acc = warp_sum_d(acc);
        if (lane == 0) {
            *p.sqnorm += acc;
            *p.ticket = 0u;  // leave the workspace ready for the next call
        }
    }
}

// Register-streaming kernel: each thread loads its kVec elements of every
// stream straight into registers.  Used for buffers whose 16-byte phases
// differ, for small calls and for very large N.
template <typename GT, typename PT>
__global__ void __launch_bounds__(kThreads) fused_step_kernel(const __grid_constant__ StepParams p) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    const int world = p.world;
    Consts c = p.c;
    if (!step_prologue(p, c)) return;
    bool bad = false;
    double sq = 0.0;

    // ---- vector path: kVec elements per iteration, 16-byte accesses
    for (int64_t vi = tid; vi < p.nvec; vi += nthreads) {
        const int64_t e0 = p.head + vi * kVec;
        if (out_of_bounds(e0 + kVec <= p.count, p.overflow)) continue;
        // state first, so that its loads are in flight while gradients arrive
        const float4 pa = ld_state16(p.master_in + e0), pb = ld_state16(p.master_in + e0 + 4);
        const float4 ma = ld_state16(p.m_in + e0), mb = ld_state16(p.m_in + e0 + 4);
        const float4 va = ld_state16(p.v_in + e0), vb = ld_state16(p.v_in + e0 + 4);

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

        float pw[kVec] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
        float mw[kVec] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
        float vw[kVec] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            bad |= !isfinite(s[e]);
            const float g = adam(s[e], pw[e], mw[e], vw[e], c);
            if (p.sqnorm) sq = fma(static_cast<double>(g), static_cast<double>(g), sq);
        }
        st_state16(p.master_out + e0, pw[0], pw[1], pw[2], pw[3]);
        st_state16(p.master_out + e0 + 4, pw[4], pw[5], pw[6], pw[7]);
        st_state16(p.m_out + e0, mw[0], mw[1], mw[2], mw[3]);
        st_state16(p.m_out + e0 + 4, mw[4], mw[5], mw[6], mw[7]);
        st_state16(p.v_out + e0, vw[0], vw[1], vw[2], vw[3]);
        st_state16(p.v_out + e0 + 4, vw[4], vw[5], vw[6], vw[7]);
        uint4 q;
        q.x = Fmt<PT>::pack(pw[0], pw[1]);
        q.y = Fmt<PT>::pack(pw[2], pw[3]);
        q.z = Fmt<PT>::pack(pw[4], pw[5]);
        q.w = Fmt<PT>::pack(pw[6], pw[7]);
        st_u16x8(static_cast<uint16_t*>(p.param_out) + e0, q);
    }

    scalar_elements<GT, PT>(p, c, tid, nthreads, bad, sq);
    finish_block<kThreads>(p, bad, sq);
}

// ------------------------------------------------------- quad-streaming kernel

constexpr int kQuadBlocksPerSm = 16;  // blocks of the grid per SM (several waves)
constexpr int kQuadMaxWorld = 16;     // largest N with a quad-kernel instance

__device__ __forceinline__ uint2 ld_u2(const void* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ float4 ld_f4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// Quad-streaming kernel for N <= B replicas: thread t updates quads (4
// consecutive elements) t, t + T, ..., U of them per iteration, issuing every
// load of those U quads before using any (U x N 8-byte gradient loads, 3U
// 16-byte state loads; plain loads, no cache hints) over a grid of several
// waves.  Measured on B200 against the pipeline kernel (at 16M elements:
// 0.95-1.06 of a measured B200 copy rate (6.43 TB/s) for N = 1..16, against
// 0.84-1.03; at 1B elements and N <= 2: 0.98 against 0.97).  The vector
// region is [head, head + 8 nvec) as for the other kernels; the rest takes
// the scalar path.
template <typename GT, typename PT, int B, int U, int NT>
__global__ void __launch_bounds__(NT, NT >= 512 ? 2 : 3) fused_step_quad_kernel(const __grid_constant__ StepParams p) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * NT + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * NT;
    const int world = p.world;
    Consts c = p.c;
    if (!step_prologue(p, c)) return;
    bool bad = false;
    double sq = 0.0;
    const int64_t nq = 2 * p.nvec;
    for (int64_t q0 = tid; q0 < nq; q0 += U * nthreads) {
        uint2 r[U][B];
        float4 pw[U], mw[U], vw[U];
        bool live[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t e0 = p.head + 4 * (q0 + u * nthreads);
            live[u] = q0 + u * nthreads < nq && !out_of_bounds(e0 + 4 <= p.count, p.overflow);
            if (!live[u]) continue;
#pragma unroll
            for (int k = 0; k < B; ++k)
                if (k < world) r[u][k] = ld_u2(static_cast<const uint16_t*>(p.grads[k]) + e0);
            pw[u] = ld_f4(p.master_in + e0);
            mw[u] = ld_f4(p.m_in + e0);
            vw[u] = ld_f4(p.v_in + e0);
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
            const float g0 = adam(s0, pw[u].x, mw[u].x, vw[u].x, c);
            const float g1 = adam(s1, pw[u].y, mw[u].y, vw[u].y, c);
            const float g2 = adam(s2, pw[u].z, mw[u].z, vw[u].z, c);
            const float g3 = adam(s3, pw[u].w, mw[u].w, vw[u].w, c);
            if (p.sqnorm) {
                sq = fma(static_cast<double>(g0), static_cast<double>(g0), sq);
                sq = fma(static_cast<double>(g1), static_cast<double>(g1), sq);
                sq = fma(static_cast<double>(g2), static_cast<double>(g2), sq);
                sq = fma(static_cast<double>(g3), static_cast<double>(g3), sq);
            }
            st_state16(p.master_out + e0, pw[u].x, pw[u].y, pw[u].z, pw[u].w);
            st_state16(p.m_out + e0, mw[u].x, mw[u].y, mw[u].z, mw[u].w);
            st_state16(p.v_out + e0, vw[u].x, vw[u].y, vw[u].z, vw[u].w);
            uint2 pk;
            pk.x = Fmt<PT>::pack(pw[u].x, pw[u].y);
            pk.y = Fmt<PT>::pack(pw[u].z, pw[u].w);
            st_u16x4(static_cast<uint16_t*>(p.param_out) + e0, pk);
        }
    }
    scalar_elements<GT, PT>(p, c, tid, nthreads, bad, sq);
    finish_block<NT>(p, bad, sq);
}

// Oct-streaming kernel for N <= B replicas: thread t updates octs (8
// consecutive elements) t, t + T, ..., issuing every load of an oct (N
// 16-byte gradient loads, 6 16-byte state loads) before using any, then one
// 32-byte store per state array and one 16-byte parameter store; a grid of
// several waves.  It needs the fp32 outputs 32-byte aligned at the vector
// region's start (StepParams::st32, set by the host).
template <typename GT, typename PT, int B, int NT, int MINB>
__global__ void __launch_bounds__(NT, MINB) fused_step_oct_kernel(const __grid_constant__ StepParams p) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * NT + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * NT;
    const int world = p.world;
    Consts c = p.c;
    if (!step_prologue(p, c)) return;
    bool bad = false;
    double sq = 0.0;
    for (int64_t vi = tid; vi < p.nvec; vi += nthreads) {
        const int64_t e0 = p.head + vi * kVec;
        if (out_of_bounds(e0 + kVec <= p.count, p.overflow)) continue;
        uint4 r[B];
#pragma unroll
        for (int k = 0; k < B; ++k)
            if (k < world) r[k] = ld_grad16(static_cast<const uint16_t*>(p.grads[k]) + e0);
        const float4 p0 = ld_f4(p.master_in + e0), p1 = ld_f4(p.master_in + e0 + 4);
        const float4 m0 = ld_f4(p.m_in + e0), m1 = ld_f4(p.m_in + e0 + 4);
        const float4 v0 = ld_f4(p.v_in + e0), v1 = ld_f4(p.v_in + e0 + 4);
        // rank-order fp32 sum
        float s[kVec];
        cvt8<GT>(r[0], s);
#pragma unroll
        for (int k = 1; k < B; ++k)
            if (k < world) add8<GT>(r[k], s);
        float pw[kVec] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        float mw[kVec] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        float vw[kVec] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            bad |= !isfinite(s[e]);
            const float g = adam(s[e], pw[e], mw[e], vw[e], c);
            if (p.sqnorm) sq = fma(static_cast<double>(g), static_cast<double>(g), sq);
        }
        st_state32(p.master_out + e0, pw);
        st_state32(p.m_out + e0, mw);
        st_state32(p.v_out + e0, vw);
        uint4 q;
        q.x = Fmt<PT>::pack(pw[0], pw[1]);
        q.y = Fmt<PT>::pack(pw[2], pw[3]);
        q.z = Fmt<PT>::pack(pw[4], pw[5]);
        q.w = Fmt<PT>::pack(pw[6], pw[7]);
        st_u16x8(static_cast<uint16_t*>(p.param_out) + e0, q);
    }
    scalar_elements<GT, PT>(p, c, tid, nthreads, bad, sq);
    finish_block<NT>(p, bad, sq);
}

// Shapes of the oct kernel by replica count: NT threads per block, the
// blocks per SM its registers are sized for (no spills) and the blocks per
// SM of the grid (several waves).
template <int B> struct OctShape;
template <> struct OctShape<2> { static constexpr int NT = 512, MINB = 2, BPS = 16; };
template <> struct OctShape<4> { static constexpr int NT = 256, MINB = 3, BPS = 16; };
template <> struct OctShape<8> { static constexpr int NT = 256, MINB = 2, BPS = 16; };
template <> struct OctShape<16> { static constexpr int NT = 256, MINB = 2, BPS = 16; };

// Shapes of the quad kernel by replica count: B replicas' loads and U quads
// in flight per thread, NT threads per block (two or three blocks per SM at
// the registers these shapes take).
template <int B> struct QuadShape;
template <> struct QuadShape<2> { static constexpr int U = 2, NT = 512; };
template <> struct QuadShape<4> { static constexpr int U = 2, NT = 512; };
template <> struct QuadShape<8> { static constexpr int U = 1, NT = 512; };
template <> struct QuadShape<16> { static constexpr int U = 1, NT = 256; };

// ------------------------------------------------------- bulk-copy pipeline

constexpr int kPipeStages = 2;
constexpr int kPipeConsumerWarps = 16;
constexpr int kPipeThreads = (kPipeConsumerWarps + 1) * 32;   // + one producer warp

// Device bit set in *overflow when a pipeline wait ran out of time: the
// call's outputs are incomplete and must not be committed.
constexpr int32_t kFlagDeviceTimeout = 2;

// Pipeline kernel: one CTA per SM.  A producer warp streams tiles of `tile`
// elements of every input (N gradient slices, master, m, v) into a ring of
// kPipeStages shared-memory stages with 1-D bulk copies that complete on an
// mbarrier; kPipeConsumerWarps warps reduce, update and store each tile
// straight to global memory (coalesced 16-byte stores) and release the
// stage.  Stage layout: N x tile gradients, then tile x fp32 master, m, v.
template <typename GT, typename PT>
__global__ void __launch_bounds__(kPipeThreads, 1) fused_step_pipe_kernel(const __grid_constant__ StepParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kPipeStages];
    __shared__ __align__(8) uint64_t empty[kPipeStages];
    __shared__ int abort_flag;
    const int world = p.world;
    const int T = p.tile;
    const uint32_t gbytes = 2u * static_cast<uint32_t>(T);
    const uint32_t sbytes = 4u * static_cast<uint32_t>(T);
    const uint32_t stage = static_cast<uint32_t>(world) * gbytes + 3u * sbytes;
    const int64_t ntiles = p.nvec * kVec / T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Consts c = p.c;
    if (!step_prologue(p, c)) return;   // uniform over the grid: before any barrier is set up
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
        // ---- producer warp: lane 0 arms the stage, all lanes issue copies
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
            for (int q = lane; q < world + 3; q += 32) {
                if (q < 3) {
                    const float* src = q == 0 ? p.master_in : (q == 1 ? p.m_in : p.v_in);
                    bulk_load(st + static_cast<size_t>(world) * gbytes + q * sbytes, src + e0, sbytes, &full[s]);
                } else {
                    const int k = q - 3;
                    bulk_load(st + static_cast<size_t>(k) * gbytes, static_cast<const uint16_t*>(p.grads[k]) + e0,
                              gbytes, &full[s]);
                }
            }
        }
        // drain: this CTA's copies must land before it exits (bounded)
        if (lane == 0) {
            const int64_t issued = i;
            for (int64_t j = issued > kPipeStages ? issued - kPipeStages : 0; j < issued; ++j)
                if (!mbar_wait_bounded(&full[j % kPipeStages], static_cast<uint32_t>((j / kPipeStages) & 1)))
                    atomicOr(p.overflow, kFlagDeviceTimeout);
        }
        __syncwarp();
    } else {
        // ---- consumer warps: thread t takes 4 elements per chunk
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
            const float* sm_p = reinterpret_cast<const float*>(st + static_cast<size_t>(world) * gbytes);
            const float* sm_m = sm_p + T;
            const float* sm_v = sm_m + T;
            const int64_t base = p.head + tile * T;
            for (int ch = t; ch < T / 4; ch += C) {
                const int j = 4 * ch;
                if (out_of_bounds(j + 4 <= T && base + j + 4 <= p.count, p.overflow)) continue;
                float sacc[4];
                const uint2 r0 = *reinterpret_cast<const uint2*>(st + 2 * j);
                sacc[0] = Fmt<GT>::lo(r0.x);
                sacc[1] = Fmt<GT>::hi(r0.x);
                sacc[2] = Fmt<GT>::lo(r0.y);
                sacc[3] = Fmt<GT>::hi(r0.y);
#pragma unroll 4
                for (int k = 1; k < world; ++k) {
                    const uint2 r = *reinterpret_cast<const uint2*>(st + static_cast<size_t>(k) * gbytes + 2 * j);
                    sacc[0] = __fadd_rn(sacc[0], Fmt<GT>::lo(r.x));
                    sacc[1] = __fadd_rn(sacc[1], Fmt<GT>::hi(r.x));
                    sacc[2] = __fadd_rn(sacc[2], Fmt<GT>::lo(r.y));
                    sacc[3] = __fadd_rn(sacc[3], Fmt<GT>::hi(r.y));
                }
                float4 pw = *reinterpret_cast<const float4*>(sm_p + j);
                float4 mw = *reinterpret_cast<const float4*>(sm_m + j);
                float4 vw = *reinterpret_cast<const float4*>(sm_v + j);
                bad |= !isfinite(sacc[0]) | !isfinite(sacc[1]) | !isfinite(sacc[2]) | !isfinite(sacc[3]);
                const float g0 = adam(sacc[0], pw.x, mw.x, vw.x, c);
                const float g1 = adam(sacc[1], pw.y, mw.y, vw.y, c);
                const float g2 = adam(sacc[2], pw.z, mw.z, vw.z, c);
                const float g3 = adam(sacc[3], pw.w, mw.w, vw.w, c);
                if (p.sqnorm) {
                    sq = fma(static_cast<double>(g0), static_cast<double>(g0), sq);
                    sq = fma(static_cast<double>(g1), static_cast<double>(g1), sq);
                    sq = fma(static_cast<double>(g2), static_cast<double>(g2), sq);
                    sq = fma(static_cast<double>(g3), static_cast<double>(g3), sq);
                }
                st_state16(p.master_out + base + j, pw.x, pw.y, pw.z, pw.w);
                st_state16(p.m_out + base + j, mw.x, mw.y, mw.z, mw.w);
                st_state16(p.v_out + base + j, vw.x, vw.y, vw.z, vw.w);
                uint2 pk;
                pk.x = Fmt<PT>::pack(pw.x, pw.y);
                pk.y = Fmt<PT>::pack(pw.z, pw.w);
                st_u16x4(static_cast<uint16_t*>(p.param_out) + base + j, pk);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        // the scalar head and tail, spread over every consumer thread of the grid
        scalar_elements<GT, PT>(p, c, static_cast<int64_t>(blockIdx.x) * C + t, static_cast<int64_t>(gridDim.x) * C,
                                bad, sq);
    }
    finish_block<kPipeThreads>(p, bad, sq);
}

// ------------------------------------------------------------------ host side

// Self-test of the bounded wait: one thread waits on an mbarrier that
// nothing ever arrives at, with a short limit.  It must give up, record
// kFlagDeviceTimeout in *status and return; the CTA's shared memory holds no
// copy in flight, so nothing else needs draining.
__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait_bounded(&bar, 0u, limit_ns)) atomicOr(status, kFlagDeviceTimeout);
}

}  // namespace
}  // namespace fused
}  // namespace zero

