// Device code of the fused ZeRO-2 step kernel and the host helpers that
// size its grid; included by every translation unit that launches it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

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

// Workspace: [ticket:uint32][pad to 256 B][partials: float x kMaxBlocks]
constexpr size_t kWsPartialsOffset = 256;
constexpr size_t kWorkspaceBytes = kWsPartialsOffset + sizeof(float) * kMaxBlocks;

struct Consts {
    float lr, b1, b2, eps, inv, omb1, omb2, rbc1, rsbc2, decay;
};

struct StepParams {
    const void* grads[ZERO_MAX_WORLD];  // already offset to the call's first element
    int32_t world;
    int64_t count;  // elements processed
    int64_t head;   // elements [0, head) take the scalar path
    int64_t nvec;   // vectors of kVec elements starting at `head`
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
    float* partials;
    unsigned int* ticket;
};

// ---------------------------------------------------------------- loads/stores

__device__ __forceinline__ uint4 ld_grad16(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ float4 ld_state16(const float* p) {
    float4 r;
    asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_state16(float* p, float a, float b, float c, float d) {
    asm volatile("st.global.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
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
    const float g = __fmul_rn(s, c.inv);
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

template <typename GT, typename PT>
__global__ void __launch_bounds__(kThreads) fused_step_kernel(const __grid_constant__ StepParams p) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    const int world = p.world;
    const Consts c = p.c;
    bool bad = false;
    float sq = 0.0f;

    // ---- vector path: kVec elements per iteration, 16-byte accesses
    for (int64_t vi = tid; vi < p.nvec; vi += nthreads) {
        const int64_t e0 = p.head + vi * kVec;
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
            sq = __fmaf_rn(g, g, sq);
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

    // ---- scalar path: the head before and the tail after the vector region
    const int64_t vec_end = p.head + p.nvec * kVec;
    const int64_t nscalar = p.head + (p.count - vec_end);
    for (int64_t q = tid; q < nscalar; q += nthreads) {
        const int64_t e = q < p.head ? q : vec_end + (q - p.head);
        float s = Fmt<GT>::one(static_cast<const uint16_t*>(p.grads[0])[e]);
        for (int k = 1; k < world; ++k)
            s = __fadd_rn(s, Fmt<GT>::one(static_cast<const uint16_t*>(p.grads[k])[e]));
        float pw = p.master_in[e], mw = p.m_in[e], vw = p.v_in[e];
        bad |= !isfinite(s);
        const float g = adam(s, pw, mw, vw, c);
        sq = __fmaf_rn(g, g, sq);
        p.master_out[e] = pw;
        p.m_out[e] = mw;
        p.v_out[e] = vw;
        static_cast<uint16_t*>(p.param_out)[e] = Fmt<PT>::round1(pw);
    }

    // ---- overflow flag: one atomic per warp that saw a non-finite sum
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.overflow, 1);

    // ---- optional squared norm, deterministic fold by the last block
    if (p.sqnorm != nullptr) {
        __shared__ float wsum[kThreads / 32];
        __shared__ bool last;
        sq = warp_sum(sq);
        if (lane == 0) wsum[warp] = sq;
        __syncthreads();
        if (warp == 0) {
            float x = lane < kThreads / 32 ? wsum[lane] : 0.0f;
            x = warp_sum(x);
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
            for (unsigned int b = lane; b < gridDim.x; b += 32) acc += static_cast<double>(__ldcg(p.partials + b));
            acc = warp_sum_d(acc);
            if (lane == 0) {
                *p.sqnorm += acc;
                *p.ticket = 0u;  // leave the workspace ready for the next call
            }
        }
    }
}

// ------------------------------------------------------------------ host side

using KernelFn = void (*)(StepParams);

inline KernelFn pick_kernel(zero_dtype_t g, zero_dtype_t pd) {
    if (g == ZERO_F16 && pd == ZERO_F16) return fused_step_kernel<__half, __half>;
    if (g == ZERO_F16 && pd == ZERO_BF16) return fused_step_kernel<__half, __nv_bfloat16>;
    if (g == ZERO_BF16 && pd == ZERO_F16) return fused_step_kernel<__nv_bfloat16, __half>;
    return fused_step_kernel<__nv_bfloat16, __nv_bfloat16>;
}

struct DeviceInfo {
    int sms = 0;
    int blocks_per_sm[4] = {0, 0, 0, 0};
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

inline int grid_limit(zero_dtype_t g, zero_dtype_t pd, int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return fail(ZERO_ERR_CUDA, "cudaGetDevice failed");
    const int which = static_cast<int>(g) * 2 + static_cast<int>(pd);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (d.sms == 0) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return fail(ZERO_ERR_CUDA, "cannot query the SM count");
    }
    if (d.blocks_per_sm[which] == 0) {
        int n = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, pick_kernel(g, pd), kThreads, 0);
        if (e != cudaSuccess || n < 1) return fail(ZERO_ERR_CUDA, "occupancy query failed: %s", cudaGetErrorString(e));
        d.blocks_per_sm[which] = n;
    }
    int lim = d.sms * d.blocks_per_sm[which];
    *out = lim < kMaxBlocks ? lim : kMaxBlocks;
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
    if (!(hp->step >= 1)) return fail(ZERO_ERR_ARG, "%s: hp->step must be >= 1", fn);
    if (!std::isfinite(hp->lr) || !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay) ||
        !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) ||
        !(hp->grad_divisor >= 0.0f) || !std::isfinite(hp->grad_divisor))
        return fail(ZERO_ERR_ARG, "%s: hyper-parameters out of range", fn);
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
        prm.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsPartialsOffset);
    }
    // constants: double, rounded once to float
    const double divisor = hp->grad_divisor > 0.0f ? static_cast<double>(hp->grad_divisor) : static_cast<double>(world);
    const double t = static_cast<double>(hp->step);
    prm.c.lr = hp->lr;
    prm.c.b1 = hp->beta1;
    prm.c.b2 = hp->beta2;
    prm.c.eps = hp->eps;
    prm.c.inv = static_cast<float>(1.0 / (divisor * static_cast<double>(loss_scale)));
    prm.c.omb1 = static_cast<float>(1.0 - static_cast<double>(hp->beta1));
    prm.c.omb2 = static_cast<float>(1.0 - static_cast<double>(hp->beta2));
    prm.c.rbc1 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(hp->beta1), t)));
    prm.c.rsbc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(hp->beta2), t)));
    prm.c.decay = static_cast<float>(1.0 - static_cast<double>(hp->lr) * static_cast<double>(hp->weight_decay));

    const int64_t h = common_phase(prm);
    if (h < 0 || h >= count) {
        prm.head = count;
        prm.nvec = 0;
    } else {
        prm.head = h;
        prm.nvec = (count - h) / kVec;
    }

    int limit = 0;
    if (int rc = grid_limit(grad_dtype, param_dtype, &limit)) return rc;
    const int64_t work = prm.nvec > 0 ? prm.nvec : count;
    int64_t blocks = (work + kThreads - 1) / kThreads;
    if (blocks > limit) blocks = limit;
    if (blocks < 1) blocks = 1;
    *prm_out = prm;
    *blocks_out = blocks;
    return ZERO_OK;
}

// Enqueue the fused kernel prepared by prepare_step.
inline int launch_step(const char* fn, const StepParams& prm, int64_t blocks, zero_dtype_t grad_dtype,
                       zero_dtype_t param_dtype, zero_stream_t stream) {
    if (blocks == 0) return ok();
    KernelFn k = pick_kernel(grad_dtype, param_dtype);
    k<<<static_cast<unsigned int>(blocks), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    return ok();
}

}  // namespace
}  // namespace fused
}  // namespace zero

