// Device code of the staged ZeRO-2 step's second half: the Adam update of a
// partition from its reduced fp32 gradients (the output of the staged
// reduce-scatter, grad_stats.cuh with kWrite).  Reads 16 bytes per element
// (gradient, master, m, v), writes 14 (master, m, v, parameter): 30 bytes,
// against the fused step's 2N + 26 read in one pass.
#pragma once

#include "fused_step.cuh"

namespace zero {
namespace fused {
namespace {

__device__ __forceinline__ float4 ld_once16(const float* p) {
    const uint4 r = ld_grad16(p);
    return make_float4(__uint_as_float(r.x), __uint_as_float(r.y), __uint_as_float(r.z), __uint_as_float(r.w));
}

// p.grads[0] holds the reduced fp32 gradients g (already unscaled), indexed
// like the state arrays; p.c.inv is 1, so adam() forms g * clip exactly as
// the fused step forms (s * inv) * clip.  Gate and clip as in the fused
// step; no flag or norm (the reduce-scatter produced them).
template <typename PT>
__global__ void __launch_bounds__(kThreads) adam_reduced_kernel(const __grid_constant__ StepParams p) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    Consts c = p.c;
    if (!step_prologue(p, c)) return;
    const float* gin = static_cast<const float*>(p.grads[0]);

    for (int64_t vi = tid; vi < p.nvec; vi += nthreads) {
        const int64_t e0 = p.head + vi * kVec;
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

    // head and tail, one element per thread and iteration
    const int64_t vec_end = p.head + p.nvec * kVec;
    const int64_t nscalar = p.head + (p.count - vec_end);
    for (int64_t q = tid; q < nscalar; q += nthreads) {
        const int64_t e = q < p.head ? q : vec_end + (q - p.head);
        float pw = p.master_in[e], mw = p.m_in[e], vw = p.v_in[e];
        adam(gin[e], pw, mw, vw, c);
        p.master_out[e] = pw;
        p.m_out[e] = mw;
        p.v_out[e] = vw;
        static_cast<uint16_t*>(p.param_out)[e] = Fmt<PT>::round1(pw);
    }
}

}  // namespace
}  // namespace fused
}  // namespace zero
