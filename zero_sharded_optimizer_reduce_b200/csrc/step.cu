// Fused ZeRO-2 step for sm_100a: reduce-scatter of N resident replica
// gradient buffers + loss-scale unscaling + overflow test + Adam/AdamW on the
// fp32 partition + low-precision parameter write-back, in one streaming pass.
//
// Method: ZeRO explainer (azimuth.plus, "ZeRO: Memory Optimizations Toward
// Training Trillion Parameter Models"), "Stage 2 - Gradient Partitioning
// (P_os+g)": each rank receives by reduce-scatter only the reduced gradients
// of its partition and updates that partition of the fp32 optimizer states;
// the updated fp16 parameters are what the all-gather then distributes
// ("Stage 1 - Optimizer State Partitioning (P_os)"); model states are fp16
// parameters and gradients plus fp32 master, momentum and variance
// (model-states paragraph).
//
// Per element the kernel moves 2N bytes of gradients in, 12 bytes of fp32
// state in, 12 bytes of state out and 2 bytes of parameters out, and does
// about 20 fp32 operations: HBM-bound, no tensor-core work.  Design:
//  - one element of work per (thread, vector of 8 elements); a persistent
//    grid of (SM count x resident blocks) strides over the vectors;
//  - 16-byte loads and stores for every stream (8 gradients of one replica,
//    2 x float4 of each state array, 8 parameters) on a common 16-byte phase;
//    elements outside that phase (head and tail) take a scalar path;
//  - gradients are read-only for the kernel's lifetime: non-coherent loads
//    that do not allocate in L1; state loads do not allocate in L1 either;
//  - the rank-order fp32 sum is kept per element in registers, replicas are
//    loaded in batches of 8 so that their loads are in flight together;
//  - the overflow test ORs !isfinite over the whole call with one warp vote
//    and at most one atomicOr per warp that saw a non-finite sum;
//  - the optional squared gradient norm is summed per thread in fp32, per
//    block by a fixed shuffle tree, and the last block (atomic ticket, no
//    grid barrier, no waiting) folds the per-block partials in block order in
//    double, so the result is deterministic.
#include "step_launch.h"

using zero::fail;

extern "C" size_t zero_step_workspace_bytes(void) { return zero::fused::kWorkspaceBytes; }

extern "C" int zero_reduce_scatter_adam_step(
    const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
    zero_dtype_t grad_dtype, const float* master_in, const float* m_in, const float* v_in,
    float* master_out, float* m_out, float* v_out, void* param_out, zero_dtype_t param_dtype,
    const zero_adam_hparams_t* hp, float loss_scale, int32_t* overflow_flag, double* grad_sqnorm,
    void* workspace, zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_reduce_scatter_adam_step";
    StepParams prm{};
    int64_t blocks = 0;
    if (int rc = prepare_step(fn, grad_bufs, world, padded_numel, partition, grad_dtype, master_in, m_in, v_in,
                              master_out, m_out, v_out, param_out, param_dtype, hp, loss_scale, overflow_flag,
                              grad_sqnorm, workspace, &prm, &blocks))
        return rc;
    return launch_step(fn, prm, blocks, grad_dtype, param_dtype, stream);
}
