// Statistics pre-pass and gated step: the in-place ZeRO step with an exact
// skip, and global gradient-norm clipping.
//
// The fused single-pass step writes its update before the step-wide
// overflow verdict exists, so an exact skip needs a second bank of states.
// The pages count the optimizer states once, 12 Psi / N bytes per rank (ZeRO
// explainer, "Stage 1 - Optimizer State Partitioning (P_os)").  With a
// statistics pass first (rank-order sums, overflow OR, squared norm; 2N bytes
// per element), the update can run in place, gated by the step's flag in
// device memory, and can scale the gradients by a clipping coefficient
// computed on the device from the norm: 4N + 26 bytes per element in total.
#include "step_launch.h"

using zero::fail;

extern "C" int zero_grad_stats(const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
                               zero_dtype_t grad_dtype, float loss_scale, float grad_divisor, int32_t* overflow_flag,
                               double* grad_sqnorm, void* workspace, zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_grad_stats";
    StepParams prm{};
    int64_t blocks = 0;
    if (int rc = prepare_stats(fn, grad_bufs, world, padded_numel, partition, grad_dtype, loss_scale, grad_divisor,
                               nullptr, overflow_flag, grad_sqnorm, workspace, &prm, &blocks))
        return rc;
    return launch_stats(fn, prm, blocks, grad_dtype, nullptr, stream);
}

extern "C" int zero_reduce_scatter_adam_step_gated(
    const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition, zero_dtype_t grad_dtype,
    const float* master_in, const float* m_in, const float* v_in, float* master_out, float* m_out, float* v_out,
    void* param_out, zero_dtype_t param_dtype, const zero_adam_hparams_t* hp, float loss_scale,
    int32_t* overflow_flag, double* grad_sqnorm, void* workspace, const int32_t* gate, const double* clip_sqnorm,
    float max_norm, zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_reduce_scatter_adam_step_gated";
    StepParams prm{};
    int64_t blocks = 0;
    if (int rc = prepare_step(fn, grad_bufs, world, padded_numel, partition, grad_dtype, master_in, m_in, v_in,
                              master_out, m_out, v_out, param_out, param_dtype, hp, loss_scale, overflow_flag,
                              grad_sqnorm, workspace, &prm, &blocks))
        return rc;
    if (int rc = add_gate_and_clip(fn, &prm, gate, clip_sqnorm, max_norm)) return rc;
    return launch_step(fn, prm, blocks, grad_dtype, param_dtype, stream);
}

