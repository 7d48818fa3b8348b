// The staged ZeRO-2 step: a reduce-scatter that stores each partition's
// reduced gradients in fp32, then the Adam update from them.
//
// ZeRO explainer (azimuth.plus), "Stage 2 - Gradient Partitioning (P_os+g)":
// the gradients are reduce-scattered so that each rank keeps only the
// reduced gradients of its own partition, and updates that partition.  The
// fused step never materialises them (2N + 26 bytes per element, but its
// exact skip needs a second bank of states); the statistics route re-reads
// the N replicas (4N + 26).  Staged, the reduce-scatter writes the reduced
// gradients once (2N + 4) and the update reads them back (30): 2N + 34 bytes
// per element with one bank of states plus 4 bytes per element of reduced
// gradients, the exact skip taken by the update's device-side gate.
#include "staged_launch.h"

using zero::fail;

extern "C" int zero_reduce_scatter_grads(const void* const* grad_bufs, int32_t world, int64_t padded_numel,
                                         int32_t partition, zero_dtype_t grad_dtype, float loss_scale,
                                         float grad_divisor, float* reduced_out, int32_t* overflow_flag,
                                         double* grad_sqnorm, void* workspace, zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_reduce_scatter_grads";
    if (!reduced_out) return fail(ZERO_ERR_ARG, "%s: NULL reduced_out", fn);
    StepParams prm{};
    int64_t blocks = 0;
    if (int rc = prepare_stats(fn, grad_bufs, world, padded_numel, partition, grad_dtype, loss_scale, grad_divisor,
                               reduced_out, overflow_flag, grad_sqnorm, workspace, &prm, &blocks))
        return rc;
    return launch_stats(fn, prm, blocks, grad_dtype, reduced_out, stream);
}

extern "C" int zero_adam_step_reduced(const float* reduced_grad, int64_t count, const float* master_in,
                                      const float* m_in, const float* v_in, float* master_out, float* m_out,
                                      float* v_out, void* param_out, zero_dtype_t param_dtype,
                                      const zero_adam_hparams_t* hp, int32_t* status, const int32_t* gate,
                                      const double* clip_sqnorm, float max_norm, zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_adam_step_reduced";
    if (!status) return fail(ZERO_ERR_ARG, "%s: NULL status", fn);
    if (!zero::aligned(status, 4)) return fail(ZERO_ERR_ALIGN, "%s: status misaligned", fn);
    StepParams prm{};
    int64_t work = 0;
    if (int rc = prepare_reduced(fn, reduced_grad, count, master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                                 param_dtype, hp, &prm, &work))
        return rc;
    prm.overflow = status;
    if (int rc = add_gate_and_clip(fn, &prm, gate, clip_sqnorm, max_norm)) return rc;
    if (work == 0) return zero::ok();
    ParamDsts d{};
    if (int rc = launch_reduced(fn, prm, d, work, param_dtype, false, stream)) return rc;
    return zero::ok();
}

extern "C" int zero_adam_step_reduced_bcast(const float* reduced_grad, int64_t count, const float* master_in,
                                            const float* m_in, const float* v_in, float* master_out, float* m_out,
                                            float* v_out, void* const* param_dsts, int32_t n_dsts,
                                            zero_dtype_t param_dtype, const zero_adam_hparams_t* hp, int32_t* status,
                                            const int32_t* gate, const double* clip_sqnorm, float max_norm,
                                            zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_adam_step_reduced_bcast";
    if (!status) return fail(ZERO_ERR_ARG, "%s: NULL status", fn);
    if (!zero::aligned(status, 4)) return fail(ZERO_ERR_ALIGN, "%s: status misaligned", fn);
    if (!param_dsts || n_dsts < 1 || n_dsts > ZERO_MAX_WORLD)
        return fail(ZERO_ERR_ARG, "%s: param_dsts must hold 1..%d destinations", fn, ZERO_MAX_WORLD);
    StepParams prm{};
    int64_t work = 0;
    // the first destination stands for all in the shared checks
    if (int rc = prepare_reduced(fn, reduced_grad, count, master_in, m_in, v_in, master_out, m_out, v_out,
                                 param_dsts[0], param_dtype, hp, &prm, &work))
        return rc;
    prm.overflow = status;
    if (int rc = add_gate_and_clip(fn, &prm, gate, clip_sqnorm, max_norm)) return rc;
    if (work == 0) return zero::ok();
    ParamDsts d{};
    d.n = n_dsts;
    const void* others[] = {reduced_grad, master_in, m_in, v_in, master_out, m_out, v_out};
    bool same_phase = true;
    for (int k = 0; k < n_dsts; ++k) {
        if (!param_dsts[k]) return fail(ZERO_ERR_ARG, "%s: param_dsts[%d] is NULL", fn, k);
        if (!zero::aligned(param_dsts[k], 2)) return fail(ZERO_ERR_ALIGN, "%s: param_dsts[%d] misaligned", fn, k);
        for (const void* o : others)
            if (zero::overlaps(param_dsts[k], count * 2, o, count * 4))
                return fail(ZERO_ERR_ARG, "%s: param_dsts[%d] overlaps an input or state array", fn, k);
        for (int j = 0; j < k; ++j)
            if (zero::overlaps(param_dsts[k], count * 2, param_dsts[j], count * 2))
                return fail(ZERO_ERR_ARG, "%s: param_dsts[%d] overlaps param_dsts[%d]", fn, k, j);
        same_phase = same_phase && ((reinterpret_cast<uintptr_t>(param_dsts[k]) -
                                     reinterpret_cast<uintptr_t>(param_dsts[0])) % 16) == 0;
        d.dst[k] = param_dsts[k];
    }
    if (!same_phase) {      // the destinations' 16-byte phases differ: element-wise stores only
        prm.head = count;
        prm.nvec = 0;
        work = count;
    }
    if (int rc = launch_reduced(fn, prm, d, work, param_dtype, true, stream)) return rc;
    return zero::ok();
}
