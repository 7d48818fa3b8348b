// zero_runner: the whole ZeRO-2 step over a list of buckets, in C.
//
// A runner holds, for every bucket, the N replicas' gradient buffers and two
// banks of fp32 master / m / v and low-precision parameters (all owned by the
// caller), plus the step's scalars: t, the loss scale and the good-step
// count.  zero_runner_launch enqueues one step: clear the flag, run the
// fused kernel over every bucket reading bank `cur` and writing bank
// `cur ^ 1`, and copy the flag into the caller's pinned host word, all on
// one stream without waiting.  zero_runner_commit waits for that copy, then
// flips the bank when no reduced gradient of the step was inf or NaN,
// advances t, and updates the loss scale (zero_loss_scale_update); on
// overflow nothing changes but the scale (ZeRO explainer, "Stage 2 -
// Gradient Partitioning (P_os+g)" for the step; the skip and the scale
// rule are not on the pages).
//
// A staged runner (zero_runner_create_staged) keeps one bank: launch runs the
// staged reduce-scatter of every bucket into the caller's reduced-gradient
// buffers, then the update of every bucket from them in place, gated on the
// device by the step's flag; commit advances t when the flag stayed 0.  The
// bank never changes.
#include <cmath>
#include <new>
#include <vector>

#include "staged_launch.h"
#include "step_launch.h"

struct zero_runner {
    int32_t staged = 0;           // 0: two banks, fused step; 1: one bank, staged route
    std::vector<float*> reduced;  // staged: each bucket's reduced-gradient buffer
    float max_norm = 0.0f;        // staged: clip to this global norm when > 0
    int32_t world = 0;
    zero_dtype_t grad_dtype = ZERO_F16, param_dtype = ZERO_F16;
    zero_adam_hparams_t hp{};
    std::vector<int64_t> numel;
    std::vector<std::vector<const void*>> grads;
    std::vector<zero_bucket_banks_t> banks;
    int32_t* flag_dev = nullptr;
    volatile int32_t* flag_host = nullptr;
    double* sqnorm = nullptr;
    void* workspace = nullptr;
    int32_t cur = 0, good = 0, growth_interval = 1000, launched = 0;
    int64_t t = 0;
    float scale = 1.0f, min_scale = 1.0f;
};

using zero::fail;

extern "C" int zero_runner_create(const zero_bucket_banks_t* buckets, int64_t n_buckets, int32_t world,
                                  zero_dtype_t grad_dtype, zero_dtype_t param_dtype, const zero_adam_hparams_t* hp,
                                  float loss_scale, int32_t growth_interval, float min_scale, int32_t* flag_dev,
                                  int32_t* flag_host, double* grad_sqnorm, void* workspace, zero_runner_t** out) {
    const char* fn = "zero_runner_create";
    if (!out || !hp || !flag_dev || !flag_host || (n_buckets > 0 && !buckets) || n_buckets < 0)
        return fail(ZERO_ERR_ARG, "%s: NULL or bad argument", fn);
    if (world < 1 || world > ZERO_MAX_WORLD) return fail(ZERO_ERR_ARG, "%s: world %d outside 1..%d", fn, world, ZERO_MAX_WORLD);
    if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale) || !(min_scale > 0.0f) || growth_interval < 1)
        return fail(ZERO_ERR_ARG, "%s: bad loss-scale settings", fn);
    if (grad_sqnorm && !workspace) return fail(ZERO_ERR_ARG, "%s: grad_sqnorm needs a workspace", fn);
    zero_runner* r = new (std::nothrow) zero_runner();
    if (!r) return fail(ZERO_ERR_NOMEM, "%s: out of host memory", fn);
    r->world = world;
    r->grad_dtype = grad_dtype;
    r->param_dtype = param_dtype;
    r->hp = *hp;
    r->flag_dev = flag_dev;
    r->flag_host = flag_host;
    r->sqnorm = grad_sqnorm;
    r->workspace = workspace;
    r->scale = loss_scale;
    r->min_scale = min_scale;
    r->growth_interval = growth_interval;
    r->t = hp->step > 0 ? hp->step - 1 : 0;
    for (int64_t b = 0; b < n_buckets; ++b) {
        const zero_bucket_banks_t& d = buckets[b];
        if (!d.grad_bufs) {
            delete r;
            return fail(ZERO_ERR_ARG, "%s: bucket %lld has no gradient buffers", fn, (long long)b);
        }
        r->numel.push_back(d.padded_numel);
        r->grads.emplace_back(d.grad_bufs, d.grad_bufs + world);
        r->banks.push_back(d);
        r->banks.back().grad_bufs = nullptr;   // the runner keeps its own copy of the pointer list
    }
    // validate every bucket's call once, for both bank directions
    zero_adam_hparams_t probe = r->hp;
    probe.step = 1;
    for (size_t b = 0; b < r->banks.size(); ++b) {
        for (int c = 0; c < 2; ++c) {
            const zero_bucket_banks_t& d = r->banks[b];
            zero::fused::StepParams prm{};
            int64_t blocks = 0;
            int rc = zero::fused::prepare_step(fn, r->grads[b].data(), world, r->numel[b], ZERO_ALL_PARTITIONS,
                                               grad_dtype, d.master[c], d.m[c], d.v[c], d.master[c ^ 1], d.m[c ^ 1],
                                               d.v[c ^ 1], d.params[c ^ 1], param_dtype, &probe, loss_scale, flag_dev,
                                               grad_sqnorm, workspace, &prm, &blocks);
            if (rc) {
                delete r;
                return rc;
            }
        }
    }
    *out = r;
    return zero::ok();
}

extern "C" int zero_runner_create_staged(const zero_bucket_banks_t* buckets, int64_t n_buckets, int32_t world,
                                         zero_dtype_t grad_dtype, zero_dtype_t param_dtype,
                                         const zero_adam_hparams_t* hp, float loss_scale, int32_t growth_interval,
                                         float min_scale, float* const* reduced, float max_norm, int32_t* flag_dev,
                                         int32_t* flag_host, double* grad_sqnorm, void* workspace,
                                         zero_runner_t** out) {
    const char* fn = "zero_runner_create_staged";
    if (!out || !hp || !flag_dev || !flag_host || (n_buckets > 0 && (!buckets || !reduced)) || n_buckets < 0)
        return fail(ZERO_ERR_ARG, "%s: NULL or bad argument", fn);
    if (world < 1 || world > ZERO_MAX_WORLD) return fail(ZERO_ERR_ARG, "%s: world %d outside 1..%d", fn, world, ZERO_MAX_WORLD);
    if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale) || !(min_scale > 0.0f) || growth_interval < 1)
        return fail(ZERO_ERR_ARG, "%s: bad loss-scale settings", fn);
    if (!(max_norm >= 0.0f) || !std::isfinite(max_norm))
        return fail(ZERO_ERR_ARG, "%s: max_norm must be >= 0 and finite", fn);
    if (max_norm > 0.0f && !grad_sqnorm) return fail(ZERO_ERR_ARG, "%s: clipping needs grad_sqnorm", fn);
    if (grad_sqnorm && !workspace) return fail(ZERO_ERR_ARG, "%s: grad_sqnorm needs a workspace", fn);
    if (!zero::aligned(flag_dev, 8)) return fail(ZERO_ERR_ALIGN, "%s: flag_dev must be 8-byte aligned (2 words)", fn);
    zero_runner* r = new (std::nothrow) zero_runner();
    if (!r) return fail(ZERO_ERR_NOMEM, "%s: out of host memory", fn);
    r->staged = 1;
    r->max_norm = max_norm;
    r->world = world;
    r->grad_dtype = grad_dtype;
    r->param_dtype = param_dtype;
    r->hp = *hp;
    r->flag_dev = flag_dev;
    r->flag_host = flag_host;
    r->sqnorm = grad_sqnorm;
    r->workspace = workspace;
    r->scale = loss_scale;
    r->min_scale = min_scale;
    r->growth_interval = growth_interval;
    r->t = hp->step > 0 ? hp->step - 1 : 0;
    for (int64_t b = 0; b < n_buckets; ++b) {
        const zero_bucket_banks_t& d = buckets[b];
        if (!d.grad_bufs || !reduced[b]) {
            delete r;
            return fail(ZERO_ERR_ARG, "%s: bucket %lld has no gradient or reduced buffers", fn, (long long)b);
        }
        r->numel.push_back(d.padded_numel);
        r->grads.emplace_back(d.grad_bufs, d.grad_bufs + world);
        r->banks.push_back(d);
        r->banks.back().grad_bufs = nullptr;
        r->reduced.push_back(reduced[b]);
    }
    // validate every bucket's two calls once
    zero_adam_hparams_t probe = r->hp;
    probe.step = 1;
    for (size_t b = 0; b < r->banks.size(); ++b) {
        using namespace zero::fused;
        const zero_bucket_banks_t& d = r->banks[b];
        StepParams prm{};
        int64_t blocks = 0;
        int rc = prepare_stats(fn, r->grads[b].data(), world, r->numel[b], ZERO_ALL_PARTITIONS, grad_dtype,
                               loss_scale, probe.grad_divisor, r->reduced[b], flag_dev, grad_sqnorm, workspace, &prm,
                               &blocks);
        if (rc == ZERO_OK)
            rc = prepare_reduced(fn, r->reduced[b], r->numel[b], d.master[0], d.m[0], d.v[0], d.master[0], d.m[0],
                                 d.v[0], d.params[0], param_dtype, &probe, &prm, &blocks);
        if (rc) {
            delete r;
            return rc;
        }
    }
    *out = r;
    return zero::ok();
}

extern "C" int zero_runner_launch(zero_runner_t* r, zero_stream_t stream) {
    using namespace zero::fused;
    const char* fn = "zero_runner_launch";
    if (!r) return fail(ZERO_ERR_ARG, "%s: NULL runner", fn);
    if (r->launched) return fail(ZERO_ERR_ARG, "%s: the previous step was not committed", fn);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t flag_bytes = r->staged ? 2 * sizeof(int32_t) : sizeof(int32_t);
    cudaError_t e = cudaMemsetAsync(r->flag_dev, 0, flag_bytes, s);
    if (e == cudaSuccess && r->sqnorm) e = cudaMemsetAsync(r->sqnorm, 0, sizeof(double), s);
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: memset failed: %s", fn, cudaGetErrorString(e));
    zero_adam_hparams_t hp = r->hp;
    hp.step = r->t + 1;
    if (r->staged) {
        for (size_t b = 0; b < r->banks.size(); ++b) {
            StepParams prm{};
            int64_t blocks = 0;
            if (int rc = prepare_stats(fn, r->grads[b].data(), r->world, r->numel[b], ZERO_ALL_PARTITIONS,
                                       r->grad_dtype, r->scale, r->hp.grad_divisor, r->reduced[b], r->flag_dev,
                                       r->sqnorm, r->workspace, &prm, &blocks))
                return rc;
            if (int rc = launch_stats(fn, prm, blocks, r->grad_dtype, r->reduced[b], stream)) return rc;
        }
        for (size_t b = 0; b < r->banks.size(); ++b) {
            const zero_bucket_banks_t& d = r->banks[b];
            StepParams prm{};
            int64_t work = 0;
            if (int rc = prepare_reduced(fn, r->reduced[b], r->numel[b], d.master[0], d.m[0], d.v[0], d.master[0],
                                         d.m[0], d.v[0], d.params[0], r->param_dtype, &hp, &prm, &work))
                return rc;
            prm.overflow = r->flag_dev + 1;
            if (int rc = add_gate_and_clip(fn, &prm, r->flag_dev, r->max_norm > 0.0f ? r->sqnorm : nullptr,
                                           r->max_norm))
                return rc;
            if (work == 0) continue;
            ParamDsts pd{};
            if (int rc = launch_reduced(fn, prm, pd, work, r->param_dtype, false, stream)) return rc;
        }
        e = cudaMemcpyAsync(const_cast<int32_t*>(r->flag_host), r->flag_dev, flag_bytes, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: flag copy failed: %s", fn, cudaGetErrorString(e));
        r->launched = 1;
        return zero::ok();
    }
    const int c = r->cur, n = c ^ 1;
    for (size_t b = 0; b < r->banks.size(); ++b) {
        const zero_bucket_banks_t& d = r->banks[b];
        StepParams prm{};
        int64_t blocks = 0;
        if (int rc = prepare_step(fn, r->grads[b].data(), r->world, r->numel[b], ZERO_ALL_PARTITIONS, r->grad_dtype,
                                  d.master[c], d.m[c], d.v[c], d.master[n], d.m[n], d.v[n], d.params[n],
                                  r->param_dtype, &hp, r->scale, r->flag_dev, r->sqnorm, r->workspace, &prm, &blocks))
            return rc;
        if (int rc = launch_step(fn, prm, blocks, r->grad_dtype, r->param_dtype, stream)) return rc;
    }
    e = cudaMemcpyAsync(const_cast<int32_t*>(r->flag_host), r->flag_dev, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: flag copy failed: %s", fn, cudaGetErrorString(e));
    r->launched = 1;
    return zero::ok();
}

extern "C" int zero_runner_commit(zero_runner_t* r, zero_stream_t stream, int32_t* applied) {
    const char* fn = "zero_runner_commit";
    if (!r || !applied) return fail(ZERO_ERR_ARG, "%s: NULL argument", fn);
    if (!r->launched) return fail(ZERO_ERR_ARG, "%s: no step was launched", fn);
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: stream failed: %s", fn, cudaGetErrorString(e));
    r->launched = 0;
    const int32_t flag = r->staged ? (r->flag_host[0] | r->flag_host[1]) : *r->flag_host;
    if (flag & 2) {
        *applied = 0;
        return fail(ZERO_ERR_CUDA, "%s: a kernel gave up waiting on its copy pipeline; step not committed", fn);
    }
    const int32_t overflow = flag != 0;
    if (!overflow) {
        if (!r->staged) r->cur ^= 1;
        r->t += 1;
    }
    if (int rc = zero_loss_scale_update(&r->scale, &r->good, overflow, r->growth_interval, r->min_scale)) return rc;
    *applied = !overflow;
    return zero::ok();
}

extern "C" int zero_runner_state(const zero_runner_t* r, int64_t* t, float* loss_scale, int32_t* good_steps,
                                 int32_t* bank) {
    if (!r) return fail(ZERO_ERR_ARG, "zero_runner_state: NULL runner");
    if (t) *t = r->t;
    if (loss_scale) *loss_scale = r->scale;
    if (good_steps) *good_steps = r->good;
    if (bank) *bank = r->cur;
    return zero::ok();
}

extern "C" int zero_runner_set_state(zero_runner_t* r, int64_t t, float loss_scale, int32_t good_steps, int32_t bank) {
    if (!r) return fail(ZERO_ERR_ARG, "zero_runner_set_state: NULL runner");
    if (t < 0 || !(loss_scale > 0.0f) || !std::isfinite(loss_scale) || good_steps < 0 || (bank != 0 && bank != 1) ||
        (r->staged && bank != 0))
        return fail(ZERO_ERR_ARG, "zero_runner_set_state: bad value");
    if (r->launched) return fail(ZERO_ERR_ARG, "zero_runner_set_state: a launched step is not committed");
    r->t = t;
    r->scale = loss_scale;
    r->good = good_steps;
    r->cur = bank;
    return zero::ok();
}

extern "C" int zero_runner_bucket_kernel(const zero_runner_t* r, int64_t bucket, int32_t* kind) {
    const char* fn = "zero_runner_bucket_kernel";
    if (!r || !kind) return fail(ZERO_ERR_ARG, "%s: NULL argument", fn);
    if (r->staged) return fail(ZERO_ERR_ARG, "%s: a staged runner has no fused-step kernel", fn);
    if (bucket < 0 || bucket >= static_cast<int64_t>(r->banks.size()))
        return fail(ZERO_ERR_ARG, "%s: bucket %lld outside 0..%lld", fn, (long long)bucket,
                    (long long)r->banks.size() - 1);
    // the same preparation the next launch makes (bank cur -> cur ^ 1)
    const int c = r->cur, n = c ^ 1;
    const zero_bucket_banks_t& d = r->banks[bucket];
    zero_adam_hparams_t hp = r->hp;
    hp.step = r->t + 1;
    zero::fused::StepParams prm{};
    int64_t blocks = 0;
    if (int rc = zero::fused::prepare_step(fn, r->grads[bucket].data(), r->world, r->numel[bucket],
                                           ZERO_ALL_PARTITIONS, r->grad_dtype, d.master[c], d.m[c], d.v[c],
                                           d.master[n], d.m[n], d.v[n], d.params[n], r->param_dtype, &hp, r->scale,
                                           r->flag_dev, r->sqnorm, r->workspace, &prm, &blocks))
        return rc;
    *kind = prm.kind;
    return zero::ok();
}

extern "C" void zero_runner_destroy(zero_runner_t* r) { delete r; }
