// Host-only parts of the libzero C ABI: partition layout of constant-size
// buffers, the dynamic loss-scale rule, and error strings.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "common.h"

namespace zero {

static thread_local char g_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_last_error[0] = '\0';
    return ZERO_OK;
}

static std::atomic<int> g_step_kernel_override{-1};

int step_kernel_override() { return g_step_kernel_override.load(std::memory_order_relaxed); }

}  // namespace zero

using zero::fail;

extern "C" {

const char* zero_last_error(void) { return zero::g_last_error; }

int zero_test_force_step_kernel(int32_t kind) {
    if (kind < -1 || kind > 3) return fail(ZERO_ERR_ARG, "zero_test_force_step_kernel: kind %d outside -1..3", kind);
    zero::g_step_kernel_override.store(kind, std::memory_order_relaxed);
    return zero::ok();
}

const char* zero_strerror(int code) {
    switch (code) {
        case ZERO_OK: return "ok";
        case ZERO_ERR_ARG: return "invalid argument";
        case ZERO_ERR_ALIGN: return "misaligned pointer";
        case ZERO_ERR_DTYPE: return "unsupported dtype";
        case ZERO_ERR_RANGE: return "index out of range";
        case ZERO_ERR_CUDA: return "CUDA error";
        case ZERO_ERR_NOMEM: return "host allocation failed";
        default: return "unknown error";
    }
}

const char* zero_version(void) { return "zero-step 0.1 (sm_100a)"; }

void zero_layout_free(zero_layout_t* L) {
    if (!L) return;
    int64_t** arrays[] = {&L->bucket_numel, &L->bucket_padded, &L->bucket_offset, &L->bucket_first,
                          &L->bucket_count, &L->tensor_numel, &L->tensor_bucket, &L->tensor_offset};
    for (int64_t** a : arrays) {
        std::free(*a);
        *a = nullptr;
    }
    L->n_buckets = 0;
    L->n_tensors = 0;
}

// Greedy packing in list order into buckets of capacity bucket_elems (ZeRO
// explainer, "Constant-size buffers"), each padded to a multiple of
// world*align_elems so that it splits into `world` equal partitions (Stage 1:
// each GPU holds 1/N of the states).
int zero_partition_layout(const int64_t* numels, int64_t n_tensors, int32_t world,
                          int64_t bucket_elems, int32_t align_elems, zero_layout_t* out) {
    if (!out) return fail(ZERO_ERR_ARG, "zero_partition_layout: out is NULL");
    if (n_tensors < 0 || (n_tensors > 0 && !numels))
        return fail(ZERO_ERR_ARG, "zero_partition_layout: bad tensor list");
    if (world < 1 || world > ZERO_MAX_WORLD)
        return fail(ZERO_ERR_ARG, "zero_partition_layout: world %d outside 1..%d", world, ZERO_MAX_WORLD);
    if (bucket_elems < 0 || align_elems < 1)
        return fail(ZERO_ERR_ARG, "zero_partition_layout: bucket_elems >= 0 and align_elems >= 1 required");
    for (int64_t i = 0; i < n_tensors; ++i)
        if (numels[i] < 0) return fail(ZERO_ERR_ARG, "zero_partition_layout: tensor %lld has negative size",
                                       (long long)i);

    // first pass: bucket boundaries
    std::vector<int64_t> first, count, numel;
    int64_t cur_n = 0, cur_first = 0, cur_count = 0;
    for (int64_t i = 0; i < n_tensors; ++i) {
        if (cur_count > 0 && bucket_elems > 0 && cur_n + numels[i] > bucket_elems) {
            first.push_back(cur_first);
            count.push_back(cur_count);
            numel.push_back(cur_n);
            cur_first = i;
            cur_count = 0;
            cur_n = 0;
        }
        cur_n += numels[i];
        ++cur_count;
    }
    if (cur_count > 0) {
        first.push_back(cur_first);
        count.push_back(cur_count);
        numel.push_back(cur_n);
    }
    const int64_t nb = static_cast<int64_t>(first.size());

    zero_layout_t L{};
    L.world = world;
    L.align_elems = align_elems;
    L.n_tensors = n_tensors;
    L.n_buckets = nb;
    auto alloc = [](int64_t n) { return static_cast<int64_t*>(std::calloc(n > 0 ? n : 1, sizeof(int64_t))); };
    L.bucket_numel = alloc(nb);
    L.bucket_padded = alloc(nb);
    L.bucket_offset = alloc(nb);
    L.bucket_first = alloc(nb);
    L.bucket_count = alloc(nb);
    L.tensor_numel = alloc(n_tensors);
    L.tensor_bucket = alloc(n_tensors);
    L.tensor_offset = alloc(n_tensors);
    if (!L.bucket_numel || !L.bucket_padded || !L.bucket_offset || !L.bucket_first || !L.bucket_count ||
        !L.tensor_numel || !L.tensor_bucket || !L.tensor_offset) {
        zero_layout_free(&L);
        return fail(ZERO_ERR_NOMEM, "zero_partition_layout: out of host memory");
    }
    const int64_t unit = static_cast<int64_t>(world) * align_elems;
    int64_t flat = 0;
    for (int64_t b = 0; b < nb; ++b) {
        L.bucket_numel[b] = numel[b];
        L.bucket_padded[b] = (numel[b] + unit - 1) / unit * unit;
        L.bucket_offset[b] = flat;
        L.bucket_first[b] = first[b];
        L.bucket_count[b] = count[b];
        flat += L.bucket_padded[b];
        int64_t off = 0;
        for (int64_t i = first[b]; i < first[b] + count[b]; ++i) {
            L.tensor_numel[i] = numels[i];
            L.tensor_bucket[i] = b;
            L.tensor_offset[i] = off;
            off += numels[i];
        }
    }
    *out = L;
    return zero::ok();
}

// Dynamic loss scaling: halve on overflow (floor min_scale), double after
// growth_interval consecutive good steps.
int zero_loss_scale_update(float* scale, int32_t* good_steps, int32_t overflow,
                           int32_t growth_interval, float min_scale) {
    if (!scale || !good_steps) return fail(ZERO_ERR_ARG, "zero_loss_scale_update: NULL pointer");
    if (growth_interval < 1) return fail(ZERO_ERR_ARG, "zero_loss_scale_update: growth_interval < 1");
    if (!(*scale > 0.0f) || !std::isfinite(*scale) || !(min_scale > 0.0f))
        return fail(ZERO_ERR_ARG, "zero_loss_scale_update: scales must be positive and finite");
    if (overflow) {
        float half = *scale * 0.5f;
        *scale = half < min_scale ? min_scale : half;
        *good_steps = 0;
    } else if (++*good_steps >= growth_interval) {
        const float twice = *scale * 2.0f;
        if (std::isfinite(twice)) *scale = twice;   // the scale never grows to inf
        *good_steps = 0;
    }
    return zero::ok();
}

}  // extern "C"
