// Bit-exact segment copies for sm_100a: flattening a tensor list into a
// constant-size fused buffer, and the all-gather that rebuilds full
// parameters from N rank shards.
//
// Method: ZeRO explainer (azimuth.plus), "Constant-size buffers" (small
// tensors fused into one buffer of fixed size), and "Stage 3 - Parameter
// Partitioning (P_os+g+p)" (a layer's parameters are rebuilt on the fly by
// all-gather from the ranks owning its slices).  On one GPU both are
// HBM-bound copies: each byte is read once and written once.
//
// One launch copies up to kMaxSegs segments; blockIdx.y selects the segment,
// the x-blocks stride over it.  When source and destination share their
// 16-byte phase the body moves 16 bytes per access (head and tail per
// element); otherwise every element is copied on its own.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <vector>

#include "common.h"

namespace zero {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxSegs = 64;
constexpr int kUnroll = 4;

struct Seg {
    const char* src;
    char* dst;
    int64_t bytes;
};

struct CopyParams {
    Seg seg[kMaxSegs];
    int32_t esize;  // 2 or 4
};

template <typename E>
__device__ __forceinline__ void copy_elems(const char* src, char* dst, int64_t n, int64_t t, int64_t nt) {
    const E* s = reinterpret_cast<const E*>(src);
    E* d = reinterpret_cast<E*>(dst);
    for (int64_t i = t; i < n; i += nt) d[i] = s[i];
}

__global__ void __launch_bounds__(kThreads) copy_segments_kernel(const __grid_constant__ CopyParams p) {
    const Seg sg = p.seg[blockIdx.y];
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    const int64_t nt = static_cast<int64_t>(gridDim.x) * kThreads;
    const uintptr_t sa = reinterpret_cast<uintptr_t>(sg.src), da = reinterpret_cast<uintptr_t>(sg.dst);
    const int es = p.esize;
    if (((sa ^ da) & 15u) != 0) {
        if (es == 2) copy_elems<uint16_t>(sg.src, sg.dst, sg.bytes / 2, t, nt);
        else copy_elems<uint32_t>(sg.src, sg.dst, sg.bytes / 4, t, nt);
        return;
    }
    int64_t head = static_cast<int64_t>((16u - (sa & 15u)) & 15u);
    if (head > sg.bytes) head = sg.bytes;
    const int64_t nvec = (sg.bytes - head) / 16;
    const int64_t tail0 = head + nvec * 16;
    // head and tail, element by element
    const int64_t nhead = head / es, ntail = (sg.bytes - tail0) / es;
    for (int64_t i = t; i < nhead + ntail; i += nt) {
        const int64_t off = i < nhead ? i * es : tail0 + (i - nhead) * es;
        if (es == 2) *reinterpret_cast<uint16_t*>(sg.dst + off) = *reinterpret_cast<const uint16_t*>(sg.src + off);
        else *reinterpret_cast<uint32_t*>(sg.dst + off) = *reinterpret_cast<const uint32_t*>(sg.src + off);
    }
    // body, 16 bytes per access, kUnroll accesses in flight per thread
    const uint4* s4 = reinterpret_cast<const uint4*>(sg.src + head);
    uint4* d4 = reinterpret_cast<uint4*>(sg.dst + head);
    int64_t i = t;
    for (; i + (kUnroll - 1) * nt < nvec; i += kUnroll * nt) {
        uint4 r[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) r[u] = __ldcs(s4 + i + u * nt);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) __stcs(d4 + i + u * nt, r[u]);
    }
    for (; i < nvec; i += nt) __stcs(d4 + i, __ldcs(s4 + i));
}

std::mutex g_sms_mu;
int g_sms[64] = {};

// SM count of the current device, queried once per device.
int device_sms(const char* fn, int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return fail(ZERO_ERR_CUDA, "%s: cannot query the device", fn);
    std::lock_guard<std::mutex> lk(g_sms_mu);
    if (g_sms[dev] == 0 && cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return fail(ZERO_ERR_CUDA, "%s: cannot query the SM count", fn);
    *sms = g_sms[dev];
    return ZERO_OK;
}

int launch_segments(const std::vector<Seg>& segs, int esize, cudaStream_t stream, const char* fn) {
    int sms = 0;
    if (int rc = device_sms(fn, &sms)) return rc;
    for (size_t first = 0; first < segs.size(); first += kMaxSegs) {
        const size_t n = std::min<size_t>(kMaxSegs, segs.size() - first);
        CopyParams prm{};
        prm.esize = esize;
        int64_t max_bytes = 0;
        for (size_t i = 0; i < n; ++i) {
            prm.seg[i] = segs[first + i];
            max_bytes = std::max(max_bytes, segs[first + i].bytes);
        }
        if (max_bytes == 0) continue;
        // enough blocks to cover the largest segment with kUnroll 16-byte
        // accesses per thread, at most 16 blocks per SM in total (measured on
        // B200, all-gather of 8 x 25M fp16 elements: 5.96 TB/s; with 8 per
        // SM 5.78; 8-deep unrolling or non-streaming loads and stores were
        // not faster)
        int64_t want = (max_bytes + int64_t(kThreads) * 16 * kUnroll - 1) / (int64_t(kThreads) * 16 * kUnroll);
        int64_t cap = std::max<int64_t>(1, int64_t(sms) * 16 / int64_t(n));
        const unsigned int gx = static_cast<unsigned int>(std::max<int64_t>(1, std::min(want, cap)));
        copy_segments_kernel<<<dim3(gx, static_cast<unsigned int>(n)), kThreads, 0, stream>>>(prm);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    }
    return ZERO_OK;
}

}  // namespace
}  // namespace zero

using zero::fail;

extern "C" int zero_flatten_bucket(const zero_layout_t* L, int64_t bucket, const void* const* tensor_ptrs,
                                   zero_dtype_t dtype, void* bucket_buf, zero_stream_t stream) {
    using namespace zero;
    const char* fn = "zero_flatten_bucket";
    if (!L || !tensor_ptrs || !bucket_buf) return fail(ZERO_ERR_ARG, "%s: NULL argument", fn);
    if (!L->bucket_numel || !L->tensor_offset || !L->tensor_numel)
        return fail(ZERO_ERR_ARG, "%s: layout not filled", fn);
    if (bucket < 0 || bucket >= L->n_buckets)
        return fail(ZERO_ERR_RANGE, "%s: bucket %lld outside 0..%lld", fn, (long long)bucket, (long long)L->n_buckets - 1);
    const int es = dtype_size(dtype);
    if (es == 0) return fail(ZERO_ERR_DTYPE, "%s: unsupported dtype %d", fn, static_cast<int>(dtype));
    if (!aligned(bucket_buf, es)) return fail(ZERO_ERR_ALIGN, "%s: bucket_buf misaligned", fn);
    const int64_t first = L->bucket_first[bucket], cnt = L->bucket_count[bucket];
    const int64_t padded_bytes = L->bucket_padded[bucket] * es;
    std::vector<Seg> segs;
    segs.reserve(static_cast<size_t>(cnt));
    for (int64_t i = first; i < first + cnt; ++i) {
        const int64_t n = L->tensor_numel[i];
        if (n == 0) continue;
        if (!tensor_ptrs[i]) return fail(ZERO_ERR_ARG, "%s: tensor_ptrs[%lld] is NULL", fn, (long long)i);
        if (!aligned(tensor_ptrs[i], es)) return fail(ZERO_ERR_ALIGN, "%s: tensor %lld misaligned", fn, (long long)i);
        if (overlaps(tensor_ptrs[i], n * es, bucket_buf, padded_bytes))
            return fail(ZERO_ERR_ARG, "%s: tensor %lld overlaps the bucket buffer", fn, (long long)i);
        segs.push_back(Seg{static_cast<const char*>(tensor_ptrs[i]),
                           static_cast<char*>(bucket_buf) + L->tensor_offset[i] * es, n * es});
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (int rc = launch_segments(segs, es, s, fn)) return rc;
    const int64_t pad = L->bucket_padded[bucket] - L->bucket_numel[bucket];
    if (pad > 0) {
        cudaError_t e = cudaMemsetAsync(static_cast<char*>(bucket_buf) + L->bucket_numel[bucket] * es, 0,
                                        static_cast<size_t>(pad * es), s);
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: padding memset failed: %s", fn, cudaGetErrorString(e));
    }
    return ok();
}

extern "C" int zero_allgather_params(const void* const* shards, int32_t world, int64_t shard_offset,
                                     int64_t part_numel, zero_dtype_t dtype, void* dst, zero_stream_t stream) {
    using namespace zero;
    const char* fn = "zero_allgather_params";
    if (!shards || !dst) return fail(ZERO_ERR_ARG, "%s: NULL argument", fn);
    if (world < 1 || world > ZERO_MAX_WORLD) return fail(ZERO_ERR_ARG, "%s: world %d outside 1..%d", fn, world, ZERO_MAX_WORLD);
    if (shard_offset < 0 || part_numel < 0) return fail(ZERO_ERR_ARG, "%s: negative offset or size", fn);
    const int es = dtype_size(dtype);
    if (es == 0) return fail(ZERO_ERR_DTYPE, "%s: unsupported dtype %d", fn, static_cast<int>(dtype));
    if (!aligned(dst, es)) return fail(ZERO_ERR_ALIGN, "%s: dst misaligned", fn);
    if (part_numel == 0) return ok();
    const int64_t dst_bytes = static_cast<int64_t>(world) * part_numel * es;
    std::vector<Seg> segs;
    for (int r = 0; r < world; ++r) {
        if (!shards[r]) return fail(ZERO_ERR_ARG, "%s: shards[%d] is NULL", fn, r);
        if (!aligned(shards[r], es)) return fail(ZERO_ERR_ALIGN, "%s: shards[%d] misaligned", fn, r);
        const char* src = static_cast<const char*>(shards[r]) + shard_offset * es;
        if (overlaps(src, part_numel * es, dst, dst_bytes))
            return fail(ZERO_ERR_ARG, "%s: shards[%d] overlaps dst", fn, r);
        segs.push_back(Seg{src, static_cast<char*>(dst) + static_cast<int64_t>(r) * part_numel * es, part_numel * es});
    }
    if (int rc = launch_segments(segs, es, reinterpret_cast<cudaStream_t>(stream), fn)) return rc;
    return ok();
}
