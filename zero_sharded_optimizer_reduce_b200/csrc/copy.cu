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
// One kernel, two bodies.  The grid is (blocks per segment) x (segments):
// every segment is copied by its own column of blocks at the same time, each
// thread moving several aligned 32-byte destination blocks per iteration with
// plain 16-byte loads and one 32-byte store per block (no streaming or L1
// no-allocate hints: on B200 they cost 3-17 % in this copy), with a grid of
// several waves.  The store width is what sets the rate of a 1:1 copy: on
// B200, 16-byte stores reach 0.96 of a device-to-device cudaMemcpy and 32-byte
// stores 0.99-1.00, whatever the load width.
//  - source and destination share their 16-byte phase (the usual case: every
//    slice of a Stage-3 unit, every bucket whose partition is a multiple of 8
//    elements): each destination block is two aligned source blocks;
//  - the phases differ (an odd partition size puts every rank but the first
//    off its destination's phase): each thread loads the three aligned
//    source blocks that its destination block straddles (the third is the
//    next thread's first, read again from L1) and realigns them with funnel
//    shifts, so loads and stores stay aligned and coalesced.
// The edges of each segment (before its first 32-byte aligned destination
// byte, after its last whole block) are copied element by element by the
// segment's first block.  A source block read this way always holds at least
// one byte of the segment, so it never reaches a page the segment does not
// touch; bytes outside the segment are never written.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <vector>

#include "common.h"

namespace zero {
namespace copyk {
namespace {

constexpr int kMaxSegs = 64;          // segments per launch
constexpr int kCopyThreads = 256;
constexpr int kBlk = 32;              // bytes per destination block (one 32-byte store)
// Destination blocks per thread per iteration (128 and 64 bytes stored), and
// blocks of the whole grid per SM (several waves), for the phase-matched and
// the realigning body.
constexpr int kKMatched = 4, kKShifted = 2;
constexpr int kBlocksPerSmMatched = 64, kBlocksPerSmShifted = 32;
constexpr int32_t kStatusBounds = 4;  // debug builds: an index check failed, access skipped

// Index check of debug builds (ZERO_DEBUG_BOUNDS): when `ok` is false, record
// kStatusBounds in *status (when given) and return true so that the caller
// skips the access.  In release builds it is the constant false.
__device__ __forceinline__ bool out_of_bounds(bool ok, int32_t* status) {
#ifdef ZERO_DEBUG_BOUNDS
    if (!ok) {
        if (status) atomicOr(status, kStatusBounds);
        return true;
    }
#endif
    (void)ok;
    (void)status;
    (void)kStatusBounds;
    return false;
}

struct CopySeg {
    const char* src;      // first source byte
    char* dst;            // first destination byte
    const char* src_al;   // aligned source block holding the byte copied to dst + head
    int64_t bytes;        // segment length
    int64_t head;         // bytes before the first 32-byte aligned destination byte
    int64_t nblk;         // whole aligned 32-byte destination blocks after the head
    int32_t shift;        // (src + head) - src_al; 0 when the 16-byte phases agree
};

struct CopyParams {
    CopySeg seg[kMaxSegs];
    int32_t esize;        // 2 or 4
    int32_t* status;      // debug-build bounds reports; may be NULL
};

__device__ __forceinline__ uint4 ld16(const char* p) { return *reinterpret_cast<const uint4*>(p); }

// One 32-byte store (a 32-byte aligned address): lo then hi.
__device__ __forceinline__ void st32(char* p, const uint4& lo, const uint4& hi) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(lo.x), "r"(lo.y), "r"(lo.z),
                 "r"(lo.w), "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
                 : "memory");
}

// Bytes [4Q + sh/8, 4Q + sh/8 + 16) of the 32-byte concatenation a:b.
template <int Q>
__device__ __forceinline__ uint4 realign(const uint4& a, const uint4& b, uint32_t sh) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    return make_uint4(__funnelshift_r(w[Q], w[Q + 1], sh), __funnelshift_r(w[Q + 1], w[Q + 2], sh),
                      __funnelshift_r(w[Q + 2], w[Q + 3], sh), __funnelshift_r(w[Q + 3], w[Q + 4], sh));
}

// Bytes [shift, shift + 16) of a:b (shift uniform over the segment).
__device__ __forceinline__ uint4 realign_rt(const uint4& a, const uint4& b, int shift) {
    const uint32_t sh = static_cast<uint32_t>(shift & 3) * 8u;
    switch (shift >> 2) {
        case 0: return realign<0>(a, b, sh);
        case 1: return realign<1>(a, b, sh);
        case 2: return realign<2>(a, b, sh);
        default: return realign<3>(a, b, sh);
    }
}

// True when the aligned source block at `a` holds a byte of the segment.
__device__ __forceinline__ bool src_block_ok(const CopySeg& sg, const char* a) {
    return a < sg.src + sg.bytes && a + 16 > sg.src;
}

__device__ __forceinline__ void copy_elem(const CopySeg& sg, int64_t off, int es, int32_t* status) {
    if (out_of_bounds(off >= 0 && off + es <= sg.bytes, status)) return;
    if (es == 2) *reinterpret_cast<uint16_t*>(sg.dst + off) = *reinterpret_cast<const uint16_t*>(sg.src + off);
    else *reinterpret_cast<uint32_t*>(sg.dst + off) = *reinterpret_cast<const uint32_t*>(sg.src + off);
}

// Segment blockIdx.y takes the phase-matched or the realigning body by its
// shift (uniform over the segment's blocks).
__global__ void __launch_bounds__(kCopyThreads) copy_grid_kernel(const __grid_constant__ CopyParams p) {
    const CopySeg& sg = p.seg[blockIdx.y];
    const int es = p.esize;
    if (blockIdx.x == 0) {
        for (int64_t i = threadIdx.x; i < sg.head / es; i += kCopyThreads) copy_elem(sg, i * es, es, p.status);
        const int64_t tail0 = sg.head + kBlk * sg.nblk;
        for (int64_t i = threadIdx.x; i < (sg.bytes - tail0) / es; i += kCopyThreads)
            copy_elem(sg, tail0 + i * es, es, p.status);
    }
    char* const dst_al = sg.dst + sg.head;
    const int64_t n = sg.nblk;
    const int64_t nt = static_cast<int64_t>(gridDim.x) * kCopyThreads;
    const int64_t body = sg.bytes - sg.head;   // bytes from the first aligned destination byte
    int64_t i = static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x;
    if (sg.shift == 0) {
        constexpr int kCopyK = kKMatched;
        for (; i + (kCopyK - 1) * nt < n; i += kCopyK * nt) {
            uint4 r[kCopyK][2];
#pragma unroll
            for (int k = 0; k < kCopyK; ++k) {
                const char* s0 = sg.src_al + kBlk * (i + k * nt);
                r[k][0] = ld16(s0);
                r[k][1] = ld16(s0 + 16);
            }
#pragma unroll
            for (int k = 0; k < kCopyK; ++k) {
                if (out_of_bounds(kBlk * (i + k * nt) + kBlk <= body, p.status)) continue;
                st32(dst_al + kBlk * (i + k * nt), r[k][0], r[k][1]);
            }
        }
        for (; i < n; i += nt) {
            if (out_of_bounds(kBlk * i + kBlk <= body, p.status)) continue;
            const char* s0 = sg.src_al + kBlk * i;
            st32(dst_al + kBlk * i, ld16(s0), ld16(s0 + 16));
        }
    } else {
        // destination block j straddles source blocks 2j, 2j + 1 and 2j + 2;
        // the last one needed, 2n, still holds segment bytes (shift > 0)
        constexpr int kCopyK = kKShifted;
        const int shift = sg.shift;
        for (; i + (kCopyK - 1) * nt < n; i += kCopyK * nt) {
            uint4 a[kCopyK], b[kCopyK], c[kCopyK];
#pragma unroll
            for (int k = 0; k < kCopyK; ++k) {
                const char* s0 = sg.src_al + kBlk * (i + k * nt);
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                a[k] = out_of_bounds(src_block_ok(sg, s0), p.status) ? z : ld16(s0);
                b[k] = out_of_bounds(src_block_ok(sg, s0 + 16), p.status) ? z : ld16(s0 + 16);
                c[k] = out_of_bounds(src_block_ok(sg, s0 + 32), p.status) ? z : ld16(s0 + 32);
            }
#pragma unroll
            for (int k = 0; k < kCopyK; ++k) {
                if (out_of_bounds(kBlk * (i + k * nt) + kBlk <= body, p.status)) continue;
                st32(dst_al + kBlk * (i + k * nt), realign_rt(a[k], b[k], shift), realign_rt(b[k], c[k], shift));
            }
        }
        for (; i < n; i += nt) {
            const char* s0 = sg.src_al + kBlk * i;
            if (out_of_bounds(src_block_ok(sg, s0) && src_block_ok(sg, s0 + 16) && src_block_ok(sg, s0 + 32) &&
                                  kBlk * i + kBlk <= body,
                              p.status))
                continue;
            const uint4 b = ld16(s0 + 16);
            st32(dst_al + kBlk * i, realign_rt(ld16(s0), b, shift), realign_rt(b, ld16(s0 + 32), shift));
        }
    }
}

// ------------------------------------------------------------------ host side

struct Seg {
    const char* src;
    char* dst;
    int64_t bytes;
};

std::mutex g_mu;
int g_sms[64] = {};

int device_sms(const char* fn, int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return fail(ZERO_ERR_CUDA, "%s: cannot query the device", fn);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sms[dev] == 0 && cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        g_sms[dev] = 0;
        return fail(ZERO_ERR_CUDA, "%s: cannot query the SM count", fn);
    }
    *sms = g_sms[dev];
    return ZERO_OK;
}

// Host-side description of one segment.
CopySeg make_seg(const Seg& g) {
    CopySeg r{};
    r.src = g.src;
    r.dst = g.dst;
    r.bytes = g.bytes;
    r.head = static_cast<int64_t>((32u - (reinterpret_cast<uintptr_t>(g.dst) & 31u)) & 31u);
    if (r.head > g.bytes) r.head = g.bytes;
    r.nblk = (g.bytes - r.head) / kBlk;
    const uintptr_t a = reinterpret_cast<uintptr_t>(g.src + r.head);
    r.src_al = reinterpret_cast<const char*>(a & ~static_cast<uintptr_t>(15));
    r.shift = r.nblk > 0 ? static_cast<int32_t>(a & 15u) : 0;
    return r;
}

// Enqueue copy_grid_kernel over `segs`, at most kMaxSegs per launch: one
// launch copies phase-matched and realigned segments side by side.
int launch_copy(const std::vector<Seg>& segs, int esize, int32_t* status, cudaStream_t stream, const char* fn) {
    int sms = 0;
    if (int rc = device_sms(fn, &sms)) return rc;
    std::vector<CopySeg> all;
    for (const Seg& g : segs)
        if (g.bytes > 0) all.push_back(make_seg(g));
    for (size_t first = 0; first < all.size(); first += kMaxSegs) {
        const size_t n = std::min<size_t>(kMaxSegs, all.size() - first);
        CopyParams prm{};
        prm.esize = esize;
        prm.status = status;
        int64_t want = 1;
        bool shifted = false;
        for (size_t i = 0; i < n; ++i) {
            prm.seg[i] = all[first + i];
            const int64_t per_block = int64_t(kCopyThreads) * (prm.seg[i].shift ? kKShifted : kKMatched);
            want = std::max(want, (prm.seg[i].nblk + per_block - 1) / per_block);
            shifted = shifted || prm.seg[i].shift != 0;
        }
        // a grid of several waves over all segments, no more blocks per
        // segment than its largest body can use
        const int64_t cap = std::max<int64_t>(
            1, int64_t(sms) * (shifted ? kBlocksPerSmShifted : kBlocksPerSmMatched) / int64_t(n));
        const unsigned int gx = static_cast<unsigned int>(std::max<int64_t>(1, std::min(want, cap)));
        copy_grid_kernel<<<dim3(gx, static_cast<unsigned int>(n)), kCopyThreads, 0, stream>>>(prm);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    }
    return ZERO_OK;
}

}  // namespace
}  // namespace copyk
}  // namespace zero

using zero::fail;

extern "C" int zero_flatten_bucket(const zero_layout_t* L, int64_t bucket, const void* const* tensor_ptrs,
                                   zero_dtype_t dtype, void* bucket_buf, zero_stream_t stream) {
    using namespace zero;
    using namespace zero::copyk;
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
    if (!segs.empty())
        if (int rc = launch_copy(segs, es, nullptr, s, fn)) return rc;
    const int64_t pad = L->bucket_padded[bucket] - L->bucket_numel[bucket];
    if (pad > 0) {
        cudaError_t e = cudaMemsetAsync(static_cast<char*>(bucket_buf) + L->bucket_numel[bucket] * es, 0,
                                        static_cast<size_t>(pad * es), s);
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: padding memset failed: %s", fn, cudaGetErrorString(e));
    }
    return ok();
}

extern "C" int zero_allgather_params(const void* const* shards, int32_t world, int64_t shard_offset,
                                     int64_t part_numel, zero_dtype_t dtype, void* dst, int32_t* status,
                                     zero_stream_t stream) {
    using namespace zero;
    using namespace zero::copyk;
    const char* fn = "zero_allgather_params";
    if (!shards || !dst) return fail(ZERO_ERR_ARG, "%s: NULL argument", fn);
    if (world < 1 || world > ZERO_MAX_WORLD) return fail(ZERO_ERR_ARG, "%s: world %d outside 1..%d", fn, world, ZERO_MAX_WORLD);
    if (shard_offset < 0 || part_numel < 0) return fail(ZERO_ERR_ARG, "%s: negative offset or size", fn);
    const int es = dtype_size(dtype);
    if (es == 0) return fail(ZERO_ERR_DTYPE, "%s: unsupported dtype %d", fn, static_cast<int>(dtype));
    if (!aligned(dst, es)) return fail(ZERO_ERR_ALIGN, "%s: dst misaligned", fn);
    if (status && !aligned(status, 4)) return fail(ZERO_ERR_ALIGN, "%s: status misaligned", fn);
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
    if (status && overlaps(status, 4, dst, dst_bytes)) return fail(ZERO_ERR_ARG, "%s: status overlaps dst", fn);
    if (int rc = launch_copy(segs, es, status, reinterpret_cast<cudaStream_t>(stream), fn)) return rc;
    return ok();
}
