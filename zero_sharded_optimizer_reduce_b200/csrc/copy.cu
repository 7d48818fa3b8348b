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
// Two kernels:
//  - copy_bulk_kernel (all-gather bodies whose source and destination share
//    their 16-byte phase and are both this GPU's memory): one CTA per SM, one
//    thread drives a ring of shared-memory stages with 1-D bulk copies, global
//    -> shared completing on an mbarrier, shared -> global in bulk groups, so
//    that about 7 stages of loads are in flight per SM without any register
//    traffic.  The bytes of all such bodies are split evenly over the CTAs.
//  - copy_reg_kernel (everything else: flatten, bodies whose phases differ,
//    sources or destinations in another GPU's memory, the sub-16-byte edges):
//    each warp task moves 32 x kRegK aligned 16-byte destination blocks.
//    When the phases differ, every lane loads the aligned source block that
//    holds the start of its destination block, takes the following one from
//    its neighbour lane (one extra load for the last lane), and realigns the
//    pair with funnel shifts, so loads and stores both stay 16-byte and
//    coalesced whatever the offsets.
// A source block read this way always holds at least one byte of the
// segment, so it never reaches a page the segment does not touch; bytes
// outside the segment are never written anywhere.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <vector>

#include "bulk.cuh"
#include "common.h"

namespace zero {
namespace copyk {
namespace {

using fused::bulk_commit;
using fused::bulk_load;
using fused::bulk_store;
using fused::bulk_wait_all;
using fused::bulk_wait_read;
using fused::fence_proxy_async_smem;
using fused::mbar_arrive_expect_tx;
using fused::mbar_init;
using fused::mbar_wait_bounded;

constexpr int kMaxSegs = 64;                   // segments per launch
constexpr int kRegThreads = 256;
constexpr int kRegK = 4;                       // destination blocks per lane per task
constexpr int64_t kTaskBlocks = 32 * kRegK;    // 16-byte blocks per warp task (2 KB)
constexpr int kBulkStages = 8;
constexpr uint32_t kBulkChunk = 24u * 1024u;   // bytes per stage
constexpr uint32_t kBulkSmem = kBulkStages * kBulkChunk;
constexpr int32_t kStatusTimeout = 2;          // a bounded wait gave up: the copy is incomplete
constexpr int32_t kStatusBounds = 4;           // debug builds: an index check failed, access skipped

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
    return false;
}

// ----------------------------------------------------------- register path

struct RegSeg {
    const char* src;      // first source byte
    char* dst;            // first destination byte
    const char* src_al;   // aligned source block holding the byte copied to dst + head
    int64_t bytes;        // segment length
    int64_t head;         // bytes before the first 16-byte aligned destination byte
    int64_t nblk;         // whole aligned 16-byte destination blocks after the head
    int64_t task0;        // first warp task of this segment
    int32_t shift;        // (src + head) - src_al; 0 when the 16-byte phases agree
};

struct RegParams {
    RegSeg seg[kMaxSegs];
    int32_t nseg;
    int32_t esize;        // 2 or 4
    int64_t ntasks;
    int32_t* status;      // debug-build bounds reports; may be NULL
};

__device__ __forceinline__ uint4 ld16(const char* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void st16(char* p, uint4 v) { __stcs(reinterpret_cast<uint4*>(p), v); }

// Bytes [4Q + sh/8, 4Q + sh/8 + 16) of the 32-byte concatenation a:b.
template <int Q>
__device__ __forceinline__ uint4 realign(const uint4& a, const uint4& b, uint32_t sh) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    return make_uint4(__funnelshift_r(w[Q], w[Q + 1], sh), __funnelshift_r(w[Q + 1], w[Q + 2], sh),
                      __funnelshift_r(w[Q + 2], w[Q + 3], sh), __funnelshift_r(w[Q + 3], w[Q + 4], sh));
}

// Bytes [shift, shift + 16) of a:b (shift uniform over the warp).
__device__ __forceinline__ uint4 realign_rt(const uint4& a, const uint4& b, int shift) {
    const uint32_t sh = static_cast<uint32_t>(shift & 3) * 8u;
    switch (shift >> 2) {
        case 0: return realign<0>(a, b, sh);
        case 1: return realign<1>(a, b, sh);
        case 2: return realign<2>(a, b, sh);
        default: return realign<3>(a, b, sh);
    }
}

__device__ __forceinline__ uint4 shfl_down16(const uint4& v) {
    return make_uint4(__shfl_down_sync(0xffffffffu, v.x, 1), __shfl_down_sync(0xffffffffu, v.y, 1),
                      __shfl_down_sync(0xffffffffu, v.z, 1), __shfl_down_sync(0xffffffffu, v.w, 1));
}

__device__ __forceinline__ void copy_elem(const RegSeg& sg, int64_t off, int es, int32_t* status) {
    if (out_of_bounds(off >= 0 && off + es <= sg.bytes, status)) return;
    if (es == 2) *reinterpret_cast<uint16_t*>(sg.dst + off) = *reinterpret_cast<const uint16_t*>(sg.src + off);
    else *reinterpret_cast<uint32_t*>(sg.dst + off) = *reinterpret_cast<const uint32_t*>(sg.src + off);
}

// True when the aligned source block at `a` holds a byte of the segment.
__device__ __forceinline__ bool src_block_ok(const RegSeg& sg, const char* a) {
    return a < sg.src + sg.bytes && a + 16 > sg.src;
}

// kShift: every segment of the launch has shift != 0 (or no whole block);
// otherwise every segment has shift == 0.
template <bool kShift>
__global__ void __launch_bounds__(kRegThreads) copy_reg_kernel(const __grid_constant__ RegParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kRegThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kRegThreads) >> 5;
    const int es = p.esize;
    int s = 0;
    for (int64_t t = warp; t < p.ntasks; t += nwarps) {
        // tasks are visited in increasing order, so the segment index only grows
        while (s + 1 < p.nseg && p.seg[s + 1].task0 <= t) ++s;
        const RegSeg& sg = p.seg[s];
        const int64_t lt = t - sg.task0;
        const int64_t seg_tasks = (s + 1 < p.nseg ? p.seg[s + 1].task0 : p.ntasks) - sg.task0;
        // the edges, element by element: head with the first task, tail with the last
        if (lt == 0)
            for (int64_t i = lane; i < sg.head / es; i += 32) copy_elem(sg, i * es, es, p.status);
        if (lt == seg_tasks - 1) {
            const int64_t tail0 = sg.head + 16 * sg.nblk;
            for (int64_t i = lane; i < (sg.bytes - tail0) / es; i += 32) copy_elem(sg, tail0 + i * es, es, p.status);
        }
        const int64_t b0 = lt * kTaskBlocks;
        char* const dst_al = sg.dst + sg.head;
        if constexpr (!kShift) {
            uint4 v[kRegK];
#pragma unroll
            for (int k = 0; k < kRegK; ++k) {
                const int64_t j = b0 + lane + 32 * k;
                if (j < sg.nblk && !out_of_bounds(src_block_ok(sg, sg.src_al + 16 * j), p.status))
                    v[k] = ld16(sg.src_al + 16 * j);
            }
#pragma unroll
            for (int k = 0; k < kRegK; ++k) {
                const int64_t j = b0 + lane + 32 * k;
                if (j < sg.nblk && !out_of_bounds(16 * j + 16 <= sg.bytes - sg.head, p.status))
                    st16(dst_al + 16 * j, v[k]);
            }
        } else {
            // destination block j takes source blocks j and j + 1 (nblk >= 1 here:
            // the last one needed is block nblk, which still holds segment bytes);
            // block j + 1 comes from the next lane, for the last lane from lane 0's
            // next block, and after the task's last block from one extra load
            const int64_t lim = sg.nblk > 0 ? sg.nblk + 1 : 0;
            uint4 c[kRegK];
            uint4 e = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int k = 0; k < kRegK; ++k) {
                const int64_t j = b0 + lane + 32 * k;
                c[k] = make_uint4(0u, 0u, 0u, 0u);
                if (j < lim && !out_of_bounds(src_block_ok(sg, sg.src_al + 16 * j), p.status))
                    c[k] = ld16(sg.src_al + 16 * j);
            }
            {
                const int64_t j = b0 + kTaskBlocks;
                if (lane == 31 && j < lim && !out_of_bounds(src_block_ok(sg, sg.src_al + 16 * j), p.status))
                    e = ld16(sg.src_al + 16 * j);
            }
#pragma unroll
            for (int k = 0; k < kRegK; ++k) {
                const int64_t j = b0 + lane + 32 * k;
                uint4 nx = shfl_down16(c[k]);
                const uint4 first_next = k + 1 < kRegK ? c[k + 1] : e;
                const uint4 from0 = make_uint4(__shfl_sync(0xffffffffu, first_next.x, 0), __shfl_sync(0xffffffffu, first_next.y, 0),
                                               __shfl_sync(0xffffffffu, first_next.z, 0), __shfl_sync(0xffffffffu, first_next.w, 0));
                if (lane == 31) nx = k + 1 < kRegK ? from0 : e;
                if (j < sg.nblk && !out_of_bounds(16 * j + 16 <= sg.bytes - sg.head, p.status))
                    st16(dst_al + 16 * j, realign_rt(c[k], nx, sg.shift));
            }
        }
    }
}

// --------------------------------------------------------------- bulk path

struct BulkSeg {
    const char* src;   // 16-byte aligned
    char* dst;         // 16-byte aligned
    int64_t bytes;     // a multiple of 16, > 0
    int64_t start;     // offset of the segment in the concatenation of all segments
};

struct BulkParams {
    BulkSeg seg[kMaxSegs];
    int32_t nseg;
    int64_t total;     // bytes of all segments (a multiple of 16)
    int32_t* status;   // timeout / bounds bits; may be NULL
};

// One thread per CTA: CTA b copies bytes [b*total/G, (b+1)*total/G) of the
// concatenation (16-byte granules) in chunks of at most kBulkChunk that never
// cross a segment.  Chunk i goes through stage i % kBulkStages: its bulk load
// completes on full[stage]; its bulk store is issued once that phase is seen;
// the stage is loaded again only after the store has finished reading it.
__global__ void __launch_bounds__(32, 1) copy_bulk_kernel(const __grid_constant__ BulkParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kBulkStages];
    if (threadIdx.x != 0) return;
    const int64_t units = p.total >> 4;
    const int64_t lo = units * static_cast<int64_t>(blockIdx.x) / gridDim.x * 16;
    const int64_t hi = units * (static_cast<int64_t>(blockIdx.x) + 1) / gridDim.x * 16;
    if (lo >= hi) return;
    for (int s = 0; s < kBulkStages; ++s) mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");

    int seg = 0;
    while (p.seg[seg].start + p.seg[seg].bytes <= lo) ++seg;
    int64_t pos = lo;
    char* sdst[kBulkStages];
    uint32_t sbytes[kBulkStages];
    int64_t nload = 0, nstore = 0;
    bool ok = true;

    // issue the load of the next chunk into stage nload % kBulkStages
    auto issue = [&]() -> bool {
        const BulkSeg& sg = p.seg[seg];
        const int64_t seg_end = sg.start + sg.bytes;
        int64_t n = seg_end - pos < hi - pos ? seg_end - pos : hi - pos;
        if (n > static_cast<int64_t>(kBulkChunk)) n = kBulkChunk;
        const int64_t off = pos - sg.start;
        if (out_of_bounds(seg < p.nseg && off >= 0 && n > 0 && (n & 15) == 0 && off + n <= sg.bytes, p.status))
            return false;
        const int s = static_cast<int>(nload % kBulkStages);
        sdst[s] = sg.dst + off;
        sbytes[s] = static_cast<uint32_t>(n);
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(n));
        bulk_load(smem + static_cast<size_t>(s) * kBulkChunk, sg.src + off, static_cast<uint32_t>(n), &full[s]);
        ++nload;
        pos += n;
        if (pos == seg_end) ++seg;
        return true;
    };

    while (nload < kBulkStages && pos < hi && ok) ok = issue();
    while (ok && nstore < nload) {
        const int s = static_cast<int>(nstore % kBulkStages);
        if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>((nstore / kBulkStages) & 1))) {
            if (p.status) atomicOr(p.status, kStatusTimeout);
            ok = false;
            break;
        }
        fence_proxy_async_smem();
        bulk_store(sdst[s], smem + static_cast<size_t>(s) * kBulkChunk, sbytes[s]);
        bulk_commit();
        ++nstore;
        // the stage of load nload last held chunk nload - kBulkStages; once at
        // most one store group (the one just issued) still reads, every older
        // stage is free
        if (pos < hi && nload <= nstore + kBulkStages - 2) {
            bulk_wait_read<1>();
            ok = issue();
        }
    }
    if (!ok) {
        // stop: let this CTA's loads in flight land before it exits (bounded)
        for (int64_t j = nstore; j < nload; ++j)
            if (!mbar_wait_bounded(&full[j % kBulkStages], static_cast<uint32_t>((j / kBulkStages) & 1)) && p.status)
                atomicOr(p.status, kStatusTimeout);
    }
    bulk_wait_all();
}

// ------------------------------------------------------------------ host side

struct Seg {
    const char* src;
    char* dst;
    int64_t bytes;
};

struct DeviceCopyInfo {
    int sms = 0;
    int reg_blocks_per_sm[2] = {0, 0};   // [kShift]
    bool bulk_ready = false;
};

std::mutex g_mu;
DeviceCopyInfo g_info[64];

int device_copy_info(const char* fn, DeviceCopyInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return fail(ZERO_ERR_CUDA, "%s: cannot query the device", fn);
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceCopyInfo& d = g_info[dev];
    if (d.sms == 0 && cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        d.sms = 0;
        return fail(ZERO_ERR_CUDA, "%s: cannot query the SM count", fn);
    }
    for (int k = 0; k < 2; ++k) {
        if (d.reg_blocks_per_sm[k] != 0) continue;
        int n = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, k ? copy_reg_kernel<true> : copy_reg_kernel<false>, kRegThreads, 0);
        if (e != cudaSuccess || n < 1) return fail(ZERO_ERR_CUDA, "%s: occupancy query failed: %s", fn, cudaGetErrorString(e));
        d.reg_blocks_per_sm[k] = n;
    }
    if (!d.bulk_ready) {
        cudaError_t e = cudaFuncSetAttribute(copy_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kBulkSmem));
        if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: cannot raise the shared-memory limit: %s", fn, cudaGetErrorString(e));
        d.bulk_ready = true;
    }
    *out = d;
    return ZERO_OK;
}

int check_launch(const char* fn) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
    return ZERO_OK;
}

// Host-side description of one register-kernel segment.
RegSeg make_reg_seg(const Seg& g) {
    RegSeg r{};
    r.src = g.src;
    r.dst = g.dst;
    r.bytes = g.bytes;
    r.head = static_cast<int64_t>((16u - (reinterpret_cast<uintptr_t>(g.dst) & 15u)) & 15u);
    if (r.head > g.bytes) r.head = g.bytes;
    r.nblk = (g.bytes - r.head) / 16;
    const uintptr_t a = reinterpret_cast<uintptr_t>(g.src + r.head);
    r.src_al = reinterpret_cast<const char*>(a & ~static_cast<uintptr_t>(15));
    r.shift = r.nblk > 0 ? static_cast<int32_t>(a & 15u) : 0;
    return r;
}

// Enqueue copy_reg_kernel<kShift> over `segs` (all of one class).
template <bool kShift>
int launch_reg_class(const std::vector<RegSeg>& segs, int esize, int32_t* status, const DeviceCopyInfo& d,
                     cudaStream_t stream, const char* fn) {
    for (size_t first = 0; first < segs.size(); first += kMaxSegs) {
        const size_t n = std::min<size_t>(kMaxSegs, segs.size() - first);
        RegParams prm{};
        prm.esize = esize;
        prm.status = status;
        int64_t tasks = 0;
        for (size_t i = 0; i < n; ++i) {
            prm.seg[i] = segs[first + i];
            prm.seg[i].task0 = tasks;
            tasks += std::max<int64_t>(1, (prm.seg[i].nblk + kTaskBlocks - 1) / kTaskBlocks);
        }
        prm.nseg = static_cast<int32_t>(n);
        prm.ntasks = tasks;
        const int64_t warps_per_block = kRegThreads / 32;
        int64_t blocks = (tasks + warps_per_block - 1) / warps_per_block;
        blocks = std::min<int64_t>(blocks, static_cast<int64_t>(d.sms) * d.reg_blocks_per_sm[kShift ? 1 : 0]);
        copy_reg_kernel<kShift><<<static_cast<unsigned int>(std::max<int64_t>(1, blocks)), kRegThreads, 0, stream>>>(prm);
        if (int rc = check_launch(fn)) return rc;
    }
    return ZERO_OK;
}

// Enqueue the register kernel over `segs` (any phases, any memory): the
// segments whose phases agree (and the edge-only ones) in one launch, those
// that need realigning in another.
int launch_reg(const std::vector<Seg>& segs, int esize, int32_t* status, const DeviceCopyInfo& d,
               cudaStream_t stream, const char* fn) {
    std::vector<RegSeg> same, shifted;
    for (const Seg& g : segs) {
        if (g.bytes <= 0) continue;
        const RegSeg r = make_reg_seg(g);
        (r.shift == 0 ? same : shifted).push_back(r);
    }
    if (!same.empty())
        if (int rc = launch_reg_class<false>(same, esize, status, d, stream, fn)) return rc;
    if (!shifted.empty())
        if (int rc = launch_reg_class<true>(shifted, esize, status, d, stream, fn)) return rc;
    return ZERO_OK;
}

// Enqueue the bulk kernel over `segs` (each 16-byte aligned on both sides,
// a multiple of 16 bytes long, both ends in this GPU's memory).
int launch_bulk(const std::vector<Seg>& segs, int32_t* status, const DeviceCopyInfo& d, cudaStream_t stream,
                const char* fn) {
    for (size_t first = 0; first < segs.size(); first += kMaxSegs) {
        const size_t n = std::min<size_t>(kMaxSegs, segs.size() - first);
        BulkParams prm{};
        prm.status = status;
        int64_t total = 0;
        for (size_t i = 0; i < n; ++i) {
            const Seg& g = segs[first + i];
            prm.seg[i] = BulkSeg{g.src, g.dst, g.bytes, total};
            total += g.bytes;
        }
        prm.nseg = static_cast<int32_t>(n);
        prm.total = total;
        // one CTA per SM; fewer when there are fewer 16-byte granules than SMs
        const int64_t blocks = std::min<int64_t>(d.sms, total / 16);
        copy_bulk_kernel<<<static_cast<unsigned int>(blocks), 32, kBulkSmem, stream>>>(prm);
        if (int rc = check_launch(fn)) return rc;
    }
    return ZERO_OK;
}

// Copy every segment: bodies that can take the bulk kernel go there, the
// rest (and the bodies' sub-16-byte edges) through the register kernel.
// `dst_local`: every destination lies in this GPU's memory (the caller
// checked); each source is checked here.  Without it nothing takes the bulk
// kernel.
int launch_copy(const std::vector<Seg>& segs, int esize, bool dst_local, int32_t* status, cudaStream_t stream,
                const char* fn) {
    DeviceCopyInfo d;
    if (int rc = device_copy_info(fn, &d)) return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: cannot query the device", fn);
    std::vector<Seg> bulk, reg;
    for (const Seg& g : segs) {
        if (g.bytes <= 0) continue;
        const uintptr_t sa = reinterpret_cast<uintptr_t>(g.src), da = reinterpret_cast<uintptr_t>(g.dst);
        const int64_t head = std::min<int64_t>(g.bytes, static_cast<int64_t>((16u - (da & 15u)) & 15u));
        const int64_t body = (g.bytes - head) / 16 * 16;
        if (dst_local && ((sa ^ da) & 15u) == 0 && body > 0 && local_device_memory(g.src, dev)) {
            bulk.push_back(Seg{g.src + head, g.dst + head, body});
            if (head > 0) reg.push_back(Seg{g.src, g.dst, head});
            if (head + body < g.bytes) reg.push_back(Seg{g.src + head + body, g.dst + head + body, g.bytes - head - body});
        } else {
            reg.push_back(g);
        }
    }
    if (!bulk.empty())
        if (int rc = launch_bulk(bulk, status, d, stream, fn)) return rc;
    if (!reg.empty())
        if (int rc = launch_reg(reg, esize, status, d, stream, fn)) return rc;
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
    // setup-time copy: the register kernel only (no waits, nothing to report)
    if (!segs.empty())
        if (int rc = launch_copy(segs, es, /*dst_local=*/false, nullptr, s, fn)) return rc;
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
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(ZERO_ERR_CUDA, "%s: cannot query the device", fn);
    if (int rc = launch_copy(segs, es, local_device_memory(dst, dev), status, reinterpret_cast<cudaStream_t>(stream),
                             fn))
        return rc;
    return ok();
}
