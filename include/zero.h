/*
 * zero.h - C ABI of the ZeRO-DP partitioned mixed-precision Adam step (B200).
 *
 * The method: ZeRO, "Memory Optimizations Toward Training Trillion Parameter
 * Models" (arXiv 1910.02054), as described by the azimuth.plus explainer of
 * that title ("ZeRO explainer" below) and the codewithpapers method record
 * "ZeRO".  Data-parallel replicas keep only 1/N of the model states; the
 * gradients of the N replicas are reduce-scattered so that every rank holds
 * the reduced gradients of its own partition, every rank updates its
 * partition of the fp32 Adam states, and the updated low-precision parameters
 * are all-gathered.
 *
 * Conventions shared by every call:
 *  - Device pointers are CUDA global-memory addresses on the current device.
 *    Host pointers are ordinary process memory.  Each argument says which.
 *  - The caller owns all memory.  No call allocates device memory; only
 *    zero_partition_layout allocates host arrays, released by
 *    zero_layout_free.
 *  - Device work is enqueued on `stream` (NULL = the legacy default stream)
 *    and is asynchronous: nothing synchronizes inside a call.  Results written
 *    to device memory (flags, norms) are valid once the stream reaches them.
 *  - Every call returns ZERO_OK (0) or a negative ZERO_ERR_* code, validates
 *    all arguments before launching anything, and launches nothing on error.
 *    zero_last_error() returns a message for the calling thread's last error.
 *  - Element counts and offsets are in elements of the named dtype.
 */
#ifndef ZERO_STEP_H
#define ZERO_STEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); declared opaque so that this header needs no
 * CUDA include. */
typedef struct CUstream_st* zero_stream_t;

typedef enum {
    ZERO_F16 = 0,   /* IEEE binary16 */
    ZERO_BF16 = 1,  /* bfloat16 */
    ZERO_F32 = 2    /* IEEE binary32 (flatten only) */
} zero_dtype_t;

enum {
    ZERO_OK = 0,
    ZERO_ERR_ARG = -1,            /* null pointer, bad count, bad world size */
    ZERO_ERR_ALIGN = -2,          /* pointer not aligned to its element size */
    ZERO_ERR_DTYPE = -3,          /* dtype not supported by this call */
    ZERO_ERR_RANGE = -4,          /* partition / bucket / range out of bounds */
    ZERO_ERR_CUDA = -5,           /* a CUDA launch or query failed */
    ZERO_ERR_NOMEM = -6           /* host allocation failed (layout only) */
};

/* Largest number of replicas (ranks) one call accepts. */
#define ZERO_MAX_WORLD 128

/* `partition` value that processes every rank's partition in one launch. */
#define ZERO_ALL_PARTITIONS (-1)

/* ------------------------------------------------------------------------ */
/* Partition layout                                                          */
/* ------------------------------------------------------------------------ */

/* Layout of a parameter list in constant-size fused buffers ("buckets").
 * All arrays are library-owned host memory. */
typedef struct {
    int32_t world;              /* N */
    int32_t align_elems;        /* padding unit factor (>= 1) */
    int64_t n_tensors;
    int64_t n_buckets;
    int64_t* bucket_numel;      /* [n_buckets] real elements */
    int64_t* bucket_padded;     /* [n_buckets] multiple of world*align_elems */
    int64_t* bucket_offset;     /* [n_buckets] start in the flat concatenation of padded buckets */
    int64_t* bucket_first;      /* [n_buckets] first tensor index */
    int64_t* bucket_count;      /* [n_buckets] number of tensors */
    int64_t* tensor_numel;      /* [n_tensors] copy of the input element counts */
    int64_t* tensor_bucket;     /* [n_tensors] bucket of each tensor */
    int64_t* tensor_offset;     /* [n_tensors] start of each tensor inside its bucket */
} zero_layout_t;

/*
 * zero_partition_layout - pack tensors into constant-size buffers and split
 * each buffer into N equal partitions.
 *
 * Source: ZeRO explainer, "Constant-size buffers" (many small tensors fused
 * into one buffer of a fixed size that does not grow with the model) and
 * "Stage 1 - Optimizer State Partitioning (P_os)" (each of N GPUs holds 1/N
 * of the states).  The pages fix no packing rule; this one is: tensors in
 * list order, appended to the open bucket while the bucket stays within
 * `bucket_elems`; a tensor that does not fit closes the bucket; a tensor
 * larger than the capacity gets a bucket of its own; tensors are never split.
 * `bucket_elems == 0` means one bucket.  Each bucket is padded with zeros up
 * to a multiple of world*align_elems; rank r's partition of bucket b is
 * elements [r*P_b, (r+1)*P_b) with P_b = bucket_padded[b] / world.
 *
 * numels      host, [n_tensors] element counts (>= 0)
 * n_tensors   >= 0
 * world       N, 1..ZERO_MAX_WORLD
 * bucket_elems capacity in elements, >= 0
 * align_elems >= 1 (1 = pad to a multiple of N only)
 * out         host; filled on success, untouched on error
 * Errors: ZERO_ERR_ARG, ZERO_ERR_NOMEM.  Host only, no CUDA call.
 */
int zero_partition_layout(const int64_t* numels, int64_t n_tensors, int32_t world,
                          int64_t bucket_elems, int32_t align_elems, zero_layout_t* out);

/* Release the arrays of a layout filled by zero_partition_layout (safe on a
 * zeroed struct; the struct itself is the caller's). */
void zero_layout_free(zero_layout_t* layout);

/*
 * zero_flatten_bucket - copy one bucket's tensors into its fused buffer.
 *
 * Source: ZeRO explainer, "Constant-size buffers" and "Memory
 * defragmentation" (state lives in pre-allocated contiguous blocks).  Tensor
 * i of bucket b is copied to bucket_buf[tensor_offset[i] ...]; the padding
 * [bucket_numel[b], bucket_padded[b]) is set to zero.
 *
 * layout      host, from zero_partition_layout
 * bucket      0 .. n_buckets-1
 * tensor_ptrs host array of n_tensors DEVICE pointers indexed by tensor id;
 *             only the bucket's entries are read; each holds numels[i]
 *             contiguous elements of `dtype`
 * dtype       ZERO_F16, ZERO_BF16 or ZERO_F32
 * bucket_buf  device, bucket_padded[b] elements, must not overlap a source
 * Errors: ZERO_ERR_ARG, ZERO_ERR_RANGE, ZERO_ERR_DTYPE, ZERO_ERR_ALIGN,
 * ZERO_ERR_CUDA.
 */
int zero_flatten_bucket(const zero_layout_t* layout, int64_t bucket,
                        const void* const* tensor_ptrs, zero_dtype_t dtype,
                        void* bucket_buf, zero_stream_t stream);

/* ------------------------------------------------------------------------ */
/* The fused step                                                            */
/* ------------------------------------------------------------------------ */

typedef struct {
    float lr;
    float beta1;
    float beta2;
    float eps;
    float weight_decay;   /* decoupled (AdamW): weights scale by 1 - lr*wd */
    int64_t step;         /* t of THIS update, 1-based; counts applied updates only */
    float grad_divisor;   /* replicas' sum is divided by this; 0 = world (the mean) */
} zero_adam_hparams_t;

/* Bytes of device workspace that zero_reduce_scatter_adam_step needs when it
 * is asked for the gradient square-norm. */
size_t zero_step_workspace_bytes(void);

/*
 * zero_reduce_scatter_adam_step - one fused pass of the ZeRO-2 step over one
 * bucket: reduce-scatter + unscale + overflow test + Adam + parameter
 * write-back.
 *
 * Sources: ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)" (each
 * rank receives by reduce-scatter only the reduced gradients of its own
 * partition and updates that partition), "Stage 1 - Optimizer State
 * Partitioning (P_os)" (each rank updates its parameters with its 1/N of the
 * fp32 optimizer states, then an all-gather distributes the updated
 * parameters), model-states paragraph (fp16 parameters and gradients, fp32
 * master weights, momentum and variance).
 *
 * The N replicas' gradient buffers are resident on this GPU.  For each
 * processed element i (see `partition`):
 *   s   = fp32(G_0[i]) + fp32(G_1[i]) + ... + fp32(G_{N-1}[i])   (left to right)
 *   g   = s * fp32(1 / (divisor * loss_scale))
 *   overflow if s is inf or NaN (any element of the call)
 *   m'  = fma(b1, m, (1-b1)*g);  v' = fma(b2, v, ((1-b2)*g)*g)
 *   u   = (m' * 1/(1-b1^t)) / fma(sqrt(v'), 1/sqrt(1-b2^t), eps)
 *   p'  = fma(-lr, u, p * (1 - lr*wd));   param = round_to_nearest_even(p')
 * Scalar constants are computed in double and rounded once to float; the
 * division and square root are IEEE correctly rounded.  The results do not
 * depend on the launch configuration.
 *
 * grad_bufs    host array of `world` DEVICE pointers, each padded_numel
 *              elements of grad_dtype (replica k's bucket, unscaled by nothing)
 * world        N, 1..ZERO_MAX_WORLD
 * padded_numel elements of a replica's bucket, a multiple of world (>= 0)
 * partition    ZERO_ALL_PARTITIONS: every rank's partition in one launch; the
 *              state arrays and param_out then hold padded_numel elements in
 *              flat order (the concatenation of the partitions in rank order).
 *              r in 0..world-1: rank r only; state arrays and param_out hold
 *              P = padded_numel/world elements, element j reads gradient
 *              element r*P + j.
 * grad_dtype   ZERO_F16 or ZERO_BF16
 * master_in, m_in, v_in       device fp32, the current state (read)
 * master_out, m_out, v_out    device fp32, the updated state (written).  May
 *              equal the *_in pointers (in-place update); otherwise they must
 *              not overlap them.  Writing to a second bank and committing it
 *              only when *overflow_flag stays 0 keeps a skipped step's state
 *              bit-identical.
 * param_out    device, updated parameters in param_dtype (ZERO_F16/ZERO_BF16):
 *              the all-gather payload, in the same indexing as the states
 * hp           host, hyper-parameters; hp->step >= 1
 * loss_scale   > 0 and finite: the gradients carry this factor
 * overflow_flag device int32, OR-ed into, never cleared by the call:
 *              bit 0 (value 1) when any reduced gradient of this call is inf
 *              or NaN; bit 1 (value 2) when the kernel gave up waiting on its
 *              own shared-memory copy pipeline (2 s without progress: a device
 *              fault, not a property of the data) and its outputs are
 *              incomplete.  Commit a step only when the flag is 0.  Clear it
 *              before the first call of a step; calls over several buckets
 *              then OR into one flag for the whole step.
 * grad_sqnorm  device double or NULL; when not NULL, sum over the call's
 *              elements of g*g is ADDED to it (clear it at the start of a
 *              step).  Each g*g is exact in double; per-thread and per-block
 *              sums in double, folded over blocks in a fixed order:
 *              deterministic.
 * workspace    device, zero_step_workspace_bytes() bytes, zero-filled once
 *              before its first use; required when grad_sqnorm is not NULL
 *              (NULL allowed otherwise).  Each call leaves it zero-filled
 *              again.  Calls that share a workspace must not run concurrently.
 * Errors: ZERO_ERR_ARG, ZERO_ERR_RANGE, ZERO_ERR_DTYPE, ZERO_ERR_ALIGN
 * (fp32 pointers need 4-byte, 16-bit pointers 2-byte alignment; 16-byte
 * alignment of all arrays at the same element gives the vector path),
 * ZERO_ERR_CUDA.
 */
int zero_reduce_scatter_adam_step(
    const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
    zero_dtype_t grad_dtype,
    const float* master_in, const float* m_in, const float* v_in,
    float* master_out, float* m_out, float* v_out,
    void* param_out, zero_dtype_t param_dtype,
    const zero_adam_hparams_t* hp, float loss_scale,
    int32_t* overflow_flag, double* grad_sqnorm, void* workspace,
    zero_stream_t stream);

/*
 * zero_grad_stats - the reduce-scatter's sums without the update: overflow
 * flag and squared norm of one bucket's reduced gradients.
 *
 * Source: the reduce-scatter of ZeRO explainer, "Stage 2 - Gradient
 * Partitioning (P_os+g)", taken alone.  For each processed element (same
 * `partition` convention as zero_reduce_scatter_adam_step) it forms the
 * rank-order fp32 sum s of the N replicas and g = s * fp32(1/(divisor *
 * loss_scale)); it sets bit 0 of *overflow_flag when any s is inf or NaN
 * (never clears it) and, when grad_sqnorm is not NULL, adds the sum of g*g
 * (each g*g exact in double, summed in double, deterministic) to
 * *grad_sqnorm.  It reads 2N bytes per element and writes no state.
 *
 * Purpose: decide skip and clipping for a whole step before any state is
 * written.  Followed by zero_reduce_scatter_adam_step_gated, the update can
 * run in place (one bank of states: the pages' 12 Psi / N bytes per rank)
 * with an exact skip, for 4N + 26 bytes per element in total.
 *
 * grad_bufs, world, padded_numel, partition, grad_dtype: as for
 *              zero_reduce_scatter_adam_step
 * loss_scale   > 0, finite;  grad_divisor >= 0 (0 = world)
 * overflow_flag device int32, OR-ed into
 * grad_sqnorm  device double or NULL (added to; needs `workspace`)
 * workspace    as for zero_reduce_scatter_adam_step
 * Errors: ZERO_ERR_ARG, ZERO_ERR_RANGE, ZERO_ERR_DTYPE, ZERO_ERR_ALIGN,
 * ZERO_ERR_CUDA.
 */
int zero_grad_stats(const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
                    zero_dtype_t grad_dtype, float loss_scale, float grad_divisor,
                    int32_t* overflow_flag, double* grad_sqnorm, void* workspace, zero_stream_t stream);

/*
 * zero_reduce_scatter_adam_step_gated - zero_reduce_scatter_adam_step with
 * a device-side gate and global-norm gradient clipping.
 *
 * Same arguments and results as zero_reduce_scatter_adam_step, plus:
 * gate         device int32 or NULL.  When not NULL and non-zero when the
 *              kernel starts, the call writes nothing at all (no state, no
 *              parameters, no flag, no norm).  Pass the flag that
 *              zero_grad_stats filled for the whole step: an overflowing
 *              step then leaves in-place states bit-identical.  It must not
 *              be this call's own overflow_flag, and nothing may write it
 *              while the kernel runs.
 * clip_sqnorm  device double or NULL.  When not NULL, the unscaled gradient
 *              is multiplied by clip = min(1, max_norm / (sqrt(*clip_sqnorm)
 *              + 1e-6)) (computed in double, rounded once to float):
 *              g = (s * inv) * clip.  Pass the step's total squared norm from
 *              zero_grad_stats.  Global-norm clipping is not on the pages.
 * max_norm     > 0 and finite when clip_sqnorm is not NULL
 * Errors: those of zero_reduce_scatter_adam_step.
 */
int zero_reduce_scatter_adam_step_gated(
    const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
    zero_dtype_t grad_dtype,
    const float* master_in, const float* m_in, const float* v_in,
    float* master_out, float* m_out, float* v_out,
    void* param_out, zero_dtype_t param_dtype,
    const zero_adam_hparams_t* hp, float loss_scale,
    int32_t* overflow_flag, double* grad_sqnorm, void* workspace,
    const int32_t* gate, const double* clip_sqnorm, float max_norm,
    zero_stream_t stream);

/*
 * zero_reduce_scatter_grads - the reduce-scatter of a staged step: store
 * each processed element's reduced, unscaled gradient in fp32.
 *
 * Source: ZeRO explainer (azimuth.plus), "Stage 2 - Gradient Partitioning
 * (P_os+g)": the gradients are reduce-scattered so that each rank keeps the
 * reduced gradients of its own partition only.  For each processed element
 * (same `partition` convention as zero_reduce_scatter_adam_step) it forms
 * the rank-order fp32 sum s of the N replicas and stores
 * g = s * fp32(1/(divisor * loss_scale)) to reduced_out; the flag and the
 * norm are those of zero_grad_stats.  2N + 4 bytes per element.
 *
 * reduced_out  device fp32, one element per processed element (P elements
 *              for one partition, padded_numel for ZERO_ALL_PARTITIONS),
 *              4-byte aligned (16-byte aligned at the same element as the
 *              gradient buffers for the vector path); must not overlap a
 *              gradient buffer.  Caller-owned.
 * other arguments: as for zero_grad_stats.
 * Errors: those of zero_grad_stats; ZERO_ERR_ARG for a NULL reduced_out.
 */
int zero_reduce_scatter_grads(const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
                              zero_dtype_t grad_dtype, float loss_scale, float grad_divisor, float* reduced_out,
                              int32_t* overflow_flag, double* grad_sqnorm, void* workspace, zero_stream_t stream);

/*
 * zero_adam_step_reduced - the update of a staged step: Adam/AdamW on a
 * partition from the reduced gradients that zero_reduce_scatter_grads
 * stored.
 *
 * Source: ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)" (each
 * rank updates its own partition from its reduced gradients); the update is
 * the one of zero_reduce_scatter_adam_step with g read from reduced_grad
 * instead of formed from the replicas, so both give identical bits for the
 * same inputs.  Reads 16 and writes 14 bytes per element.
 *
 * reduced_grad  device fp32, `count` elements (unscaled gradients)
 * count         elements, >= 0 (0: nothing is launched)
 * master_in .. param_out, param_dtype, hp: as for
 *               zero_reduce_scatter_adam_step, `count` elements each
 *               (hp->grad_divisor is not used: the gradients are already
 *               unscaled); in place when each *_out equals its *_in
 * status        device int32, required: bit 1 (value 2) is OR-ed in when
 *               the kernel's copy pipeline gave up waiting (then the
 *               outputs are incomplete; see zero_reduce_scatter_adam_step);
 *               otherwise untouched.  Must not be `gate`.
 * gate, clip_sqnorm, max_norm: as for zero_reduce_scatter_adam_step_gated
 *               (pass the flag and the norm of the step's
 *               zero_reduce_scatter_grads calls: an overflowing step then
 *               writes nothing)
 * No overflow flag or norm is produced (the reduce-scatter made them).
 * Errors: ZERO_ERR_ARG, ZERO_ERR_DTYPE, ZERO_ERR_ALIGN, ZERO_ERR_CUDA.
 */
int zero_adam_step_reduced(const float* reduced_grad, int64_t count,
                           const float* master_in, const float* m_in, const float* v_in,
                           float* master_out, float* m_out, float* v_out,
                           void* param_out, zero_dtype_t param_dtype,
                           const zero_adam_hparams_t* hp, int32_t* status,
                           const int32_t* gate, const double* clip_sqnorm, float max_norm,
                           zero_stream_t stream);

/*
 * zero_adam_step_reduced_bcast - zero_adam_step_reduced that writes the
 * updated parameters to several destinations: the all-gather of the
 * updated parameters done by the update's own stores.
 *
 * Source: ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)" (after
 * the update the parameters are all-gathered, so every rank again holds all
 * of them).  Rank r passes, for every rank q, the address of slot r of rank
 * q's parameter buffer (peers' buffers mapped into this process, e.g. with
 * zero_ipc_import); each updated parameter is stored to all of them, so no
 * separate gather is needed once every rank's call has completed.  Results
 * equal those of zero_adam_step_reduced at every destination.
 *
 * param_dsts  host array of n_dsts device pointers (1 .. ZERO_MAX_WORLD),
 *             each `count` elements of param_dtype, 2-byte aligned, not
 *             overlapping each other or any input or state array.  When
 *             their 16-byte phases differ from the first's, every element
 *             is stored on its own (slower, same results).
 * other arguments: as for zero_adam_step_reduced.
 * Errors: those of zero_adam_step_reduced.
 */
int zero_adam_step_reduced_bcast(const float* reduced_grad, int64_t count,
                                 const float* master_in, const float* m_in, const float* v_in,
                                 float* master_out, float* m_out, float* v_out,
                                 void* const* param_dsts, int32_t n_dsts, zero_dtype_t param_dtype,
                                 const zero_adam_hparams_t* hp, int32_t* status,
                                 const int32_t* gate, const double* clip_sqnorm, float max_norm,
                                 zero_stream_t stream);

/*
 * zero_reduce_scatter_adam_step_noalloc - zero_reduce_scatter_adam_step for
 * callers that cannot allocate device memory.
 *
 * The paper has no counterpart: this is a calling convention of this
 * library, not a step of the method.  Some callers cannot provide the
 * device workspace that the gradient norm needs: code under an allocator
 * that owns all device memory and forbids direct cudaMalloc, a host thread
 * that must not take cudaMalloc's implicit device synchronization, or a C
 * caller with no device allocator.  This entry point takes the same
 * arguments minus `workspace` and keeps that scratch in a fixed array in the
 * library's device image instead (33,024 bytes per GPU that loads the
 * library, held until exit); it calls no cudaMalloc, cudaFree or other
 * allocating routine.  Inputs and outputs are still the caller's.
 *
 * Results equal those of zero_reduce_scatter_adam_step.  Limits:
 *  - the scratch holds 4096 per-block partial sums; the kernels' grids are
 *    at most 16 blocks per SM (2368 on a B200), so every input size fits,
 *    and a call whose grid would exceed 4096 blocks returns
 *    ZERO_ERR_RANGE;
 *  - all calls on a device share the scratch: calls that overlap on the GPU
 *    (other streams, other host threads) race on it; each call clears the
 *    ticket word it needs before its kernel, stream-ordered;
 *  - the first call on a device that passes grad_sqnorm looks up the
 *    scratch's device address (cudaGetSymbolAddress, once per device, with
 *    that device current): make that first call before any stream capture.
 * Errors: those of zero_reduce_scatter_adam_step, plus ZERO_ERR_RANGE above.
 */
int zero_reduce_scatter_adam_step_noalloc(
    const void* const* grad_bufs, int32_t world, int64_t padded_numel, int32_t partition,
    zero_dtype_t grad_dtype,
    const float* master_in, const float* m_in, const float* v_in,
    float* master_out, float* m_out, float* v_out,
    void* param_out, zero_dtype_t param_dtype,
    const zero_adam_hparams_t* hp, float loss_scale,
    int32_t* overflow_flag, double* grad_sqnorm,
    zero_stream_t stream);

/* Bytes of the fixed scratch array used by
 * zero_reduce_scatter_adam_step_noalloc (per GPU that loads the library). */
size_t zero_step_static_scratch_bytes(void);

/*
 * zero_allgather_params - rebuild full parameters from N rank shards.
 *
 * Source: ZeRO explainer, "Stage 3 - Parameter Partitioning (P_os+g+p)" (each
 * layer's parameters are reconstructed by all-gather from the ranks that own
 * its slices, used, then discarded) and Stage 1/2 (all-gather of the updated
 * parameters).  dst[r*part_numel + j] = shards[r][shard_offset + j] for
 * r < world, j < part_numel: a bit-exact copy.  With shards that concatenate
 * each unit's slices in unit order, shard_offset selects one unit.
 *
 * shards       host array of `world` DEVICE pointers (this GPU's memory, or
 *              another GPU's memory mapped into this process: the copy uses
 *              plain loads only)
 * world        1..ZERO_MAX_WORLD
 * shard_offset first element of the slice in every shard (>= 0)
 * part_numel   elements per rank (>= 0); any value: slices whose 16-byte
 *              phase differs from their destination's are realigned in
 *              registers, so odd sizes keep 16-byte loads and stores
 * dtype        ZERO_F16, ZERO_BF16 or ZERO_F32
 * dst          device, world*part_numel elements, must not overlap a shard
 * status       device int32 or NULL, 4-byte aligned: the bounds-checking
 *              debug build ORs 4 into it when an index check fails (the access
 *              is then skipped); the release build never writes it
 * Reads whole aligned 16-byte blocks that hold at least one byte of a slice,
 * so never a page outside the slices; writes exactly dst's range.
 * Errors: ZERO_ERR_ARG, ZERO_ERR_DTYPE, ZERO_ERR_ALIGN, ZERO_ERR_CUDA.
 */
int zero_allgather_params(const void* const* shards, int32_t world, int64_t shard_offset,
                          int64_t part_numel, zero_dtype_t dtype, void* dst, int32_t* status,
                          zero_stream_t stream);

/*
 * zero_test_wait_timeout - self-test of the bounded device waits.
 *
 * The paper has no counterpart: a test hook of this library.  The
 * shared-memory pipeline of the fused step waits on mbarriers that its own
 * bulk copies complete, each wait limited to 2 s of wall time; when a limit
 * runs out the kernel ORs 2 into the overflow flag, stops, and returns.
 * This call runs the same wait routine on an mbarrier that nothing ever
 * arrives at, with the limit `limit_ns`: after about that long it ORs 2 into
 * *status and the kernel returns, so a caller can check that a stuck wait
 * ends with a status instead of a hang.
 * status    device int32, OR-ed into
 * limit_ns  0 .. 1e10
 * Errors: ZERO_ERR_ARG, ZERO_ERR_ALIGN, ZERO_ERR_CUDA.
 */
int zero_test_wait_timeout(int32_t* status, int64_t limit_ns, zero_stream_t stream);

/*
 * zero_test_force_step_kernel - choose the fused step's kernel by hand.
 *
 * The paper has no counterpart: a test hook of this library.  Every fused
 * step call (zero_reduce_scatter_adam_step, its gated and no-alloc variants,
 * the runner) normally picks one of four kernels that compute the same bits:
 * the shared-memory pipeline kernel for large calls with N >= 6, the
 * oct-streaming kernel (32-byte state stores) for N <= 2, mid-size calls and
 * peer memory when the fp32 outputs are 32-byte aligned where the vector
 * region starts, the quad-streaming kernel for those calls otherwise, the
 * register kernel for large calls with 3 <= N <= 5, N > 20 or arrays off a
 * common 16-byte phase.  This call
 * makes the process's later calls take `kind` instead wherever that kernel
 * can run the call (the pipeline kernel needs a common phase, N <= 20, one
 * whole tile and gradients in this GPU's memory; the quad kernel a common
 * phase and N <= 16; the oct kernel that and the 32-byte alignment), so that
 * tests reach each kernel at small sizes.  The statistics pass, the staged
 * reduce-scatter and the staged update follow it too: 1 forces their
 * pipeline kernels, 0 their register kernels, 2 the statistics' quad kernel,
 * 3 the reduce-scatter's oct kernel (N <= 2, `reduced` 32-byte aligned; the
 * staged update keeps its automatic choice).
 * kind  -1 automatic (the default), 0 register, 1 pipeline, 2 quad, 3 oct
 * Errors: ZERO_ERR_ARG.  Host only, no CUDA call.
 */
int zero_test_force_step_kernel(int32_t kind);

/* ------------------------------------------------------------------------ */
/* Step runner: the whole step over every bucket                             */
/* ------------------------------------------------------------------------ */

/* One bucket as the runner sees it; every pointer is caller-owned device
 * memory.  Bank b of the states is master[b], m[b], v[b] (fp32, padded_numel
 * elements each) and params[b] (param dtype). */
typedef struct {
    int64_t padded_numel;           /* multiple of world */
    const void* const* grad_bufs;   /* host array of `world` device pointers; copied by create */
    float* master[2];
    float* m[2];
    float* v[2];
    void* params[2];
} zero_bucket_banks_t;

typedef struct zero_runner zero_runner_t;   /* opaque, host memory */

/*
 * zero_runner_create / _launch / _commit / _state / _set_state / _destroy -
 * the ZeRO-2 step over a list of buckets with an exact skip.
 *
 * Source: ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)" (every
 * bucket's reduce-scatter + update of the partitions) and "Constant-size
 * buffers" (the buckets); the skip on overflow and the dynamic loss scale are
 * not on the pages (zero_loss_scale_update).
 *
 * zero_runner_launch enqueues on `stream`, without waiting: clear
 * *flag_dev (and *grad_sqnorm), the fused step over every bucket reading bank
 * `cur` and writing bank `cur ^ 1` with hyper-parameters hp (step = t + 1)
 * and the current loss scale, and a copy of *flag_dev into *flag_host.
 * zero_runner_commit waits for the stream (pass the stream the launch used),
 * reads *flag_host and, when it is
 * 0, makes bank `cur ^ 1` current and advances t; it then applies
 * zero_loss_scale_update and reports *applied (1 = update applied).  A launch
 * must be followed by a commit before the next launch.
 *
 * create: buckets[n_buckets] (copied; the pointer arrays too), world 1 ..
 *   ZERO_MAX_WORLD, dtypes and hp as for zero_reduce_scatter_adam_step
 *   (hp->step is the t of the first update), loss_scale > 0, growth_interval
 *   >= 1, min_scale > 0; flag_dev device int32; flag_host host int32 (pinned,
 *   e.g. cudaHostAlloc); grad_sqnorm device double or NULL (with workspace as
 *   for zero_reduce_scatter_adam_step).  Every bucket is validated for both
 *   bank directions.  Allocates only the host-side runner object.
 * state / set_state: t (applied updates), loss scale, good-step count and the
 *   current bank, to read or to restore (e.g. from a checkpoint).
 * Errors: those of zero_reduce_scatter_adam_step; ZERO_ERR_ARG for a launch
 * without commit or a commit without launch; ZERO_ERR_CUDA from commit when
 * the kernel reported a pipeline timeout (flag bit 1): nothing is committed.
 */
int zero_runner_create(const zero_bucket_banks_t* buckets, int64_t n_buckets, int32_t world,
                       zero_dtype_t grad_dtype, zero_dtype_t param_dtype, const zero_adam_hparams_t* hp,
                       float loss_scale, int32_t growth_interval, float min_scale,
                       int32_t* flag_dev, int32_t* flag_host, double* grad_sqnorm, void* workspace,
                       zero_runner_t** out);
/*
 * zero_runner_create_staged - a runner for the staged route with one bank.
 *
 * Source: ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)" (the
 * reduce-scatter leaves each rank the reduced gradients of its partition,
 * which it then updates) and "Stage 1 - Optimizer State Partitioning (P_os)"
 * (one copy of the optimizer states: 12 Psi / N bytes per rank).
 *
 * launch enqueues: clear flag_dev[0..1] (and *grad_sqnorm); for every bucket
 * zero_reduce_scatter_grads into reduced[b] (flag_dev[0], the norm); then for
 * every bucket zero_adam_step_reduced in place on bank 0 (master[0], m[0],
 * v[0], params[0]) with gate = flag_dev[0], status = flag_dev[1] and, when
 * max_norm > 0, clipping by the step's norm; then a copy of both flag words
 * into flag_host[0..1].  commit: as for the two-bank runner, except that the
 * bank never changes (an overflowing step wrote nothing); t advances on
 * applied steps.  Bank 1 of the bucket descriptors is not used (may be NULL).
 *
 * reduced      host array of n_buckets device fp32 pointers, padded_numel
 *              elements each (caller-owned)
 * max_norm     0: no clipping; > 0: clip to this global norm (needs
 *              grad_sqnorm and workspace)
 * flag_dev     2 device int32 words, 8-byte aligned; flag_host 2 host words
 * other arguments: as for zero_runner_create.  set_state accepts bank 0 only.
 * Errors: those of zero_reduce_scatter_grads and zero_adam_step_reduced;
 * ZERO_ERR_ARG as for zero_runner_create; ZERO_ERR_CUDA from commit on a
 * pipeline timeout (bit 1 of either word).
 */
int zero_runner_create_staged(const zero_bucket_banks_t* buckets, int64_t n_buckets, int32_t world,
                              zero_dtype_t grad_dtype, zero_dtype_t param_dtype, const zero_adam_hparams_t* hp,
                              float loss_scale, int32_t growth_interval, float min_scale,
                              float* const* reduced, float max_norm,
                              int32_t* flag_dev, int32_t* flag_host, double* grad_sqnorm, void* workspace,
                              zero_runner_t** out);
int zero_runner_launch(zero_runner_t* runner, zero_stream_t stream);
int zero_runner_commit(zero_runner_t* runner, zero_stream_t stream, int32_t* applied);
int zero_runner_state(const zero_runner_t* runner, int64_t* t, float* loss_scale, int32_t* good_steps,
                      int32_t* bank);
int zero_runner_set_state(zero_runner_t* runner, int64_t t, float loss_scale, int32_t good_steps, int32_t bank);
void zero_runner_destroy(zero_runner_t* runner);
/*
 * zero_runner_bucket_kernel - which fused-step kernel the next
 * zero_runner_launch runs for bucket `bucket` of a two-bank runner: 0 the
 * register-streaming kernel, 1 the shared-memory pipeline kernel, 2 the
 * quad-streaming kernel, 3 the oct-streaming kernel (the numbering of
 * zero_test_force_step_kernel).  It
 * makes the launch's own preparation (bank cur, the current t and loss
 * scale, the kernel override in force) without enqueueing anything; the
 * choice depends on the bucket's size, N, the buffers' 16-byte phase and
 * whether every gradient buffer is this device's memory.
 * Errors: ZERO_ERR_ARG for a NULL argument, a bucket outside
 * 0..n_buckets-1 or a staged runner; else those of
 * zero_reduce_scatter_adam_step's validation.
 */
int zero_runner_bucket_kernel(const zero_runner_t* runner, int64_t bucket, int32_t* kind);


/* ------------------------------------------------------------------------ */
/* Multi-process ranks: sharing gradient and parameter buffers               */
/* ------------------------------------------------------------------------ */

/* Opaque CUDA IPC handle (the bytes of a cudaIpcMemHandle_t). */
typedef struct {
    unsigned char bytes[64];
} zero_ipc_handle_t;

/*
 * zero_ipc_export / zero_ipc_import / zero_ipc_close - share device buffers
 * between the processes (ranks) of one node.
 *
 * Source: ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)": each
 * rank needs, from every other rank, only the gradient slice of its own
 * partition.  With the peers' buffers mapped, a rank passes them (in rank
 * order, its own included) as `grad_bufs` to zero_reduce_scatter_adam_step
 * with partition = its rank: the kernel itself performs the reduce-scatter by
 * reading each peer's slice (NVLink P2P loads across GPUs), in fixed rank
 * order.  The updated parameter slots are then gathered the same way with
 * zero_allgather_params.  The ranks must synchronise on the host (a barrier)
 * between writing gradients and the step, and after the gather.
 *
 * zero_ipc_export: `ptr` any device address inside an allocation of the
 *   current process; fills `handle` (of the whole allocation) and `offset`
 *   (bytes from the allocation's start to ptr).  Host only.
 * zero_ipc_import: maps a handle exported by another process on this node
 *   (any device; peer access is enabled as needed); *ptr = mapped base +
 *   offset; *base is what zero_ipc_close takes.  Not for handles of the
 *   calling process itself.
 * zero_ipc_close: unmaps a base returned by zero_ipc_import.
 * Errors: ZERO_ERR_ARG, ZERO_ERR_CUDA.
 */
int zero_ipc_export(const void* ptr, zero_ipc_handle_t* handle, int64_t* offset);
int zero_ipc_import(const zero_ipc_handle_t* handle, int64_t offset, void** ptr, void** base);
int zero_ipc_close(void* base);

/* ------------------------------------------------------------------------ */
/* Host helpers                                                              */
/* ------------------------------------------------------------------------ */

/*
 * zero_loss_scale_update - dynamic loss scale after a step (host only).
 *
 * Not on the pages (they fix only the fp16 storage of gradients); the usual
 * rule: on overflow the update was skipped, the scale halves (not below
 * min_scale) and the good-step count restarts; otherwise the count grows and
 * the scale doubles after growth_interval consecutive good steps.
 * scale, good_steps  host, updated in place
 * Errors: ZERO_ERR_ARG (null pointer, growth_interval < 1, bad scale).
 */
int zero_loss_scale_update(float* scale, int32_t* good_steps, int32_t overflow,
                           int32_t growth_interval, float min_scale);

/* Static description of an error code. */
const char* zero_strerror(int code);

/* Message of the calling thread's most recent error ("" if none). */
const char* zero_last_error(void);

/* Version string of the library build. */
const char* zero_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_STEP_H */
