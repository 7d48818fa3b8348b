"""Python binding of libzero, the C ABI of the ZeRO-DP partitioned Adam step.

Argument marshalling only: every computation runs in the CUDA kernels of
libzero.so.  The functions carry the names of the C calls in include/zero.h
and take torch tensors (device memory, `data_ptr()`) or plain Python values;
streams default to torch's current stream.

The library is loaded from this package directory.  If it is missing, import
fails with an error that says how to build it: there is no fallback.

The C calls see bare pointers and cannot check sizes; the wrappers here check
what they can before anything is launched: device arguments must be
contiguous CUDA tensors of the right dtype holding at least the elements the
call touches (ZeroError otherwise).  A DevicePtr (another process's mapped
buffer) is passed through unchecked.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libzero.so")

ZERO_F16, ZERO_BF16, ZERO_F32 = 0, 1, 2
ZERO_ALL_PARTITIONS = -1
ZERO_MAX_WORLD = 128
ERRORS = {0: "ZERO_OK", -1: "ZERO_ERR_ARG", -2: "ZERO_ERR_ALIGN", -3: "ZERO_ERR_DTYPE",
          -4: "ZERO_ERR_RANGE", -5: "ZERO_ERR_CUDA", -6: "ZERO_ERR_NOMEM"}


class ZeroError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class _Layout(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int32), ("align_elems", ctypes.c_int32),
                ("n_tensors", ctypes.c_int64), ("n_buckets", ctypes.c_int64),
                ("bucket_numel", ctypes.POINTER(ctypes.c_int64)),
                ("bucket_padded", ctypes.POINTER(ctypes.c_int64)),
                ("bucket_offset", ctypes.POINTER(ctypes.c_int64)),
                ("bucket_first", ctypes.POINTER(ctypes.c_int64)),
                ("bucket_count", ctypes.POINTER(ctypes.c_int64)),
                ("tensor_numel", ctypes.POINTER(ctypes.c_int64)),
                ("tensor_bucket", ctypes.POINTER(ctypes.c_int64)),
                ("tensor_offset", ctypes.POINTER(ctypes.c_int64))]


class IpcHandle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


class DevicePtr:
    """A raw device address with a dtype, accepted wherever a tensor is
    (for buffers mapped from another process)."""

    def __init__(self, ptr: int, dtype):
        self.ptr, self.dtype = int(ptr), dtype

    def data_ptr(self) -> int:
        return self.ptr


class BucketBanks(ctypes.Structure):
    _fields_ = [("padded_numel", ctypes.c_int64), ("grad_bufs", ctypes.POINTER(ctypes.c_void_p)),
                ("master", ctypes.c_void_p * 2), ("m", ctypes.c_void_p * 2), ("v", ctypes.c_void_p * 2),
                ("params", ctypes.c_void_p * 2)]


class AdamHParams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("step", ctypes.c_int64), ("grad_divisor", ctypes.c_float)]


def load_library(path: str = LIB_PATH):
    """Load a build of libzero (this package's, or a variant such as the
    bounds-checking debug build) and declare its signatures.  The wrappers
    call the module-level `lib`; tests may swap it for a variant."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python zero_sharded_optimizer_reduce_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(path)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    L.zero_partition_layout.argtypes = [ctypes.POINTER(ctypes.c_int64), i64, i32, i64, i32,
                                        ctypes.POINTER(_Layout)]
    L.zero_partition_layout.restype = ctypes.c_int
    L.zero_layout_free.argtypes = [ctypes.POINTER(_Layout)]
    L.zero_layout_free.restype = None
    L.zero_flatten_bucket.argtypes = [ctypes.POINTER(_Layout), i64, ctypes.POINTER(vp), ctypes.c_int, vp, vp]
    L.zero_flatten_bucket.restype = ctypes.c_int
    L.zero_step_workspace_bytes.argtypes = []
    L.zero_step_workspace_bytes.restype = ctypes.c_size_t
    L.zero_reduce_scatter_adam_step.argtypes = [
        ctypes.POINTER(vp), i32, i64, i32, ctypes.c_int,
        vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
        ctypes.POINTER(AdamHParams), f32, vp, vp, vp, vp]
    L.zero_reduce_scatter_adam_step.restype = ctypes.c_int
    L.zero_reduce_scatter_adam_step_noalloc.argtypes = [
        ctypes.POINTER(vp), i32, i64, i32, ctypes.c_int,
        vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
        ctypes.POINTER(AdamHParams), f32, vp, vp, vp]
    L.zero_reduce_scatter_adam_step_noalloc.restype = ctypes.c_int
    L.zero_step_static_scratch_bytes.argtypes = []
    L.zero_step_static_scratch_bytes.restype = ctypes.c_size_t
    L.zero_grad_stats.argtypes = [ctypes.POINTER(vp), i32, i64, i32, ctypes.c_int, f32, f32, vp, vp, vp, vp]
    L.zero_grad_stats.restype = ctypes.c_int
    L.zero_reduce_scatter_adam_step_gated.argtypes = [
        ctypes.POINTER(vp), i32, i64, i32, ctypes.c_int,
        vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
        ctypes.POINTER(AdamHParams), f32, vp, vp, vp, vp, vp, f32, vp]
    L.zero_reduce_scatter_adam_step_gated.restype = ctypes.c_int
    L.zero_reduce_scatter_grads.argtypes = [ctypes.POINTER(vp), i32, i64, i32, ctypes.c_int, f32, f32, vp, vp, vp,
                                            vp, vp]
    L.zero_reduce_scatter_grads.restype = ctypes.c_int
    L.zero_adam_step_reduced.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
                                         ctypes.POINTER(AdamHParams), vp, vp, vp, f32, vp]
    L.zero_adam_step_reduced.restype = ctypes.c_int
    L.zero_adam_step_reduced_bcast.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, ctypes.POINTER(vp), i32, ctypes.c_int,
                                               ctypes.POINTER(AdamHParams), vp, vp, vp, f32, vp]
    L.zero_adam_step_reduced_bcast.restype = ctypes.c_int
    L.zero_ipc_export.argtypes = [vp, ctypes.POINTER(IpcHandle), ctypes.POINTER(i64)]
    L.zero_ipc_export.restype = ctypes.c_int
    L.zero_ipc_import.argtypes = [ctypes.POINTER(IpcHandle), i64, ctypes.POINTER(vp), ctypes.POINTER(vp)]
    L.zero_ipc_import.restype = ctypes.c_int
    L.zero_ipc_close.argtypes = [vp]
    L.zero_ipc_close.restype = ctypes.c_int
    L.zero_runner_create.argtypes = [ctypes.POINTER(BucketBanks), i64, i32, ctypes.c_int, ctypes.c_int,
                                     ctypes.POINTER(AdamHParams), f32, i32, f32, vp, vp, vp, vp,
                                     ctypes.POINTER(vp)]
    L.zero_runner_create.restype = ctypes.c_int
    L.zero_runner_create_staged.argtypes = [ctypes.POINTER(BucketBanks), i64, i32, ctypes.c_int, ctypes.c_int,
                                            ctypes.POINTER(AdamHParams), f32, i32, f32, ctypes.POINTER(vp), f32,
                                            vp, vp, vp, vp, ctypes.POINTER(vp)]
    L.zero_runner_create_staged.restype = ctypes.c_int
    L.zero_runner_launch.argtypes = [vp, vp]
    L.zero_runner_launch.restype = ctypes.c_int
    L.zero_runner_commit.argtypes = [vp, vp, ctypes.POINTER(i32)]
    L.zero_runner_commit.restype = ctypes.c_int
    L.zero_runner_state.argtypes = [vp, ctypes.POINTER(i64), ctypes.POINTER(f32), ctypes.POINTER(i32),
                                    ctypes.POINTER(i32)]
    L.zero_runner_state.restype = ctypes.c_int
    L.zero_runner_set_state.argtypes = [vp, i64, f32, i32, i32]
    L.zero_runner_set_state.restype = ctypes.c_int
    L.zero_runner_destroy.argtypes = [vp]
    L.zero_runner_destroy.restype = None
    L.zero_runner_bucket_kernel.argtypes = [vp, i64, ctypes.POINTER(i32)]
    L.zero_runner_bucket_kernel.restype = ctypes.c_int
    L.zero_test_wait_timeout.argtypes = [vp, i64, vp]
    L.zero_test_wait_timeout.restype = ctypes.c_int
    L.zero_test_force_step_kernel.argtypes = [i32]
    L.zero_test_force_step_kernel.restype = ctypes.c_int
    L.zero_allgather_params.argtypes = [ctypes.POINTER(vp), i32, i64, i64, ctypes.c_int, vp, vp, vp]
    L.zero_allgather_params.restype = ctypes.c_int
    L.zero_loss_scale_update.argtypes = [ctypes.POINTER(f32), ctypes.POINTER(i32), i32, i32, f32]
    L.zero_loss_scale_update.restype = ctypes.c_int
    L.zero_strerror.argtypes = [ctypes.c_int]
    L.zero_strerror.restype = ctypes.c_char_p
    L.zero_last_error.argtypes = []
    L.zero_last_error.restype = ctypes.c_char_p
    L.zero_version.argtypes = []
    L.zero_version.restype = ctypes.c_char_p
    return L


lib = load_library()


def _check(rc: int) -> None:
    if rc != 0:
        raise ZeroError(rc, lib.zero_last_error().decode())


def _dtype_code(t) -> int:
    import torch
    m = {torch.float16: ZERO_F16, torch.bfloat16: ZERO_BF16, torch.float32: ZERO_F32}
    if t.dtype not in m:
        raise ZeroError(-3, f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _ptrs(ts) -> ctypes.Array:
    return (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])


_ELEM_BYTES = {ZERO_F16: 2, ZERO_BF16: 2, ZERO_F32: 4}


def _dev(t, n: int, name: str, dtype=None) -> int:
    """Address of a device argument after the checks the C ABI cannot make
    (it sees bare pointers): a CUDA tensor, contiguous, of `dtype` when
    given, holding at least `n` elements (of `dtype`, else of its own type).
    None passes as NULL (the C call decides whether NULL is allowed); a
    DevicePtr (another process's mapped buffer) is trusted as it is."""
    if t is None:
        return 0
    if isinstance(t, DevicePtr):
        return t.ptr
    if not getattr(t, "is_cuda", False):
        raise ZeroError(-1, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ZeroError(-1, f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ZeroError(-3, f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < n:
        raise ZeroError(-4, f"{name} holds {t.numel()} elements, the call needs {n}")
    return int(t.data_ptr())


def _devs(ts, n: int, name: str) -> ctypes.Array:
    return (ctypes.c_void_p * len(ts))(*[_dev(t, n, f"{name}[{k}]") for k, t in enumerate(ts)])


def _f32():
    import torch
    return torch.float32


def _count(padded_numel: int, world: int, partition: int) -> int:
    """Elements one call processes: the whole bucket, or one partition."""
    return padded_numel if partition == ZERO_ALL_PARTITIONS else padded_numel // max(1, world)


def _flag_args(overflow_flag, grad_sqnorm, workspace):
    import torch
    ws_bytes = zero_step_workspace_bytes() if grad_sqnorm is not None else 0
    if workspace is not None and not isinstance(workspace, DevicePtr) and \
            workspace.numel() * workspace.element_size() < ws_bytes:
        raise ZeroError(-4, f"workspace holds {workspace.numel() * workspace.element_size()} bytes, "
                            f"the norm needs {ws_bytes}")
    return (_dev(overflow_flag, 1, "overflow_flag", torch.int32), _dev(grad_sqnorm, 1, "grad_sqnorm", torch.float64),
            _dev(workspace, 0, "workspace"))


def _state_args(count, names_tensors):
    return [_dev(t, count, nm, _f32()) for nm, t in names_tensors]


# ---------------------------------------------------------------------------
# Layout
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Layout:
    """Host copy of a zero_layout_t (the C arrays are freed after copying)."""
    world: int
    align_elems: int
    bucket_numel: tuple
    bucket_padded: tuple
    bucket_offset: tuple
    bucket_first: tuple
    bucket_count: tuple
    tensor_numel: tuple
    tensor_bucket: tuple
    tensor_offset: tuple

    @property
    def n_buckets(self) -> int:
        return len(self.bucket_numel)

    def part(self, b: int) -> int:
        return self.bucket_padded[b] // self.world

    def _c(self) -> _Layout:
        def arr(x):
            return (ctypes.c_int64 * max(1, len(x)))(*x)
        c = _Layout()
        c.world, c.align_elems = self.world, self.align_elems
        c.n_tensors, c.n_buckets = len(self.tensor_numel), len(self.bucket_numel)
        keep = []
        for name in ("bucket_numel", "bucket_padded", "bucket_offset", "bucket_first", "bucket_count",
                     "tensor_numel", "tensor_bucket", "tensor_offset"):
            a = arr(getattr(self, name))
            keep.append(a)
            setattr(c, name, ctypes.cast(a, ctypes.POINTER(ctypes.c_int64)))
        c._keep = keep
        return c


def zero_partition_layout(numels, world: int, bucket_elems: int = 0, align_elems: int = 1) -> Layout:
    n = len(numels)
    arr = (ctypes.c_int64 * max(1, n))(*numels)
    out = _Layout()
    _check(lib.zero_partition_layout(arr, n, world, bucket_elems, align_elems, ctypes.byref(out)))
    try:
        nb, nt = out.n_buckets, out.n_tensors
        get = lambda p, k: tuple(p[i] for i in range(k))
        return Layout(out.world, out.align_elems,
                      get(out.bucket_numel, nb), get(out.bucket_padded, nb), get(out.bucket_offset, nb),
                      get(out.bucket_first, nb), get(out.bucket_count, nb),
                      get(out.tensor_numel, nt), get(out.tensor_bucket, nt), get(out.tensor_offset, nt))
    finally:
        lib.zero_layout_free(ctypes.byref(out))


# ---------------------------------------------------------------------------
# Device calls
# ---------------------------------------------------------------------------

def zero_flatten_bucket(layout: Layout, bucket: int, tensors, bucket_buf, stream=None) -> None:
    """Copy bucket `bucket`'s tensors (list indexed by tensor id) into bucket_buf."""
    if not 0 <= bucket < layout.n_buckets:
        raise ZeroError(-4, f"bucket {bucket} outside 0..{layout.n_buckets - 1}")
    if len(tensors) != len(layout.tensor_numel):
        raise ZeroError(-1, f"{len(tensors)} tensors given, the layout has {len(layout.tensor_numel)}")
    first, cnt = layout.bucket_first[bucket], layout.bucket_count[bucket]
    addrs = [0] * len(tensors)
    for i in range(first, first + cnt):
        addrs[i] = _dev(tensors[i], layout.tensor_numel[i], f"tensors[{i}]", bucket_buf.dtype)
    ptrs = (ctypes.c_void_p * max(1, len(tensors)))(*addrs)
    c = layout._c()
    _check(lib.zero_flatten_bucket(ctypes.byref(c), bucket, ptrs, _dtype_code(bucket_buf),
                                   _dev(bucket_buf, layout.bucket_padded[bucket], "bucket_buf"), _stream(stream)))


def zero_step_workspace_bytes() -> int:
    return int(lib.zero_step_workspace_bytes())


def hparams(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1,
            grad_divisor=0.0) -> AdamHParams:
    return AdamHParams(lr, beta1, beta2, eps, weight_decay, step, grad_divisor)


def zero_reduce_scatter_adam_step(grad_bufs, padded_numel: int, partition: int,
                                  master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                                  hp: AdamHParams, loss_scale: float, overflow_flag,
                                  grad_sqnorm=None, workspace=None, stream=None) -> None:
    """One fused reduce-scatter + Adam pass over one bucket (see include/zero.h)."""
    world = len(grad_bufs)
    n = _count(padded_numel, world, partition)
    st = _state_args(n, (("master_in", master_in), ("m_in", m_in), ("v_in", v_in), ("master_out", master_out),
                         ("m_out", m_out), ("v_out", v_out)))
    _check(lib.zero_reduce_scatter_adam_step(
        _devs(grad_bufs, padded_numel, "grad_bufs"), world, padded_numel, partition, _dtype_code(grad_bufs[0]),
        *st, _dev(param_out, n, "param_out"), _dtype_code(param_out), ctypes.byref(hp), float(loss_scale),
        *_flag_args(overflow_flag, grad_sqnorm, workspace), _stream(stream)))


def zero_reduce_scatter_adam_step_noalloc(grad_bufs, padded_numel: int, partition: int,
                                          master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                                          hp: AdamHParams, loss_scale: float, overflow_flag,
                                          grad_sqnorm=None, stream=None) -> None:
    """The fused step without a workspace argument, for callers that cannot
    allocate device memory: the norm's scratch lives in a fixed array inside
    libzero (see include/zero.h for its limits)."""
    world = len(grad_bufs)
    n = _count(padded_numel, world, partition)
    st = _state_args(n, (("master_in", master_in), ("m_in", m_in), ("v_in", v_in), ("master_out", master_out),
                         ("m_out", m_out), ("v_out", v_out)))
    flag, sq, _ = _flag_args(overflow_flag, grad_sqnorm, None)
    _check(lib.zero_reduce_scatter_adam_step_noalloc(
        _devs(grad_bufs, padded_numel, "grad_bufs"), world, padded_numel, partition, _dtype_code(grad_bufs[0]),
        *st, _dev(param_out, n, "param_out"), _dtype_code(param_out), ctypes.byref(hp), float(loss_scale),
        flag, sq, _stream(stream)))


def zero_grad_stats(grad_bufs, padded_numel: int, partition: int, loss_scale: float, overflow_flag,
                    grad_sqnorm=None, workspace=None, grad_divisor: float = 0.0, stream=None) -> None:
    """Overflow flag and squared norm of one bucket's reduced gradients (no update)."""
    _check(lib.zero_grad_stats(_devs(grad_bufs, padded_numel, "grad_bufs"), len(grad_bufs), padded_numel, partition,
                               _dtype_code(grad_bufs[0]), float(loss_scale), float(grad_divisor),
                               *_flag_args(overflow_flag, grad_sqnorm, workspace), _stream(stream)))


def zero_reduce_scatter_adam_step_gated(grad_bufs, padded_numel: int, partition: int,
                                        master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                                        hp: AdamHParams, loss_scale: float, overflow_flag,
                                        grad_sqnorm=None, workspace=None, gate=None, clip_sqnorm=None,
                                        max_norm: float = 0.0, stream=None) -> None:
    """The fused step, skipped entirely when *gate != 0, with optional clipping."""
    import torch
    world = len(grad_bufs)
    n = _count(padded_numel, world, partition)
    st = _state_args(n, (("master_in", master_in), ("m_in", m_in), ("v_in", v_in), ("master_out", master_out),
                         ("m_out", m_out), ("v_out", v_out)))
    _check(lib.zero_reduce_scatter_adam_step_gated(
        _devs(grad_bufs, padded_numel, "grad_bufs"), world, padded_numel, partition, _dtype_code(grad_bufs[0]),
        *st, _dev(param_out, n, "param_out"), _dtype_code(param_out), ctypes.byref(hp), float(loss_scale),
        *_flag_args(overflow_flag, grad_sqnorm, workspace), _dev(gate, 1, "gate", torch.int32),
        _dev(clip_sqnorm, 1, "clip_sqnorm", torch.float64), float(max_norm), _stream(stream)))


def zero_reduce_scatter_grads(grad_bufs, padded_numel: int, partition: int, loss_scale: float, reduced_out,
                              overflow_flag, grad_sqnorm=None, workspace=None, grad_divisor: float = 0.0,
                              stream=None) -> None:
    """Staged reduce-scatter: reduced_out = fp32 unscaled rank-order sums, plus flag and norm."""
    n = _count(padded_numel, len(grad_bufs), partition)
    _check(lib.zero_reduce_scatter_grads(_devs(grad_bufs, padded_numel, "grad_bufs"), len(grad_bufs), padded_numel,
                                         partition, _dtype_code(grad_bufs[0]), float(loss_scale), float(grad_divisor),
                                         _dev(reduced_out, n, "reduced_out", _f32()),
                                         *_flag_args(overflow_flag, grad_sqnorm, workspace), _stream(stream)))


def zero_adam_step_reduced(reduced_grad, count: int, master_in, m_in, v_in, master_out, m_out, v_out, param_out,
                           hp: AdamHParams, status, gate=None, clip_sqnorm=None, max_norm: float = 0.0,
                           stream=None) -> None:
    """Staged update: Adam on `count` elements from fp32 reduced gradients (gated, optionally clipped);
    `status` (device int32) receives bit 1 if the kernel's copy pipeline timed out."""
    import torch
    st = _state_args(count, (("reduced_grad", reduced_grad), ("master_in", master_in), ("m_in", m_in),
                             ("v_in", v_in), ("master_out", master_out), ("m_out", m_out), ("v_out", v_out)))
    _check(lib.zero_adam_step_reduced(
        st[0], count, *st[1:], _dev(param_out, count, "param_out"), _dtype_code(param_out), ctypes.byref(hp),
        _dev(status, 1, "status", torch.int32), _dev(gate, 1, "gate", torch.int32),
        _dev(clip_sqnorm, 1, "clip_sqnorm", torch.float64), float(max_norm), _stream(stream)))


def zero_adam_step_reduced_bcast(reduced_grad, count: int, master_in, m_in, v_in, master_out, m_out, v_out,
                                 param_dsts, hp: AdamHParams, status, gate=None, clip_sqnorm=None,
                                 max_norm: float = 0.0, stream=None) -> None:
    """zero_adam_step_reduced storing the updated parameters to every tensor
    (or mapped DevicePtr) in `param_dsts`: the all-gather done by the
    update's own stores."""
    import torch
    st = _state_args(count, (("reduced_grad", reduced_grad), ("master_in", master_in), ("m_in", m_in),
                             ("v_in", v_in), ("master_out", master_out), ("m_out", m_out), ("v_out", v_out)))
    dsts = _devs(param_dsts, count, "param_dsts")
    _check(lib.zero_adam_step_reduced_bcast(
        st[0], count, *st[1:], ctypes.cast(dsts, ctypes.POINTER(ctypes.c_void_p)), len(param_dsts),
        _dtype_code(param_dsts[0]), ctypes.byref(hp), _dev(status, 1, "status", torch.int32),
        _dev(gate, 1, "gate", torch.int32), _dev(clip_sqnorm, 1, "clip_sqnorm", torch.float64), float(max_norm),
        _stream(stream)))


def zero_allgather_params(shards, shard_offset: int, part_numel: int, dst, stream=None, status=None) -> None:
    """dst[r*part + j] = shards[r][shard_offset + j] (bit-exact copy); `status`
    (device int32, optional) receives 4 from the debug build when an index
    check fails."""
    import torch
    _check(lib.zero_allgather_params(_devs(shards, shard_offset + part_numel, "shards"), len(shards), shard_offset,
                                     part_numel, _dtype_code(dst), _dev(dst, len(shards) * part_numel, "dst"),
                                     _dev(status, 1, "status", torch.int32), _stream(stream)))


def zero_loss_scale_update(scale: float, good_steps: int, overflow: bool,
                           growth_interval: int = 1000, min_scale: float = 1.0):
    s = ctypes.c_float(scale)
    g = ctypes.c_int32(good_steps)
    _check(lib.zero_loss_scale_update(ctypes.byref(s), ctypes.byref(g), int(bool(overflow)),
                                      growth_interval, min_scale))
    return s.value, g.value


class Runner:
    """zero_runner_*: the step over every bucket in two C calls (launch, commit).

    `buckets`: list of (grad_bufs, [master0, master1], [m0, m1], [v0, v1],
    [params0, params1]) tensors; flag_dev a device int32 tensor, flag_host a
    pinned int32 tensor; the tensors must outlive the runner.

    With `reduced` (one fp32 tensor per bucket) the runner takes the staged
    route on bank 0 only (zero_runner_create_staged): flag_dev and flag_host
    then hold 2 words, bank 1 may be None, and max_norm > 0 clips.
    """

    def __init__(self, buckets, hp: AdamHParams, loss_scale: float, flag_dev, flag_host, grad_sqnorm=None,
                 workspace=None, growth_interval: int = 1000, min_scale: float = 1.0, reduced=None,
                 max_norm: float = 0.0):
        import torch
        staged = reduced is not None
        nbank = 1 if staged else 2
        descs = (BucketBanks * max(1, len(buckets)))()
        self._keep = []
        world = len(buckets[0][0]) if buckets else 1
        for i, (grads, master, m, v, params) in enumerate(buckets):
            n = grads[0].numel()
            arr = _devs(grads, n, f"bucket {i} grads")
            self._keep.append(arr)
            d = descs[i]
            d.padded_numel = n
            d.grad_bufs = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
            for b in range(nbank):
                d.master[b], d.m[b], d.v[b] = _state_args(n, ((f"bucket {i} master[{b}]", master[b]),
                                                              (f"bucket {i} m[{b}]", m[b]),
                                                              (f"bucket {i} v[{b}]", v[b])))
                d.params[b] = _dev(params[b], n, f"bucket {i} params[{b}]")
        gd = _dtype_code(buckets[0][0][0]) if buckets else ZERO_F16
        pd = _dtype_code(buckets[0][4][0]) if buckets else ZERO_F16
        words = 2 if staged else 1
        if getattr(flag_host, "is_cuda", True) or flag_host.dtype != torch.int32 or flag_host.numel() < words:
            raise ZeroError(-1, f"flag_host must be a host (pinned) int32 tensor of {words} word(s)")
        flag = _dev(flag_dev, words, "flag_dev", torch.int32)
        sq = _dev(grad_sqnorm, 1, "grad_sqnorm", torch.float64)
        ws = _flag_args(flag_dev, grad_sqnorm, workspace)[2]
        h = ctypes.c_void_p()
        if staged:
            red = (ctypes.c_void_p * max(1, len(buckets)))(
                *[_dev(reduced[i], buckets[i][0][0].numel(), f"reduced[{i}]", _f32()) for i in range(len(buckets))])
            self._keep.append(red)
            _check(lib.zero_runner_create_staged(descs, len(buckets), world, gd, pd, ctypes.byref(hp),
                                                 float(loss_scale), growth_interval, min_scale,
                                                 ctypes.cast(red, ctypes.POINTER(ctypes.c_void_p)), float(max_norm),
                                                 flag, _ptr(flag_host), sq, ws, ctypes.byref(h)))
        else:
            _check(lib.zero_runner_create(descs, len(buckets), world, gd, pd, ctypes.byref(hp), float(loss_scale),
                                          growth_interval, min_scale, flag, _ptr(flag_host), sq, ws,
                                          ctypes.byref(h)))
        self._h = h

    def launch(self, stream=None) -> None:
        _check(lib.zero_runner_launch(self._h, _stream(stream)))

    def commit(self, stream=None) -> bool:
        applied = ctypes.c_int32()
        _check(lib.zero_runner_commit(self._h, _stream(stream), ctypes.byref(applied)))
        return bool(applied.value)

    def state(self):
        t, s, g, b = ctypes.c_int64(), ctypes.c_float(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib.zero_runner_state(self._h, ctypes.byref(t), ctypes.byref(s), ctypes.byref(g), ctypes.byref(b)))
        return t.value, s.value, g.value, b.value

    def set_state(self, t: int, scale: float, good: int, bank: int) -> None:
        _check(lib.zero_runner_set_state(self._h, t, scale, good, bank))

    def bucket_kernel(self, bucket: int) -> int:
        """The fused-step kernel the next launch runs for `bucket`:
        STEP_KERNEL_REGISTER, STEP_KERNEL_PIPE, STEP_KERNEL_QUAD or STEP_KERNEL_OCT."""
        kind = ctypes.c_int32()
        _check(lib.zero_runner_bucket_kernel(self._h, bucket, ctypes.byref(kind)))
        return kind.value

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and lib is not None:
            try:
                lib.zero_runner_destroy(h)
            except Exception:      # interpreter shutdown: the library may be gone
                pass
            self._h = None


def zero_test_wait_timeout(status, limit_ns: int, stream=None) -> None:
    """Run the bounded-wait self-test: ORs 2 into status after ~limit_ns."""
    import torch
    _check(lib.zero_test_wait_timeout(_dev(status, 1, "status", torch.int32), int(limit_ns), _stream(stream)))


STEP_KERNEL_AUTO, STEP_KERNEL_REGISTER, STEP_KERNEL_PIPE, STEP_KERNEL_QUAD, STEP_KERNEL_OCT = -1, 0, 1, 2, 3


def zero_test_force_step_kernel(kind: int) -> None:
    """Test hook: make later fused-step calls of this process take `kind`
    (STEP_KERNEL_*) wherever that kernel can run the call; -1 restores the
    automatic choice."""
    _check(lib.zero_test_force_step_kernel(int(kind)))


def zero_ipc_export(tensor) -> tuple:
    """(handle bytes, byte offset) of a device buffer, for another process."""
    h = IpcHandle()
    off = ctypes.c_int64()
    _check(lib.zero_ipc_export(_dev(tensor, 0, "tensor"), ctypes.byref(h), ctypes.byref(off)))
    return bytes(h.bytes), int(off.value)


def zero_ipc_import(handle: bytes, offset: int) -> tuple:
    """Map another process's buffer: returns (device address, mapping base)."""
    h = IpcHandle()
    ctypes.memmove(h.bytes, handle, 64)
    ptr, base = ctypes.c_void_p(), ctypes.c_void_p()
    _check(lib.zero_ipc_import(ctypes.byref(h), int(offset), ctypes.byref(ptr), ctypes.byref(base)))
    return int(ptr.value), int(base.value)


def zero_ipc_close(base: int) -> None:
    _check(lib.zero_ipc_close(ctypes.c_void_p(base)))


def version() -> str:
    return lib.zero_version().decode()


from .optimizer import ZeroAdam  # noqa: E402  (uses the bindings above)
from .distributed import DistributedZeroAdam  # noqa: E402
from .stage3 import ZeroStage3  # noqa: E402
from .distributed_stage3 import DistributedZeroStage3  # noqa: E402
