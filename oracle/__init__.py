"""CPU oracle of the ZeRO-DP partitioned mixed-precision Adam step.

TEST INFRASTRUCTURE ONLY: imported by `tests/`, by `__graft_entry__.smoke()`
and by the CPU-baseline leg of `bench.py`, never by the product package.  It
shares no code with the CUDA path; the only module both sides use is
`workloads` (seeded inputs, no arithmetic of the method).

The floating-point steps live in `zero_oracle.c` (plain C, compiled with
-ffp-contract=off); the partition layout, the stage drivers, the loss-scale
rule and the memory / communication accounting are plain Python here.

Sources ("ZeRO explainer" is the azimuth.plus page "ZeRO: Memory
Optimizations Toward Training Trillion Parameter Models"):
  - model states 2+2+12 bytes per parameter: ZeRO explainer, model-states
    paragraph;
  - Stage 1 / 2 / 3 partitioning and their memory formulas: ZeRO explainer,
    "Stage 1 - Optimizer State Partitioning (P_os)", "Stage 2 - Gradient
    Partitioning (P_os+g)", "Stage 3 - Parameter Partitioning (P_os+g+p)";
  - fused constant-size buffers: ZeRO explainer, "Constant-size buffers";
  - communication volumes: ZeRO explainer, communication paragraphs
    (all-reduce 2 Psi per GPU; Stage 1/2 equal to it; Stage 3 about 1.5x).

Readings where the pages are silent (summation order, Adam formula, loss-scale
rule, padding, bucket packing) are stated at each function.

Parity status: every function here is pinned by a `-m "not gpu"` test against
a closed form, a library routine, brute force or an invariant; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
import tempfile

import numpy as np

F16, BF16 = "f16", "bf16"
_DT = {F16: 0, BF16: 1}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zero_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-fopenmp"]


def build(force: bool = False) -> str:
    """Compile the C part of the oracle (gcc) into oracle/liboracle.so."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=_HERE)
    os.close(fd)
    try:
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    finally:
        if os.path.exists(tmp):
            os.unlink(tmp)
    return _LIB


_lib = None


def load_library(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    L = ctypes.CDLL(path)
    i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_double
    vp = ctypes.c_void_p
    L.orc_f16_to_f32.restype = f32
    L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_f32.restype = f32
    L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_f32_to_f16.restype = ctypes.c_uint16
    L.orc_f32_to_f16.argtypes = [f32]
    L.orc_f32_to_bf16.restype = ctypes.c_uint16
    L.orc_f32_to_bf16.argtypes = [f32]
    for n in ("orc_f16_to_f32_array", "orc_bf16_to_f32_array",
              "orc_f32_to_f16_array", "orc_f32_to_bf16_array"):
        getattr(L, n).argtypes = [vp, vp, i64]
        getattr(L, n).restype = None
    L.orc_reduce.argtypes = [vp, i32, ctypes.c_int, i64, i64, vp]
    L.orc_reduce.restype = None
    L.orc_any_nonfinite.argtypes = [vp, i64]
    L.orc_any_nonfinite.restype = i32
    L.orc_grad_sqnorm.argtypes = [vp, i64, f32]
    L.orc_grad_sqnorm.restype = f64
    L.orc_unscale.argtypes = [vp, i64, f32, vp]
    L.orc_unscale.restype = None
    L.orc_adam_constants.argtypes = [f32, f32, f32, f32, f32, i64, f64, f32, vp]
    L.orc_adam_constants.restype = None
    L.orc_adam_update.argtypes = [vp, i64, vp, vp, vp, vp, vp, ctypes.c_int]
    L.orc_adam_update.restype = None
    L.orc_clip_coefficient.argtypes = [f64, f64]
    L.orc_clip_coefficient.restype = f32
    L.orc_adam_update_clipped.argtypes = [vp, i64, vp, f32, vp, vp, vp, vp, ctypes.c_int]
    L.orc_adam_update_clipped.restype = None
    L.orc_allgather.argtypes = [vp, i32, i64, i64, vp]
    L.orc_allgather.restype = None
    L.orc_threads.restype = i32
    L.orc_threads.argtypes = []
    L.orc_set_threads.restype = None
    L.orc_set_threads.argtypes = [i32]
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _ptr_array(arrs) -> ctypes.Array:
    return (ctypes.c_void_p * len(arrs))(*[_ptr(a) for a in arrs])


def threads() -> int:
    return int(lib().orc_threads())


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


# ---------------------------------------------------------------------------
# Storage formats
# ---------------------------------------------------------------------------

def to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, np.float32)
    fn = lib().orc_f16_to_f32_array if dtype == F16 else lib().orc_bf16_to_f32_array
    fn(_ptr(bits), _ptr(out), bits.size)
    return out


def from_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round-to-nearest-even to binary16 / bfloat16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    fn = lib().orc_f32_to_f16_array if dtype == F16 else lib().orc_f32_to_bf16_array
    fn(_ptr(x), _ptr(out), x.size)
    return out


# ---------------------------------------------------------------------------
# Layout: constant-size buffers and 1/N partitions
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Layout:
    world: int
    align_elems: int
    bucket_tensors: list          # tensor indices per bucket, in list order
    bucket_numel: list            # real elements per bucket
    bucket_padded: list           # padded to a multiple of world*align_elems
    bucket_offset: list           # bucket start in the flat concatenation of padded buckets
    tensor_bucket: list
    tensor_offset: list           # tensor start inside its bucket

    @property
    def n_buckets(self) -> int:
        return len(self.bucket_numel)

    def part(self, b: int) -> int:
        """P: elements of one rank's partition of bucket b."""
        return self.bucket_padded[b] // self.world

    @property
    def flat_numel(self) -> int:
        return sum(self.bucket_padded)

    def shard_offset(self, b: int) -> int:
        """Start of bucket b's slice inside a rank's concatenated shard."""
        return sum(self.part(c) for c in range(b))

    @property
    def shard_numel(self) -> int:
        return sum(self.part(b) for b in range(self.n_buckets))


def partition_layout(numels, world: int, bucket_elems: int = 0, align_elems: int = 1) -> Layout:
    """Pack tensors into constant-size buffers and split each into N partitions.

    Fused buffers of fixed capacity [ZeRO explainer, "Constant-size buffers"]:
    tensors are taken in list order and appended to the open bucket while it
    stays within `bucket_elems`; a tensor that does not fit closes the bucket
    and opens the next one; a tensor larger than the capacity gets a bucket of
    its own; no tensor is split.  `bucket_elems == 0` puts every tensor in one
    bucket.  Each bucket is padded with zeros to a multiple of
    N * align_elems, so that it splits into N equal partitions; partition r of
    a bucket is [r*P, (r+1)*P) with P = padded / N
    [ZeRO explainer, "Stage 1 - Optimizer State Partitioning (P_os)": each GPU
    stores 1/N of the optimizer states].
    """
    if world < 1 or align_elems < 1 or bucket_elems < 0:
        raise ValueError("world >= 1, align_elems >= 1, bucket_elems >= 0 required")
    buckets, cur, cur_n = [], [], 0
    for i, n in enumerate(numels):
        if n < 0:
            raise ValueError("negative tensor size")
        if cur and bucket_elems > 0 and cur_n + n > bucket_elems:
            buckets.append(cur)
            cur, cur_n = [], 0
        cur.append(i)
        cur_n += n
    if cur:
        buckets.append(cur)
    unit = world * align_elems
    b_numel, b_pad, b_off, t_bucket, t_off = [], [], [], [0] * len(numels), [0] * len(numels)
    flat = 0
    for b, idx in enumerate(buckets):
        off = 0
        for i in idx:
            t_bucket[i] = b
            t_off[i] = off
            off += numels[i]
        b_numel.append(off)
        pad = -(-off // unit) * unit
        b_pad.append(pad)
        b_off.append(flat)
        flat += pad
    return Layout(world, align_elems, buckets, b_numel, b_pad, b_off, t_bucket, t_off)


def flatten_bucket(layout: Layout, b: int, tensors, dtype=np.uint16) -> np.ndarray:
    """Copy bucket b's tensors to their offsets in one buffer; zero the padding."""
    out = np.zeros(layout.bucket_padded[b], dtype=dtype)
    for i in layout.bucket_tensors[b]:
        t = np.asarray(tensors[i]).reshape(-1)
        o = layout.tensor_offset[i]
        out[o:o + t.size] = t
    return out


def partitions(buf: np.ndarray, world: int) -> list:
    """The N rank-major partitions of a padded buffer (views)."""
    P = buf.size // world
    return [buf[r * P:(r + 1) * P] for r in range(world)]


# ---------------------------------------------------------------------------
# Collective and update primitives (the C part)
# ---------------------------------------------------------------------------

def reduce(grads, dtype: str = F16, begin: int = 0, count: int | None = None) -> np.ndarray:
    """fp32 rank-order sum over replicas of G_k[begin:begin+count].

    Whole buffer: the all-reduce of plain data parallelism.  One partition:
    that rank's share of a reduce-scatter [ZeRO explainer, "Stage 2 - Gradient
    Partitioning (P_os+g)"].
    """
    grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
    if count is None:
        count = grads[0].size - begin
    if begin < 0 or count < 0 or any(begin + count > g.size for g in grads):
        raise ValueError("range outside a gradient buffer")
    s = np.empty(count, np.float32)
    lib().orc_reduce(_ptr_array(grads), len(grads), _DT[dtype], begin, count, _ptr(s))
    return s


def any_nonfinite(s: np.ndarray) -> int:
    s = np.ascontiguousarray(s, dtype=np.float32)
    return int(lib().orc_any_nonfinite(_ptr(s), s.size))


def grad_sqnorm(s: np.ndarray, inv: float) -> float:
    s = np.ascontiguousarray(s, dtype=np.float32)
    return float(lib().orc_grad_sqnorm(_ptr(s), s.size, float(inv)))


def unscale(s: np.ndarray, inv: float) -> np.ndarray:
    """The reduced, unscaled fp32 gradient g = s * inv of a rank's partition."""
    s = np.ascontiguousarray(s, dtype=np.float32)
    g = np.empty_like(s)
    lib().orc_unscale(_ptr(s), s.size, float(inv), _ptr(g))
    return g


def adam_constants(adam, t: int, divisor: float, loss_scale: float) -> np.ndarray:
    """[lr, b1, b2, eps, inv, 1-b1, 1-b2, 1/(1-b1^t), 1/sqrt(1-b2^t), 1-lr*wd] in fp32."""
    c = np.empty(10, np.float32)
    lib().orc_adam_constants(adam.lr, adam.beta1, adam.beta2, adam.eps, adam.weight_decay,
                             int(t), float(divisor), float(loss_scale), _ptr(c))
    return c


def adam_update(s, consts, master, m, v, p16, pdtype: str = F16) -> None:
    """In-place Adam/AdamW update of one partition (formula in zero_oracle.c)."""
    for a in (master, m, v):
        assert a.dtype == np.float32 and a.flags["C_CONTIGUOUS"] and a.size == s.size
    assert p16.dtype == np.uint16 and p16.size == s.size and p16.flags["C_CONTIGUOUS"]
    s = np.ascontiguousarray(s, dtype=np.float32)
    lib().orc_adam_update(_ptr(s), s.size, _ptr(consts), _ptr(master), _ptr(m), _ptr(v),
                          _ptr(p16), _DT[pdtype])


def clip_coefficient(total_sqnorm: float, max_norm: float) -> np.float32:
    """Global-norm clipping factor min(1, max_norm / (sqrt(total) + 1e-6)).

    Not on the pages (the usual rule of clipping by the global norm); the
    coefficient is computed in double and rounded once to float.
    """
    return np.float32(lib().orc_clip_coefficient(float(total_sqnorm), float(max_norm)))


def adam_update_clipped(s, consts, clip, master, m, v, p16, pdtype: str = F16) -> None:
    """adam_update with g = (s * inv) * clip."""
    for a in (master, m, v):
        assert a.dtype == np.float32 and a.flags["C_CONTIGUOUS"] and a.size == s.size
    assert p16.dtype == np.uint16 and p16.size == s.size and p16.flags["C_CONTIGUOUS"]
    s = np.ascontiguousarray(s, dtype=np.float32)
    lib().orc_adam_update_clipped(_ptr(s), s.size, _ptr(consts), float(clip), _ptr(master), _ptr(m), _ptr(v),
                                  _ptr(p16), _DT[pdtype])


def allgather(shards, offset: int, part: int) -> np.ndarray:
    """Concatenate shards[r][offset:offset+part] in rank order."""
    shards = [np.ascontiguousarray(x, dtype=np.uint16) for x in shards]
    if any(offset + part > x.size for x in shards):
        raise ValueError("range outside a shard")
    out = np.empty(len(shards) * part, np.uint16)
    lib().orc_allgather(_ptr_array(shards), len(shards), offset, part, _ptr(out))
    return out


# ---------------------------------------------------------------------------
# Dynamic loss scale
# ---------------------------------------------------------------------------

def loss_scale_update(scale: float, good_steps: int, overflow: bool,
                      growth_interval: int = 1000, min_scale: float = 1.0):
    """Dynamic loss scaling (not on the pages; the usual rule).

    Overflow: the update is skipped, the scale halves (not below min_scale)
    and the good-step counter restarts.  Otherwise the counter grows and the
    scale doubles after `growth_interval` consecutive good steps, unless the
    doubled fp32 scale would be infinite.
    """
    if overflow:
        return max(scale / 2.0, min_scale), 0
    good_steps += 1
    if good_steps >= growth_interval:
        twice = scale * 2.0
        fits = twice <= float(np.finfo(np.float32).max)   # the scale is an fp32 value
        return (twice if fits else scale), 0
    return scale, good_steps


# ---------------------------------------------------------------------------
# Accounting [ZeRO explainer: model-states paragraph, Stages 1-3,
# communication paragraphs]
# ---------------------------------------------------------------------------

def model_state_bytes(stage: int, layout: Layout, grad_bytes: int = 2,
                      param_bytes: int = 2, opt_bytes: int = 12) -> int:
    """Bytes of model states one rank holds, counted from the layout.

    stage 0: plain data parallelism, everything replicated (16 Psi).
    stage 1: optimizer states partitioned (4 Psi + 12 Psi / N).
    stage 2: gradients too ((2 + 14 / N) Psi).
    stage 3: parameters too (16 Psi / N).
    Psi here is the padded flat size; P = Psi_padded / N per bucket.
    """
    full = layout.flat_numel
    part = layout.shard_numel
    p = full if stage < 3 else part
    g = full if stage < 2 else part
    o = full if stage < 1 else part
    return param_bytes * p + grad_bytes * g + opt_bytes * o


def comm_elements(stage: int, layout: Layout) -> int:
    """Elements one rank sends per step with ring collectives.

    A ring all-reduce sends 2 (N-1) P elements per rank (2 Psi as N grows);
    a reduce-scatter or an all-gather sends (N-1) P.
    stage 0: all-reduce.  stage 1 / 2: reduce-scatter + all-gather of the
    updated parameters.  stage 3: all-gather before forward, all-gather before
    backward, reduce-scatter; no all-gather after the update, since each rank
    keeps only its own shard.
    """
    n = layout.world
    rs = ag = (n - 1) * layout.shard_numel
    if stage == 0:
        return 2 * rs
    if stage in (1, 2):
        return rs + ag
    if stage == 3:
        return ag + ag + rs
    raise ValueError(stage)


# ---------------------------------------------------------------------------
# Stage drivers
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class FlatState:
    """Model states of one bucket in flat (rank-major) order."""
    master: np.ndarray
    m: np.ndarray
    v: np.ndarray
    params: np.ndarray   # uint16 bits

    def copy(self) -> "FlatState":
        return FlatState(self.master.copy(), self.m.copy(), self.v.copy(), self.params.copy())


def initial_state(master_f32: np.ndarray, pdtype: str = F16) -> FlatState:
    """Adam states at t = 0: m = v = 0; parameters = rounded master."""
    master_f32 = np.ascontiguousarray(master_f32, dtype=np.float32)
    return FlatState(master_f32.copy(), np.zeros_like(master_f32), np.zeros_like(master_f32),
                     from_f32(master_f32, pdtype))


@dataclasses.dataclass
class Scaler:
    scale: float
    good_steps: int = 0
    t: int = 0                   # applied updates so far
    growth_interval: int = 1000
    min_scale: float = 1.0


class StageRun:
    """One ZeRO-DP stage run by N simulated ranks on the host.

    stage 0: plain data parallelism: every rank all-reduces the gradients and
             updates a full replica of all states.
    stage 1: every rank all-reduces (the Stage 1 paragraph says gradients are
             "reduced as usual with all-reduce"), updates only its partition of
             the optimizer states, then all-gathers the updated parameters.
    stage 2: reduce-scatter: each rank reduces only its own slice, updates it,
             then all-gathers the parameters.
    stage 3: each rank keeps only its parameter shard; full parameters are
             gathered before forward and before backward and dropped; no
             gather follows the update.
    The overflow decision is shared by every rank (OR over ranks), so all
    ranks skip together; t counts applied updates only.
    """

    def __init__(self, stage: int, layout: Layout, init_master, adam, scaler: Scaler,
                 gdtype: str = F16, pdtype: str = F16, divisor: float | None = None):
        self.stage, self.layout, self.adam, self.scaler = stage, layout, adam, scaler
        self.gdtype, self.pdtype = gdtype, pdtype
        N = layout.world
        self.divisor = float(N if divisor is None else divisor)
        self.ranks = []
        for r in range(N):
            per_bucket = []
            for b in range(layout.n_buckets):
                full = initial_state(init_master[b], pdtype)
                P = layout.part(b)
                sl = slice(r * P, (r + 1) * P)
                if stage == 0:
                    st = full
                elif stage in (1, 2):
                    st = FlatState(full.master[sl].copy(), full.m[sl].copy(), full.v[sl].copy(),
                                   full.params)          # params stay replicated
                else:
                    st = FlatState(full.master[sl].copy(), full.m[sl].copy(), full.v[sl].copy(),
                                   full.params[sl].copy())  # only the own shard
                per_bucket.append(st)
            self.ranks.append(per_bucket)
        self.gathers = 0

    def step(self, grads) -> int:
        """grads[b][k]: replica k's padded gradient bucket b (uint16 bits)."""
        L, N, sc = self.layout, self.layout.world, self.scaler
        sums = []                                     # sums[r][b]
        for r in range(N):
            per_b = []
            for b in range(L.n_buckets):
                P = L.part(b)
                if self.stage == 3:
                    # forward and backward each gather the bucket's full parameters
                    for _ in range(2):
                        full = allgather([self.ranks[q][b].params for q in range(N)], 0, P)
                        assert full.size == L.bucket_padded[b]
                        self.gathers += 1
                if self.stage in (0, 1):
                    per_b.append(reduce(grads[b], self.gdtype))
                else:
                    per_b.append(reduce(grads[b], self.gdtype, r * P, P))
            sums.append(per_b)
        overflow = int(any(any_nonfinite(s) for per_b in sums for s in per_b))
        if not overflow:
            t = sc.t + 1
            c = adam_constants(self.adam, t, self.divisor, sc.scale)
            for r in range(N):
                for b in range(L.n_buckets):
                    P = L.part(b)
                    st = self.ranks[r][b]
                    s = sums[r][b]
                    if self.stage == 0:
                        adam_update(s, c, st.master, st.m, st.v, st.params, self.pdtype)
                    elif self.stage == 1:
                        own = np.empty(P, np.uint16)
                        adam_update(np.ascontiguousarray(s[r * P:(r + 1) * P]), c,
                                    st.master, st.m, st.v, own, self.pdtype)
                        st.pending = own
                    elif self.stage == 2:
                        own = np.empty(P, np.uint16)
                        adam_update(s, c, st.master, st.m, st.v, own, self.pdtype)
                        st.pending = own
                    else:
                        adam_update(s, c, st.master, st.m, st.v, st.params, self.pdtype)
            if self.stage in (1, 2):
                # all-gather of the updated parameter shards into every replica
                for b in range(L.n_buckets):
                    P = L.part(b)
                    gathered = allgather([self.ranks[q][b].pending for q in range(N)], 0, P)
                    for r in range(N):
                        self.ranks[r][b].params = gathered.copy()
            sc.t = t
        sc.scale, sc.good_steps = loss_scale_update(sc.scale, sc.good_steps, bool(overflow),
                                                    sc.growth_interval, sc.min_scale)
        return overflow

    def flat_state(self, b: int) -> FlatState:
        """Bucket b's states in flat order (concatenated partitions)."""
        N = self.layout.world
        if self.stage == 0:
            return self.ranks[0][b].copy()
        cat = lambda name: np.concatenate([getattr(self.ranks[r][b], name) for r in range(N)])
        params = self.ranks[0][b].params.copy() if self.stage in (1, 2) else cat("params")
        return FlatState(cat("master"), cat("m"), cat("v"), params)

    def replicas_identical(self) -> bool:
        """Replicated arrays agree on every rank (stage 0: all states; 1/2: params)."""
        N = self.layout.world
        for b in range(self.layout.n_buckets):
            ref = self.ranks[0][b]
            for r in range(1, N):
                o = self.ranks[r][b]
                if self.stage == 0:
                    for name in ("master", "m", "v", "params"):
                        if not np.array_equal(getattr(ref, name).view(np.uint32 if name != "params" else np.uint16),
                                              getattr(o, name).view(np.uint32 if name != "params" else np.uint16)):
                            return False
                elif self.stage in (1, 2):
                    if not np.array_equal(ref.params, o.params):
                        return False
        return True


def flat_step(grads, state: FlatState, adam, t: int, loss_scale: float, divisor: float,
              gdtype: str = F16, pdtype: str = F16, begin: int = 0, count: int | None = None,
              apply: bool = True):
    """One step over elements [begin, begin+count) of a flat bucket.

    Reduce (rank order) -> overflow test -> Adam on the range, in place on
    `state` (whose arrays cover exactly the range).  Returns (overflow of the
    range, grad square-norm of the range).  With apply=False the state is not
    touched (a skipped step).
    """
    s = reduce(grads, gdtype, begin, count)
    ovf = any_nonfinite(s)
    c = adam_constants(adam, t, divisor, loss_scale)
    sq = grad_sqnorm(s, c[4]) if not ovf else float("nan")
    if apply and not ovf:
        adam_update(s, c, state.master, state.m, state.v, state.params, pdtype)
    return ovf, sq
