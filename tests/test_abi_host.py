"""The C ABI without a GPU: exported symbols, host-only calls, validation.

- every function declared in include/zero.h is exported by libzero.so;
- zero_partition_layout equals the oracle's layout bit for bit;
- zero_loss_scale_update follows the oracle's rule;
- every device call rejects bad arguments with its error code before it
  touches CUDA (so these run on a machine without a GPU).
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "zero.h")


def _declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zero_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(Z.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_library_reports_version_and_errors():
    assert "sm_100a" in Z.version()
    assert Z.lib.zero_strerror(0) == b"ok"
    assert Z.lib.zero_strerror(-2) == b"misaligned pointer"


@pytest.mark.parametrize("world", [1, 3, 4, 8])
@pytest.mark.parametrize("cap", [0, 7, 50])
@pytest.mark.parametrize("align", [1, 8])
def test_layout_equals_oracle(world, cap, align):
    rng = np.random.Generator(np.random.PCG64(world * 31 + cap + align))
    for _ in range(6):
        numels = rng.integers(0, 40, rng.integers(0, 15)).tolist()
        a = Z.zero_partition_layout(numels, world, cap, align)
        b = oracle.partition_layout(numels, world, cap, align)
        assert list(a.bucket_numel) == b.bucket_numel
        assert list(a.bucket_padded) == b.bucket_padded
        assert list(a.bucket_offset) == b.bucket_offset
        assert list(a.tensor_bucket) == b.tensor_bucket
        assert list(a.tensor_offset) == b.tensor_offset
        assert [list(range(f, f + c)) for f, c in zip(a.bucket_first, a.bucket_count)] == b.bucket_tensors


def test_layout_gpt2_and_6p7b():
    numels = workloads.gpt2_1p5b_tensor_numels()
    a = Z.zero_partition_layout(numels, 8, 500_000_000)
    assert list(a.bucket_padded) == oracle.partition_layout(numels, 8, 500_000_000).bucket_padded
    units = workloads.gpt_6p7b_unit_numels()
    a = Z.zero_partition_layout(units, 8, 1)
    assert a.n_buckets == 33 and a.part(0) == 25_172_480


def test_layout_errors():
    for args in [([3], 0, 0, 1), ([3], 129, 0, 1), ([3], 2, -1, 1), ([3], 2, 0, 0), ([-3], 2, 0, 1)]:
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_partition_layout(*args)
        assert e.value.code == -1
    out = Z._Layout()
    assert Z.lib.zero_partition_layout(None, 1, 2, 0, 1, ctypes.byref(out)) == -1
    assert Z.lib.zero_partition_layout(None, 0, 2, 0, 1, None) == -1
    # an empty list is a valid, empty layout
    assert Z.zero_partition_layout([], 4).n_buckets == 0


def test_loss_scale_matches_oracle():
    rng = np.random.Generator(np.random.PCG64(3))
    s, g = 65536.0, 0
    so, go = s, g
    for _ in range(200):
        ovf = bool(rng.random() < 0.2)
        s, g = Z.zero_loss_scale_update(s, g, ovf, growth_interval=5, min_scale=1.0)
        so, go = oracle.loss_scale_update(so, go, ovf, growth_interval=5, min_scale=1.0)
        assert (s, g) == (so, go)
    with pytest.raises(Z.ZeroError):
        Z.zero_loss_scale_update(1.0, 0, False, growth_interval=0)
    with pytest.raises(Z.ZeroError):
        Z.zero_loss_scale_update(-1.0, 0, False)


# ------------------------------------------------------------- validation

def _step_call(**kw):
    """Raw call with fake (never dereferenced) pointers; returns the code."""
    L = Z.lib
    world = kw.get("world", 2)
    grads = kw.get("grads", [0x10000 * (k + 1) for k in range(world)])
    g = None if grads is None else (ctypes.c_void_p * max(1, len(grads)))(*grads)
    hp = kw.get("hp", Z.hparams())
    base = 0x7000_0000
    f = lambda i: kw.get(f"p{i}", base + 0x100_0000 * i)
    return L.zero_reduce_scatter_adam_step(
        g, world, kw.get("n", 64), kw.get("part", -1), kw.get("gd", 0),
        f(1), f(2), f(3), f(4), f(5), f(6), f(7), kw.get("pd", 0),
        None if hp is None else ctypes.byref(hp), kw.get("scale", 1024.0),
        kw.get("flag", base + 0x100_0000 * 9), kw.get("norm", None), kw.get("ws", None), None)


@pytest.mark.parametrize("kw,code", [
    (dict(grads=None), -1),
    (dict(hp=None), -1),
    (dict(flag=0), -1),
    (dict(world=0, grads=[]), -1),
    (dict(world=129, grads=[0x10000] * 129), -1),
    (dict(n=63), -1),
    (dict(n=-2), -1),
    (dict(part=2), -4),
    (dict(part=-2), -4),
    (dict(gd=2), -3),
    (dict(pd=7), -3),
    (dict(hp=Z.hparams(step=0)), -1),
    (dict(hp=Z.hparams(beta1=1.0)), -1),
    (dict(hp=Z.hparams(beta2=-0.1)), -1),
    (dict(hp=Z.hparams(lr=float("nan"))), -1),
    (dict(scale=0.0), -1),
    (dict(scale=float("inf")), -1),
    (dict(norm=0x7F00_0000), -1),                 # norm without workspace
    (dict(flag=0x7000_0002), -2),                  # misaligned flag
    (dict(p1=0), -1),                              # NULL master_in
    (dict(p7=0), -1),                              # NULL param_out
    (dict(p1=0x7000_0002), -2),                    # master_in not 4-byte aligned
    (dict(p7=0x7700_0001), -2),                    # param_out not 2-byte aligned
    (dict(grads=[0x10000, 0]), -1),                # NULL replica
    (dict(grads=[0x10000, 0x10001]), -2),          # misaligned replica
    (dict(p4=0x7200_0000 + 8), -1),                # master_out overlaps m_in
    (dict(p5=0x7400_0000 + 64), -1),              # m_out overlaps master_out
    (dict(p7=0x10000 + 16), -1),                   # param_out overlaps a gradient buffer
])
def test_step_rejects_bad_arguments(kw, code):
    assert _step_call(**kw) == code
    assert Z.lib.zero_last_error() != b""


def test_step_with_nothing_to_do_is_ok():
    assert _step_call(n=0) == 0


def _reduced_call(**kw):
    """zero_adam_step_reduced with fake (never dereferenced) pointers."""
    base = 0x7000_0000
    f = lambda i: kw.get(f"p{i}", base + 0x100_0000 * i)
    hp = kw.get("hp", Z.hparams())
    return Z.lib.zero_adam_step_reduced(
        kw.get("red", base + 0x100_0000 * 12), kw.get("n", 64), f(1), f(2), f(3), f(4), f(5), f(6), f(7),
        kw.get("pd", 0), None if hp is None else ctypes.byref(hp), kw.get("status", base + 0x100_0000 * 13),
        kw.get("gate", None), kw.get("clip", None), kw.get("max_norm", 0.0), None)


@pytest.mark.parametrize("kw,code", [
    (dict(hp=None), -1),
    (dict(n=-1), -1),
    (dict(pd=2), -3),
    (dict(hp=Z.hparams(step=0)), -1),
    (dict(red=0), -1),                              # NULL reduced gradient
    (dict(red=0x7C00_0002), -2),                    # reduced gradient not 4-byte aligned
    (dict(p2=0), -1),                               # NULL m_in
    (dict(p6=0x7600_0002), -2),                     # v_out misaligned
    (dict(p7=0x7700_0001), -2),                     # param_out misaligned
    (dict(red=0x7400_0000 + 4), -1),                # reduced gradient overlaps master_out
    (dict(p5=0x7100_0000), -1),                     # m_out is master_in
    (dict(gate=0x7D00_0002), -2),                   # misaligned gate
    (dict(clip=0x7E00_0000, max_norm=0.0), -1),     # clipping without a positive max_norm
    (dict(status=0), -1),                           # NULL status
    (dict(status=0x7D00_0001), -2),                 # misaligned status
    (dict(gate=0x7D00_0000, status=0x7D00_0000), -1),   # gate is the status word
])
def test_reduced_update_rejects_bad_arguments(kw, code):
    assert _reduced_call(**kw) == code
    assert Z.lib.zero_last_error() != b""


def test_reduced_update_with_nothing_to_do_is_ok():
    assert _reduced_call(n=0) == 0


def test_staged_reduce_scatter_rejects_bad_arguments():
    L = Z.lib
    g = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    flag = 0x7000_0000
    assert L.zero_reduce_scatter_grads(g, 2, 64, -1, 0, 1.0, 0.0, None, flag, None, None, None) == -1
    assert L.zero_reduce_scatter_grads(g, 2, 64, -1, 0, 1.0, 0.0, 0x30002, flag, None, None, None) == -2
    assert L.zero_reduce_scatter_grads(g, 2, 64, -1, 0, 1.0, 0.0, 0x10040, flag, None, None, None) == -1
    assert L.zero_reduce_scatter_grads(g, 2, 63, -1, 0, 1.0, 0.0, 0x30000, flag, None, None, None) == -1
    assert L.zero_reduce_scatter_grads(g, 2, 64, 3, 0, 1.0, 0.0, 0x30000, flag, None, None, None) == -4
    assert L.zero_reduce_scatter_grads(g, 2, 64, -1, 2, 1.0, 0.0, 0x30000, flag, None, None, None) == -3
    assert L.zero_reduce_scatter_grads(g, 2, 0, -1, 0, 1.0, 0.0, 0x30000, flag, None, None, None) == 0


def test_allgather_and_flatten_reject_bad_arguments():
    L = Z.lib
    sh = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    assert L.zero_allgather_params(None, 2, 0, 8, 0, 0x30000, None, None) == -1
    assert L.zero_allgather_params(sh, 0, 0, 8, 0, 0x30000, None, None) == -1
    assert L.zero_allgather_params(sh, 2, -1, 8, 0, 0x30000, None, None) == -1
    assert L.zero_allgather_params(sh, 2, 0, 8, 9, 0x30000, None, None) == -3
    assert L.zero_allgather_params(sh, 2, 0, 8, 2, 0x30002, None, None) == -2
    assert L.zero_allgather_params(sh, 2, 0, 8, 0, 0x10008, None, None) == -1   # dst overlaps shard 0
    bad = (ctypes.c_void_p * 2)(0x10001, 0x20000)
    assert L.zero_allgather_params(bad, 2, 0, 8, 0, 0x30000, None, None) == -2
    assert L.zero_allgather_params(sh, 2, 0, 8, 0, 0x30000, 0x40002, None) == -2   # status misaligned
    assert L.zero_allgather_params(sh, 2, 0, 8, 0, 0x30000, 0x30004, None) == -1   # status inside dst
    assert L.zero_allgather_params(sh, 2, 0, 0, 0, 0x30000, None, None) == 0     # nothing to copy
    lay = Z.zero_partition_layout([5, 7], 2)._c()
    tp = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    assert L.zero_flatten_bucket(None, 0, tp, 0, 0x30000, None) == -1
    assert L.zero_flatten_bucket(ctypes.byref(lay), 1, tp, 0, 0x30000, None) == -4
    assert L.zero_flatten_bucket(ctypes.byref(lay), 0, tp, 5, 0x30000, None) == -3
    assert L.zero_flatten_bucket(ctypes.byref(lay), 0, tp, 2, 0x30002, None) == -2
    assert L.zero_flatten_bucket(ctypes.byref(lay), 0, tp, 0, 0x10004, None) == -1


def test_wait_timeout_rejects_bad_arguments():
    assert Z.lib.zero_test_wait_timeout(None, 1000, None) == -1
    assert Z.lib.zero_test_wait_timeout(0x10002, 1000, None) == -2
    assert Z.lib.zero_test_wait_timeout(0x10000, -1, None) == -1


def test_loss_scale_growth_stops_below_inf():
    big = float(np.float32(3.0e38))
    s, g = Z.zero_loss_scale_update(big, 0, False, growth_interval=1)
    so, go = oracle.loss_scale_update(big, 0, False, growth_interval=1)
    assert (s, g) == (so, go) == (big, 0)


C_PROGRAM = r"""
#include <stdio.h>
#include "zero.h"
int main(void) {
    int64_t numels[3] = {5, 7, 11};
    zero_layout_t L = {0};
    if (zero_partition_layout(numels, 3, 4, 10, 1, &L) != ZERO_OK) return 1;
    printf("%lld %lld %lld\n", (long long)L.n_buckets, (long long)L.bucket_padded[0], (long long)L.bucket_padded[1]);
    zero_layout_free(&L);
    float scale = 8.0f; int32_t good = 0;
    if (zero_loss_scale_update(&scale, &good, 1, 1000, 1.0f) != ZERO_OK || scale != 4.0f) return 2;
    if (zero_reduce_scatter_adam_step(NULL, 2, 64, ZERO_ALL_PARTITIONS, ZERO_F16, NULL, NULL, NULL, NULL, NULL,
                                      NULL, NULL, ZERO_F16, NULL, 1.0f, NULL, NULL, NULL, NULL) != ZERO_ERR_ARG) return 3;
    printf("%s|%s\n", zero_strerror(ZERO_ERR_ARG), zero_last_error());
    return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    src = tmp_path / "use_zero.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_zero"
    inc = os.path.join(os.path.dirname(HEADER))
    libdir = os.path.dirname(Z.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe),
                           "-L", libdir, "-lzero", f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    lines = out.stdout.splitlines()
    assert lines[0] == "3 8 8"          # buckets [5], [7], [11] padded to multiples of 4
    assert lines[1].startswith("invalid argument|zero_reduce_scatter_adam_step")


class _FakeCuda:
    """Stands in for a CUDA tensor in the binding's checks (nothing is launched:
    every case below fails before the C call)."""

    def __init__(self, n, dtype, cuda=True, contiguous=True, ptr=0x7000_0000):
        self.n, self.dtype, self.is_cuda, self._contig, self.ptr = n, dtype, cuda, contiguous, ptr

    def numel(self):
        return self.n

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()

    def is_contiguous(self):
        return self._contig

    def data_ptr(self):
        return self.ptr


def _fake_step(**over):
    f32, f16 = torch.float32, torch.float16
    n, world = 64, 2
    args = dict(grad_bufs=[_FakeCuda(n, f16), _FakeCuda(n, f16)], padded_numel=n, partition=-1,
                master_in=_FakeCuda(n, f32), m_in=_FakeCuda(n, f32), v_in=_FakeCuda(n, f32),
                master_out=_FakeCuda(n, f32), m_out=_FakeCuda(n, f32), v_out=_FakeCuda(n, f32),
                param_out=_FakeCuda(n, f16), hp=Z.hparams(), loss_scale=1024.0,
                overflow_flag=_FakeCuda(1, torch.int32))
    args.update(over)
    Z.zero_reduce_scatter_adam_step(**args, stream=0)


@pytest.mark.parametrize("over,code", [
    (dict(master_in=_FakeCuda(64, torch.float32, cuda=False)), -1),         # host tensor
    (dict(m_out=_FakeCuda(64, torch.float32, contiguous=False)), -1),       # strided view
    (dict(v_in=_FakeCuda(64, torch.float16)), -3),                           # wrong dtype
    (dict(master_out=_FakeCuda(63, torch.float32)), -4),                     # too small
    (dict(param_out=_FakeCuda(10, torch.float16)), -4),
    (dict(grad_bufs=[_FakeCuda(64, torch.float16), _FakeCuda(32, torch.float16)]), -4),
    (dict(overflow_flag=_FakeCuda(1, torch.float32)), -3),
    (dict(overflow_flag=_FakeCuda(1, torch.int32, cuda=False)), -1),
])
def test_binding_checks_tensors_before_the_call(over, code):
    with pytest.raises(Z.ZeroError) as e:
        _fake_step(**over)
    assert e.value.code == code


def test_binding_partition_sizes_and_staged_checks():
    f32 = torch.float32
    # one partition needs only P = 32 elements of state
    small = {k: _FakeCuda(31, f32) for k in ("master_in",)}
    with pytest.raises(Z.ZeroError) as e:
        _fake_step(partition=1, **small)
    assert e.value.code == -4
    # staged update: the reduced gradient must be fp32 and large enough
    st = [_FakeCuda(64, f32) for _ in range(6)]
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_adam_step_reduced(_FakeCuda(63, f32), 64, *st, _FakeCuda(64, torch.float16), Z.hparams(),
                                 _FakeCuda(1, torch.int32), stream=0)
    assert e.value.code == -4
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_reduce_scatter_grads([_FakeCuda(64, torch.float16)] * 2, 64, -1, 1.0, _FakeCuda(64, torch.float16),
                                    _FakeCuda(1, torch.int32), stream=0)
    assert e.value.code == -3
    with pytest.raises(Z.ZeroError) as e:           # gather source shorter than offset + part
        Z.zero_allgather_params([_FakeCuda(100, torch.float16)] * 2, 60, 50, _FakeCuda(100, torch.float16), stream=0)
    assert e.value.code == -4


def test_broadcast_update_rejects_bad_destinations():
    L = Z.lib
    base = 0x7000_0000
    st = [base + 0x100_0000 * i for i in range(1, 7)]
    red, status, hp = base + 0x100_0000 * 12, base + 0x100_0000 * 13, Z.hparams()

    def call(dsts, n_dsts=None):
        arr = None if dsts is None else (ctypes.c_void_p * max(1, len(dsts)))(*dsts)
        return L.zero_adam_step_reduced_bcast(red, 64, *st, arr, len(dsts or []) if n_dsts is None else n_dsts, 0,
                                              ctypes.byref(hp), status, None, None, 0.0, None)
    assert call(None, 1) == -1                                      # no destination array
    assert call([0x7E00_0000], 0) == -1                             # no destinations
    assert call([0x7E00_0000] * 129) == -1                          # more than ZERO_MAX_WORLD
    assert call([0x7E00_0000, 0]) == -1                             # NULL destination
    assert call([0x7E00_0000, 0x7F00_0001]) == -2                   # misaligned destination
    assert call([0x7E00_0000, 0x7E00_0040]) == -1                   # destinations overlap
    assert call([0x7E00_0000, st[0] + 16]) == -1                    # destination overlaps master_in
    assert L.zero_adam_step_reduced_bcast(red, 0, *st, (ctypes.c_void_p * 1)(0x7E00_0000), 1, 0,
                                          ctypes.byref(hp), status, None, None, 0.0, None) == 0


def test_staged_runner_rejects_bad_arguments():
    L = Z.lib
    hp = Z.hparams()
    grads = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    desc = (Z.BucketBanks * 1)()
    desc[0].padded_numel = 64
    desc[0].grad_bufs = ctypes.cast(grads, ctypes.POINTER(ctypes.c_void_p))
    red = (ctypes.c_void_p * 1)(0x30000)
    out = ctypes.c_void_p()

    def call(reduced=red, max_norm=0.0, flag=0x40000, sq=None, ws=None):
        return L.zero_runner_create_staged(desc, 1, 2, 0, 0, ctypes.byref(hp), 1024.0, 1000, 1.0,
                                           None if reduced is None else ctypes.cast(reduced, ctypes.POINTER(ctypes.c_void_p)),
                                           max_norm, flag, 0x50000, sq, ws, ctypes.byref(out))
    assert call(reduced=None) == -1                       # no reduced-gradient buffers
    assert call(reduced=(ctypes.c_void_p * 1)(0)) == -1    # NULL reduced buffer
    assert call(max_norm=-1.0) == -1
    assert call(max_norm=float("nan")) == -1
    assert call(max_norm=1.0) == -1                       # clipping without a norm
    assert call(sq=0x60000) == -1                         # a norm without a workspace
    assert call(flag=0x40004) == -2                       # the two flag words must be 8-byte aligned


def test_step_kernel_hook_validates_and_resets():
    """zero_test_force_step_kernel: host only, -1..3 accepted, anything else
    ZERO_ERR_ARG; the binding's names match the C values."""
    L = Z.lib
    for kind in (Z.STEP_KERNEL_REGISTER, Z.STEP_KERNEL_PIPE, Z.STEP_KERNEL_QUAD, Z.STEP_KERNEL_OCT,
                 Z.STEP_KERNEL_AUTO):
        assert L.zero_test_force_step_kernel(kind) == 0
    assert L.zero_test_force_step_kernel(4) == -1
    assert L.zero_test_force_step_kernel(-2) == -1
    assert b"kind" in L.zero_last_error()
    assert (Z.STEP_KERNEL_AUTO, Z.STEP_KERNEL_REGISTER, Z.STEP_KERNEL_PIPE, Z.STEP_KERNEL_QUAD,
            Z.STEP_KERNEL_OCT) == (-1, 0, 1, 2, 3)
    Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


def test_runner_bucket_kernel_rejects_bad_arguments():
    """zero_runner_bucket_kernel: a NULL runner or a NULL result is
    ZERO_ERR_ARG before anything touches CUDA."""
    L = Z.lib
    kind = ctypes.c_int32(7)
    assert L.zero_runner_bucket_kernel(None, 0, ctypes.byref(kind)) == -1
    assert kind.value == 7
    assert b"NULL" in L.zero_last_error()
