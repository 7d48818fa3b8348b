"""The bounds-checking debug build of libzero on the parity cases.

libzero_debug.so is the same library compiled with ZERO_DEBUG_BOUNDS: every
kernel of the step, the statistics pass and the staged route checks each
index it is about to touch (element ranges against the call's count, chunk
offsets against the shared-memory tile) and, when a check fails, records the
value 4 in the call's flag (or status) word and skips the access instead of
making it.  Running the parity cases through it shows, on the GPU, that
every access of those launches stayed in bounds (the flag stays 0) and that
the checks change no result (parity with the oracle is still bit-exact).
The library's device code is otherwise identical to the release build.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import Guarded, host_u16
from test_gpu_staged import Staged
from test_gpu_step import Case, _adam, _hp

pytestmark = pytest.mark.gpu

SMS = 148


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    path = os.path.join(os.path.dirname(Z.__file__), "build.py")
    spec = importlib.util.spec_from_file_location("zero_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = Z.load_library(mod.build(debug_bounds=True))
    saved = Z.lib
    Z.lib = lib
    try:
        yield lib
    finally:
        Z.lib = saved


def _pipe_T(world):
    return min(8192, (180 * 1024 // (2 * (2 * world + 12))) // 512 * 512)


@pytest.mark.parametrize("kind", [Z.STEP_KERNEL_AUTO, Z.STEP_KERNEL_REGISTER, Z.STEP_KERNEL_PIPE, Z.STEP_KERNEL_QUAD,
                                  Z.STEP_KERNEL_OCT])
@pytest.mark.parametrize("world,padded,part,offs", [
    (3, 3 * 50_001, -1, (0, 0, 0)),                                  # ragged
    (4, 4 * 20_011, -1, (3, 5, 1)),                                  # scalar path (phases differ)
    (8, 8 * ((2 * SMS * _pipe_T(8) + 4099) // 8), -1, (0, 0, 0)),    # two tiles per SM + tail
    (4, 4 * (2 * SMS * _pipe_T(4) + 8 * 100 + 4), 1, (0, 0, 0)),     # one partition, head
    (2, 2 * 1_000_003, -1, (0, 0, 0)),                               # N = 2 (quad kernel), ragged
    (64, 64 * 4099, -1, (0, 0, 0)),                                  # large N (register)
])
def test_fused_step_in_bounds(world, padded, part, offs, kind):
    # every step kernel that can run the case (the hook falls back to the
    # automatic choice where the forced one cannot)
    c = Case(padded, world, seed=700 + world, partition=part, goff=offs[0], soff=offs[1], poff=offs[2], norm=True,
             scale=65536.0)
    ref, ovf, _ = c.expect(_adam(0.01), t=2)
    Z.zero_test_force_step_kernel(kind)
    try:
        c.run(_adam(0.01), t=2)
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)
    assert int(c.flag.item()) == ovf == 0
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("kind", [Z.STEP_KERNEL_AUTO, Z.STEP_KERNEL_REGISTER, Z.STEP_KERNEL_PIPE,
                                  Z.STEP_KERNEL_QUAD, Z.STEP_KERNEL_OCT])
@pytest.mark.parametrize("world,padded,part", [(8, 8 * 250_003, -1), (16, 16 * 60_001, -1), (3, 3 * 7_001, 2),
                                                (2, 2 * 1_900_003, 1), (1, 1_000_003, -1)])
def test_staged_route_and_statistics_in_bounds(world, padded, part, kind):
    Z.zero_test_force_step_kernel(kind)
    try:
        _staged_route_and_statistics(world, padded, part)
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


def _staged_route_and_statistics(world, padded, part):
    c = Staged(padded, world, seed=720 + world, scale=65536.0, partition=part, inplace=True)
    c.reduce_scatter()
    s, inv, g = c.oracle_reduced()
    assert int(c.flag.item()) == 0
    assert np.array_equal(c.red.t.cpu().numpy().view(np.uint32), g.view(np.uint32))
    adam = _adam(0.01)
    ref, _, _ = c.expect(adam, t=3)
    c.update(adam, t=3, gate=c.flag)            # asserts status == 0
    assert c.compare(ref) == [0, 0, 0, 0]
    # the statistics pass alone and the gated fused update over the same inputs
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    Z.zero_grad_stats([x.t for x in c.g_dev], c.padded, c.partition, c.scale, flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0


def test_broadcast_update_in_bounds():
    world, padded = 4, 4 * 600_007
    c = Staged(padded, world, seed=740, scale=65536.0, inplace=True)
    c.reduce_scatter()
    dsts = [c.p_dev, Guarded(c.n, torch.float16, 3)]
    adam = _adam()
    Z.zero_adam_step_reduced_bcast(c.red.t, c.n, *[b.t for b in c.in_dev], *[b.t for b in c.out_dev],
                                   [d.t for d in dsts], _hp(adam, 1), c.status, gate=c.flag)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    ref, _, _ = c.expect(adam, t=1)
    assert c.compare(ref) == [0, 0, 0, 0]
    assert np.array_equal(host_u16(dsts[1].t), ref.params)


@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
@pytest.mark.parametrize("world,part,src_off,dst_off", [
    (8, 300_000, 0, 0),          # every slice on its destination's phase
    (4, 250_001, 0, 0),          # ranks 1-3 realigned (odd partition)
    (5, 123_457, 3, 1),          # everything off the phase, heads and tails
    (3, 5, 1, 2),                # slices shorter than one 16-byte block
    (8, 300_000, 0, 8),          # 16-byte phase shared, destinations 16 bytes off 32 (fp16)
    (3, 13, 0, 3),               # slices between one 16- and one 32-byte block
])
def test_allgather_in_bounds(dtype, world, part, src_off, dst_off):
    """Both copy kernels (phase-matched and realigned) with their element
    edges, through the debug build: the status word stays 0, every byte of
    the destination is the oracle's, the guard bytes around it are intact."""
    import oracle
    es = torch.empty((), dtype=dtype).element_size()
    npdt = np.uint16 if es == 2 else np.uint32
    rng = np.random.Generator(np.random.PCG64(world * part + src_off))
    host, dev, keep = [], [], []
    for _ in range(world):
        h = rng.integers(0, 2 ** (8 * es), src_off + part + 3, dtype=np.uint64).astype(npdt)
        base = torch.empty(h.size + src_off + 8, dtype=dtype, device="cuda")
        view = base[src_off:src_off + h.size]
        view.view(torch.int16 if es == 2 else torch.int32).copy_(
            torch.from_numpy(h.view(np.int16 if es == 2 else np.int32)))
        host.append(h)
        dev.append(view)
        keep.append(base)
    dst = Guarded(world * part, dtype, dst_off)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Z.zero_allgather_params(dev, src_off, part, dst.t, status=status)
    torch.cuda.synchronize()
    dst.check()
    assert int(status.item()) == 0
    got = dst.t.view(torch.int16 if es == 2 else torch.int32).cpu().numpy().view(npdt)
    if es == 2:
        ref = oracle.allgather(host, src_off, part)
    else:
        ref = oracle.allgather([h.view(np.uint16) for h in host], 2 * src_off, 2 * part).view(np.uint32)
    assert np.array_equal(got, ref)
