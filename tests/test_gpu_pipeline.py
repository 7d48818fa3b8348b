"""Parity of the shared-memory pipeline kernel against the oracle.

Calls whose arrays share a 16-byte phase, with N >= 3 and at least 128 tiles
per SM, run the bulk-copy pipeline kernel; this module forces it (the test
hook zero_test_force_step_kernel) at sizes that give every SM a few tiles
(two stages of at most 180 KB: 6144 elements per tile at N = 1 down to 1536
at N = 20, on 148 SMs), with ragged tails, a shifted
common phase (scalar head), single partitions, bf16 and overflow.  Above
N = 20 the register kernel runs at the same sizes; those cases (N up to 128)
check that the kernel choice at the boundary keeps parity.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_step import Case, _adam

pytestmark = pytest.mark.gpu

SMS = 148


@pytest.fixture(scope="module", autouse=True)
def pipeline_kernel():
    """These sizes give every SM a few tiles; in normal use such calls take
    the quad kernel (the pipeline kernel runs calls of 128 tiles per SM and
    more), so the module forces the pipeline kernel wherever it can run."""
    import zero_sharded_optimizer_reduce_b200 as Z
    Z.zero_test_force_step_kernel(Z.STEP_KERNEL_PIPE)
    try:
        yield
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


def _tile(world):
    """The pipeline tile for N replicas (N <= 20): the largest multiple of 512
    whose two stages fit in 180 KB.  Above N = 20 the register kernel runs;
    the size then only has to be large."""
    if world > 20:
        return 1536
    return min(8192, (180 * 1024 // (2 * (2 * world + 12))) // 512 * 512)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8, 16, 20, 21, 32, 40, 48, 64, 100, 128])
def test_pipeline_ragged(world):
    T = _tile(world)
    per_rank = (2 * SMS * T + T // 2 + 5 + world - 1) // world
    c = Case(world * per_rank, world, seed=300 + world, norm=True, scale=65536.0)
    ref, ovf, sq = c.expect(_adam(0.01), t=2)
    c.run(_adam(0.01), t=2)
    assert ovf == 0 and int(c.flag.item()) == 0
    assert c.compare(ref) == [0, 0, 0, 0]
    assert abs(float(c.norm.item()) - sq) <= 1e-5 * sq


@pytest.mark.parametrize("offs", [(3, 3, 3), (5, 5, 5)])
def test_pipeline_shifted_phase(offs):
    world = 8
    T = _tile(world)
    n = world * ((2 * SMS * T + 1001) // world)
    c = Case(n, world, seed=320, goff=offs[0], soff=offs[1], poff=offs[2])
    ref, _, _ = c.expect(_adam())
    c.run(_adam())
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("r", [0, 1, 3])
def test_pipeline_single_partition(r):
    world = 4
    T = _tile(world)
    P = 2 * SMS * T + 8 * 77          # multiple of 8: every partition keeps the phase
    c = Case(world * P, world, seed=330, partition=r)
    ref, _, _ = c.expect(_adam())
    c.run(_adam())
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("gd,pd", [(oracle.BF16, oracle.BF16), (oracle.F16, oracle.BF16)])
def test_pipeline_bf16(gd, pd):
    world = 16
    T = _tile(world)
    n = world * ((2 * SMS * T + 333) // world)
    c = Case(n, world, gdtype=gd, pdtype=pd, seed=340, scale=65536.0)
    ref, _, _ = c.expect(_adam(0.01), t=5)
    c.run(_adam(0.01), t=5)
    assert c.compare(ref) == [0, 0, 0, 0]


def test_pipeline_overflow_flag_and_in_place():
    world = 8
    T = _tile(world)
    n = world * ((3 * SMS * T + 17) // world)
    c = Case(n, world, seed=350, inplace=True)
    workloads.inject(c.G[2], np.array([7, n // 2, n - 3]), np.array([True, False, True]))
    from _gpu import to_dev_u16
    to_dev_u16(c.G[2], torch.float16, buf=c.g_dev[2])
    ref, ovf, _ = c.expect(_adam())
    c.run(_adam())
    assert ovf == 1 and int(c.flag.item()) == 1


@pytest.mark.parametrize("world", [8, 64])
def test_pipeline_deterministic(world):
    T = _tile(world)
    n = world * ((2 * SMS * T + 4099) // world)
    c = Case(n, world, seed=360, norm=True)
    outs, norms = [], []
    for _ in range(3):
        c.norm.zero_()
        c.run(_adam())
        outs.append([b.t.clone() for b in c.out_dev] + [c.p_dev.t.clone()])
        norms.append(float(c.norm.item()))
    assert norms[0] == norms[1] == norms[2]
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def test_pipeline_single_partition_with_head():
    # P = 4 (mod 8): rank r's gradient slice starts 8 bytes off the 16-byte
    # phase for odd r, the state arrays at phase 0; the common phase is
    # element 4, so the pipeline kernel runs with a 4-element scalar head
    world = 4
    T = _tile(world)
    P = 2 * SMS * T + 8 * 100 + 4
    for r in (1, 2):
        c = Case(world * P, world, seed=370 + r, partition=r)
        ref, _, _ = c.expect(_adam())
        c.run(_adam())
        assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("world,gd,pd", [(32, oracle.BF16, oracle.BF16), (64, oracle.F16, oracle.BF16),
                                         (128, oracle.BF16, oracle.F16)])
def test_pipeline_large_world_bf16_and_partition(world, gd, pd):
    # the register kernel above N = 20, both dtypes, whole bucket and one partition
    T = _tile(world)
    P = 2 * SMS * T + 8 * 31
    G = None
    for r in (-1, world - 1):
        c = Case(world * P, world, gdtype=gd, pdtype=pd, seed=380 + world, partition=r, scale=65536.0, G=G)
        G = c.G                      # both calls take the same seeded gradients
        ref, _, _ = c.expect(_adam(0.01), t=3)
        c.run(_adam(0.01), t=3)
        assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("world", [32, 64])
def test_pipeline_large_world_overflow(world):
    T = _tile(world)
    n = world * ((2 * SMS * T + 77) // world)
    c = Case(n, world, seed=390 + world)
    workloads.inject(c.G[world - 1], np.array([n // 3]), np.array([False]))
    from _gpu import to_dev_u16
    to_dev_u16(c.G[world - 1], torch.float16, buf=c.g_dev[world - 1])
    ref, ovf, _ = c.expect(_adam())
    c.run(_adam())
    assert ovf == 1 and int(c.flag.item()) == 1
