"""Parity of the quad-streaming step kernel (fused_step_quad_kernel) against
the oracle.

It runs every call with N <= 2, calls with fewer than 128 pipeline tiles per
SM, and gradient buffers in another GPU's memory: one thread per 4 elements,
two quads in flight, replicas' 8-byte loads issued in batches of 8 (so
N = 9, 17, 20 take partial batches), the vector region from the common
16-byte phase, everything else on the scalar path.  Here the kernel is forced
(zero_test_force_step_kernel) or reached by the automatic choice; every case
is bit-exact against the oracle, flag and norm included.
"""
import numpy as np
import pytest
import torch

import oracle
import zero_sharded_optimizer_reduce_b200 as Z
from test_gpu_step import Case, _adam

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["quad", "oct"])
def quad(request):
    """The quad kernel, then the oct kernel (8 elements per thread, 32-byte
    state stores; it runs where the fp32 outputs are 32-byte aligned at the
    vector region, elsewhere the call keeps its automatic choice)."""
    Z.zero_test_force_step_kernel(Z.STEP_KERNEL_QUAD if request.param == "quad" else Z.STEP_KERNEL_OCT)
    try:
        yield request.param
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8, 9, 16, 17, 20])
def test_quad_ragged_every_world(quad, world):
    # a per-rank size that leaves a tail of 1-7 elements after the last vector
    per_rank = 33_333 + world
    c = Case(world * per_rank, world, seed=900 + world, norm=True, scale=65536.0)
    ref, ovf, sq = c.expect(_adam(0.01), t=2)
    c.run(_adam(0.01), t=2)
    assert ovf == 0 and int(c.flag.item()) == 0
    assert c.compare(ref) == [0, 0, 0, 0]
    assert abs(float(c.norm.item()) - sq) <= 2.0 * c.n * 2.0 ** -53 * sq


@pytest.mark.parametrize("gd,pd", [(oracle.BF16, oracle.BF16), (oracle.F16, oracle.BF16), (oracle.BF16, oracle.F16)])
@pytest.mark.parametrize("partition", [-1, 1])
def test_quad_dtypes_and_partition_with_head(quad, gd, pd, partition):
    # buffers shifted by 3 elements: the common phase starts 5 elements in
    world = 4
    c = Case(world * 250_001, world, gdtype=gd, pdtype=pd, seed=920, partition=partition, goff=3, soff=3, poff=3,
             scale=65536.0)
    ref, _, _ = c.expect(_adam(0.01), t=3)
    c.run(_adam(0.01), t=3)
    assert c.compare(ref) == [0, 0, 0, 0]


def test_quad_overflow_and_in_place(quad):
    world = 2
    c = Case(world * 1_000_003, world, seed=930, inplace=True)
    pos = np.array([7, 1_000_000, 1_999_999])
    from _gpu import to_dev_u16
    for k, p in enumerate(pos):
        oracle_bits = c.G[k % world]
        oracle_bits[p] = 0x7C00 if k % 2 == 0 else 0x7E00
    for k in range(world):
        to_dev_u16(c.G[k], torch.float16, buf=c.g_dev[k])
    ref, ovf, _ = c.expect(_adam())
    c.run(_adam())
    assert ovf == 1 and int(c.flag.item()) == 1


def test_quad_deterministic_norm(quad):
    c = Case(2 * 3_000_001, 2, seed=940, norm=True, scale=65536.0)
    vals = []
    for _ in range(3):
        c.norm.zero_()
        c.run(_adam())
        vals.append(float(c.norm.item()))
    assert vals[0] == vals[1] == vals[2]


@pytest.mark.parametrize("world", [1, 4, 8])
def test_automatic_choice_mid_size(world):
    # 16M-class calls (fewer than 128 tiles per SM) take the quad kernel on
    # their own; the result is the oracle's either way
    c = Case(world * ((1 << 21) + 3), world, seed=950 + world, norm=True, scale=65536.0)
    ref, ovf, sq = c.expect(_adam(0.01), t=1)
    c.run(_adam(0.01), t=1)
    assert ovf == 0 and c.compare(ref) == [0, 0, 0, 0]


def test_runner_reports_the_kernel_choice():
    """zero_runner_bucket_kernel names the kernel the next launch runs: the
    pipeline kernel for a 64M-element bucket at N = 8 (147 tiles per SM), the
    oct kernel for a 1M-element bucket (the optimizer's buffers are 32-byte
    aligned), the register kernel above N = 20, and whatever the override
    forces."""
    from zero_sharded_optimizer_reduce_b200.optimizer import ZeroAdam
    opt = ZeroAdam([64 << 20, 1 << 20], world=8, bucket_elems=64 << 20)
    assert opt.layout.n_buckets == 2
    assert opt.bucket_kernels() == [Z.STEP_KERNEL_PIPE, Z.STEP_KERNEL_OCT]
    for kind in (Z.STEP_KERNEL_REGISTER, Z.STEP_KERNEL_QUAD):
        Z.zero_test_force_step_kernel(kind)
        try:
            assert opt.bucket_kernels() == [kind, kind]
        finally:
            Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)
    del opt
    assert ZeroAdam([240_000], world=24).bucket_kernels() == [Z.STEP_KERNEL_REGISTER]
    assert ZeroAdam([240_000], world=2).bucket_kernels() == [Z.STEP_KERNEL_OCT]
    assert ZeroAdam([240_000], world=4, mode="staged").bucket_kernels() is None
    torch.cuda.empty_cache()
