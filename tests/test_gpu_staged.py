"""Parity of the staged step (zero_reduce_scatter_grads, then
zero_adam_step_reduced) against the oracle.

The reduce-scatter's fp32 output must equal the oracle's unscaled rank-order
sums bit for bit (flag exact, norm within the fp64 reordering bound); the
update from it must equal the oracle's step on the same inputs bit for bit,
in and out of place, gated and clipped.  Every case runs twice: with the
automatic kernel choice and with the pipeline kernels forced (the
test hook zero_test_force_step_kernel), so that both the register and the
pipeline statistics and update kernels run at these sizes; ragged tails,
single partitions, bf16, a reduced buffer off the gradients' 16-byte phase
(scalar path), N up to 64, and sizes of at least two update tiles per SM.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import Guarded, host_f32, host_u16, to_dev_f32, to_dev_u16
from test_gpu_gated import _norm_tol
from test_gpu_step import Case, _adam, _hp

pytestmark = pytest.mark.gpu

SMS = 148


_KINDS = {"auto": Z.STEP_KERNEL_AUTO, "pipeline": Z.STEP_KERNEL_PIPE, "register": Z.STEP_KERNEL_REGISTER,
          "quad": Z.STEP_KERNEL_QUAD}


@pytest.fixture(autouse=True, params=list(_KINDS))
def kernel_choice(request):
    """Every case four times: the automatic choice (at these sizes the
    reduce-scatter takes the oct kernel at N <= 2 with `reduced` 32-byte
    aligned, else the quad kernel up to N = 16, and the update the register
    kernel), the pipeline kernels forced wherever they can run, the register
    kernels forced, and the quad reduce-scatter forced."""
    Z.zero_test_force_step_kernel(_KINDS[request.param])
    try:
        yield request.param
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


class Staged(Case):
    def __init__(self, *a, roff=0, **k):
        super().__init__(*a, norm=True, **k)
        self.red = Guarded(self.n, torch.float32, roff)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def reduce_scatter(self, divisor=0.0):
        Z.zero_reduce_scatter_grads([g.t for g in self.g_dev], self.padded, self.partition, self.scale,
                                    self.red.t, self.flag, self.norm, self.ws, divisor)
        torch.cuda.synchronize()
        for b in self.g_dev + [self.red]:
            b.check()

    def update(self, adam, t=1, gate=None, clip_sqnorm=None, max_norm=0.0):
        Z.zero_adam_step_reduced(self.red.t, self.n, *[b.t for b in self.in_dev], *[b.t for b in self.out_dev],
                                 self.p_dev.t, _hp(adam, t), self.status, gate=gate, clip_sqnorm=clip_sqnorm,
                                 max_norm=max_norm)
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0
        for b in self.in_dev + list(self.out_dev) + [self.p_dev, self.red]:
            b.check()

    def oracle_reduced(self, divisor=None):
        s = oracle.reduce(self.G, self.gdtype, self.begin, self.n)
        d = float(self.world if divisor is None else divisor)
        inv = oracle.adam_constants(_adam(), 1, d, self.scale)[4]
        return s, inv, oracle.unscale(s, inv)


def _pipe_count(world):
    """Elements that give the statistics pipeline at least two tiles per SM."""
    t = min(8192, (180 * 1024 // (2 * 2 * world)) // 512 * 512)
    return 2 * SMS * t + t // 3 + 7


CASES = [
    # world, padded, gdtype, partition, goff, roff
    (1, 1_000_003, oracle.F16, -1, 0, 0),
    (3, 3 * 100_003, oracle.BF16, -1, 0, 0),
    (8, 8 * (_pipe_count(8) // 8 + 1), oracle.F16, -1, 0, 0),
    (16, 16 * (_pipe_count(16) // 16 + 1), oracle.BF16, -1, 0, 0),
    (8, 8 * 50_001, oracle.F16, 5, 0, 0),
    (4, 4 * 20_011, oracle.F16, -1, 3, 0),
    (4, 4 * 20_011, oracle.F16, -1, 0, 1),
    (64, 64 * 4099, oracle.F16, -1, 0, 0),
    # about 4 update tiles of 4096 per SM: the update's pipeline kernel when forced
    (4, 4 * 600_007, oracle.F16, -1, 0, 0),
    (2, 2 * 1_000_003, oracle.BF16, -1, 0, 0),
    (2, 2 * 1_900_003, oracle.F16, 1, 0, 0),
]


@pytest.mark.parametrize("world,padded,gd,part,goff,roff", CASES)
def test_reduce_scatter_grads_bit_exact(world, padded, gd, part, goff, roff):
    c = Staged(padded, world, gdtype=gd, pdtype=gd, seed=500 + world, scale=65536.0, partition=part, goff=goff,
               roff=roff)
    c.reduce_scatter()
    s, inv, g = c.oracle_reduced()
    got = host_f32(c.red.t)
    assert np.array_equal(got.view(np.uint32), g.view(np.uint32))
    assert int(c.flag.item()) == oracle.any_nonfinite(s) == 0
    sq = oracle.grad_sqnorm(s, inv)
    assert abs(float(c.norm.item()) - sq) <= _norm_tol(c.n) * sq


def test_reduce_scatter_grads_sum_divisor_and_overflow():
    world, padded = 8, 8 * (_pipe_count(8) // 8 + 1)
    c = Staged(padded, world, seed=520, scale=1024.0)
    workloads.inject(c.G[6], np.array([11, padded // 2, padded - 1]), np.array([True, False, True]))
    to_dev_u16(c.G[6], torch.float16, buf=c.g_dev[6])
    c.reduce_scatter(divisor=1.0)
    s, inv, g = c.oracle_reduced(divisor=1.0)
    assert int(c.flag.item()) == oracle.any_nonfinite(s) == 1
    got = host_f32(c.red.t)
    # finite entries bit-exact; the non-finite ones non-finite on both sides
    fin = np.isfinite(g)
    assert np.array_equal(got[fin].view(np.uint32), g[fin].view(np.uint32))
    assert not np.isfinite(got[~fin]).any() and (~fin).sum() == 3


@pytest.mark.parametrize("world,padded,gd,part,goff,roff", CASES)
@pytest.mark.parametrize("inplace", [False, True])
def test_staged_step_equals_oracle_step(world, padded, gd, part, goff, roff, inplace):
    c = Staged(padded, world, gdtype=gd, pdtype=gd, seed=540 + world, scale=65536.0, partition=part, goff=goff,
               roff=roff, inplace=inplace)
    adam = _adam(0.01)
    ref, ovf, _ = c.expect(adam, t=4)
    c.reduce_scatter()
    c.update(adam, t=4, gate=c.flag)
    assert ovf == 0
    assert c.compare(ref) == [0, 0, 0, 0]


def test_staged_update_from_oracle_reduced_input():
    """The update alone, fed the oracle's reduced gradients (uploaded, not
    produced by the GPU reduce-scatter), against the oracle's update."""
    world, padded = 4, 4 * 600_007
    c = Staged(padded, world, seed=560, scale=4096.0, pdtype=oracle.BF16)
    s, inv, g = c.oracle_reduced()
    to_dev_f32(g, buf=c.red)
    adam = _adam(0.01)
    c.update(adam, t=7)
    ref, _, _ = c.expect(adam, t=7)
    assert c.compare(ref) == [0, 0, 0, 0]


def test_staged_gate_writes_nothing():
    world, padded = 8, 8 * 250_003
    c = Staged(padded, world, seed=570, scale=65536.0, inplace=True)
    workloads.inject(c.G[0], np.array([5]), np.array([False]))
    to_dev_u16(c.G[0], torch.float16, buf=c.g_dev[0])
    before = [b.t.clone() for b in c.in_dev] + [c.p_dev.t.clone()]
    c.reduce_scatter()
    assert int(c.flag.item()) == 1
    c.update(_adam(), gate=c.flag)
    after = [b.t for b in c.in_dev] + [c.p_dev.t]
    for x, y in zip(before, after):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_staged_clip_matches_oracle():
    world, padded = 8, 8 * 250_003
    c = Staged(padded, world, seed=580, scale=65536.0)
    c.reduce_scatter()
    s, inv, _ = c.oracle_reduced()
    sq = oracle.grad_sqnorm(s, inv)
    max_norm = 0.25 * float(np.sqrt(sq))
    adam = _adam(0.01)
    c.update(adam, t=2, gate=c.flag, clip_sqnorm=c.norm, max_norm=max_norm)
    clip = oracle.clip_coefficient(sq, np.float32(max_norm))
    assert clip < 1
    ref = c.host.copy()
    cst = oracle.adam_constants(adam, 2, float(world), c.scale)
    oracle.adam_update_clipped(s, cst, clip, ref.master, ref.m, ref.v, ref.params)
    diffs = c.compare(ref)
    if oracle.clip_coefficient(float(c.norm.item()), np.float32(max_norm)) == clip:
        assert diffs == [0, 0, 0, 0], diffs


@pytest.mark.parametrize("shift", [0, 3])
def test_staged_update_broadcasts_parameters(shift):
    """zero_adam_step_reduced_bcast: the same update, its parameters stored to
    several destinations (one of them off the 16-byte phase when shift > 0:
    then every element is stored on its own); each equals the oracle."""
    world, padded = 4, 4 * 600_007          # the pipeline size
    c = Staged(padded, world, seed=590, scale=65536.0, inplace=True)
    c.reduce_scatter()
    dsts = [c.p_dev] + [Guarded(c.n, torch.float16, shift if k == 1 else 0) for k in range(2)]
    adam = _adam(0.01)
    Z.zero_adam_step_reduced_bcast(c.red.t, c.n, *[b.t for b in c.in_dev], *[b.t for b in c.out_dev],
                                   [d.t for d in dsts], _hp(adam, 2), c.status, gate=c.flag)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    for b in c.in_dev + dsts + [c.red]:
        b.check()
    ref, _, _ = c.expect(adam, t=2)
    assert c.compare(ref) == [0, 0, 0, 0]
    for d in dsts[1:]:
        assert np.array_equal(host_u16(d.t), ref.params)
