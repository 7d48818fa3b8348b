"""Parity of the fused step, the all-gather and the flatten against the oracle.

Every call goes through the C ABI (libzero.so via the ctypes binding); every
expected value comes from `oracle/` on the same seeded inputs.  Sizes span
several vectors and blocks plus ragged heads and tails; edge cases cover
N = 1 .. 64, sizes down to one element per rank, unaligned buffers (scalar
path), in-place updates, bf16, injected inf / NaN and the norm.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import Guarded, assert_f32_close, assert_u16_close, host_f32, host_u16, to_dev_f32, to_dev_u16

pytestmark = pytest.mark.gpu

TD = {oracle.F16: torch.float16, oracle.BF16: torch.bfloat16}


def _adam(wd=0.0):
    return workloads.AdamConfig(weight_decay=wd)


def _hp(adam, t, divisor=0.0):
    return Z.hparams(adam.lr, adam.beta1, adam.beta2, adam.eps, adam.weight_decay, t, divisor)


class Case:
    """Inputs of one step on the device (guarded) and on the host."""

    def __init__(self, padded, world, gdtype=oracle.F16, pdtype=oracle.F16, seed=0, scale=1024.0,
                 partition=-1, goff=0, soff=0, poff=0, inplace=False, master=None, norm=False, G=None):
        self.padded, self.world, self.gdtype, self.pdtype = padded, world, gdtype, pdtype
        self.partition, self.scale, self.inplace = partition, scale, inplace
        self.P = padded // world
        n = padded if partition < 0 else self.P
        self.n = n
        self.begin = 0 if partition < 0 else partition * self.P
        # G: the same draws handed over by a caller that runs several cases on them
        self.G = G if G is not None else [workloads.grads(padded, 10_000 * seed + k, 1e-3, scale, gdtype)
                                          for k in range(world)]
        m0 = workloads.master(n, 10_000 * seed + 999) if master is None else master
        self.host = oracle.initial_state(m0, pdtype)
        rng = np.random.Generator(np.random.PCG64(seed + 5))
        # non-zero moments so that every term of the update is exercised
        self.host.m[:] = (rng.standard_normal(n) * 1e-4).astype(np.float32)
        self.host.v[:] = (rng.random(n) * 1e-7).astype(np.float32)
        self.g_dev = [to_dev_u16(g, TD[gdtype], elem_offset=goff) for g in self.G]
        self.in_dev = [to_dev_f32(a, elem_offset=soff) for a in (self.host.master, self.host.m, self.host.v)]
        self.out_dev = self.in_dev if inplace else [Guarded(n, torch.float32, soff) for _ in range(3)]
        self.p_dev = Guarded(n, TD[pdtype], poff)
        self.flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.norm = torch.zeros(1, dtype=torch.float64, device="cuda") if norm else None
        self.ws = torch.zeros(Z.zero_step_workspace_bytes(), dtype=torch.uint8, device="cuda") if norm else None

    def run(self, adam, t=1, divisor=0.0):
        Z.zero_reduce_scatter_adam_step([g.t for g in self.g_dev], self.padded, self.partition,
                                        *[b.t for b in self.in_dev], *[b.t for b in self.out_dev],
                                        self.p_dev.t, _hp(adam, t, divisor), self.scale, self.flag,
                                        self.norm, self.ws)
        torch.cuda.synchronize()
        for b in self.g_dev + self.in_dev + list(self.out_dev) + [self.p_dev]:
            b.check()

    def expect(self, adam, t=1, divisor=None):
        ref = self.host.copy()
        d = float(self.world if divisor is None else divisor)
        ovf, sq = oracle.flat_step(self.G, ref, adam, t, self.scale, d, self.gdtype, self.pdtype,
                                   begin=self.begin, count=self.n)
        return ref, ovf, sq

    def compare(self, ref):
        got = [host_f32(b.t) for b in self.out_dev]
        diffs = [assert_f32_close(got[i], getattr(ref, nm), nm) for i, nm in enumerate(("master", "m", "v"))]
        diffs.append(assert_u16_close(host_u16(self.p_dev.t), ref.params, "params"))
        return diffs


def test_tiny_flat_workload_three_steps_bit_exact():
    """Ψ = 1,000,003 padded to 1,000,004, N = 4, loss scale 1024, 3 steps."""
    w = workloads.tiny_flat()
    (psi,) = w.numels
    L = oracle.partition_layout([psi], w.world)
    padded = L.bucket_padded[0]
    m0 = workloads.master(psi, 7)
    m0 = np.concatenate([m0, np.zeros(padded - psi, np.float32)])
    ref = oracle.initial_state(m0)
    banks = [[to_dev_f32(a) for a in (ref.master, ref.m, ref.v)],
             [Guarded(padded, torch.float32) for _ in range(3)]]
    params = [to_dev_u16(ref.params, torch.float16), Guarded(padded, torch.float16)]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    cur = 0
    for t in range(1, w.steps + 1):
        G = []
        for k in range(w.world):
            g = workloads.grads(padded, workloads.seed_for(w.seed, t, k), 1e-3, w.loss_scale)
            g[psi:] = 0
            G.append(g)
        gd = [to_dev_u16(g, torch.float16) for g in G]
        Z.zero_reduce_scatter_adam_step([g.t for g in gd], padded, Z.ZERO_ALL_PARTITIONS,
                                        *[b.t for b in banks[cur]], *[b.t for b in banks[cur ^ 1]],
                                        params[cur ^ 1].t, _hp(w.adam, t), w.loss_scale, flag)
        ovf, _ = oracle.flat_step(G, ref, w.adam, t, w.loss_scale, float(w.world))
        torch.cuda.synchronize()
        assert ovf == 0 and int(flag.item()) == 0
        cur ^= 1
        got = [host_f32(b.t) for b in banks[cur]]
        for arr, nm in zip(got, ("master", "m", "v")):
            assert assert_f32_close(arr, getattr(ref, nm), nm) == 0, f"{nm} not bit-exact at step {t}"
        assert assert_u16_close(host_u16(params[cur].t), ref.params, "params") == 0
        # padding stays zero
        assert (got[0][psi:] == 0).all() and (host_u16(params[cur].t)[psi:] == 0).all()
        for b in banks[0] + banks[1] + params:
            b.check()


@pytest.mark.parametrize("r", [0, 1, 2, 3])
def test_single_partition_each_rank(r):
    c = Case(1_000_004, 4, seed=1, partition=r)
    c.run(_adam())
    ref, ovf, _ = c.expect(_adam())
    assert ovf == 0 and int(c.flag.item()) == 0
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("world", [1, 2, 3, 5, 8, 16, 64])
@pytest.mark.parametrize("per_rank", [1, 7, 8, 9, 257, 4099])
def test_sizes_and_world(world, per_rank):
    c = Case(world * per_rank, world, seed=world * 7 + per_rank)
    c.run(_adam(0.01))
    ref, ovf, _ = c.expect(_adam(0.01))
    assert ovf == 0 and int(c.flag.item()) == 0
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("offs", [(1, 0, 0), (0, 1, 0), (0, 0, 1), (3, 3, 3), (2, 1, 6)])
def test_unaligned_buffers_take_scalar_or_shifted_path(offs):
    goff, soff, poff = offs
    c = Case(8 * 5003, 8, seed=3, goff=goff, soff=soff, poff=poff)
    c.run(_adam())
    ref, _, _ = c.expect(_adam())
    assert c.compare(ref) == [0, 0, 0, 0]


def test_in_place_update():
    c = Case(4 * 100_003, 4, seed=4, inplace=True)
    ref, _, _ = c.expect(_adam())
    c.run(_adam())
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("gd,pd", [(oracle.BF16, oracle.BF16), (oracle.F16, oracle.BF16), (oracle.BF16, oracle.F16)])
def test_bf16_variants(gd, pd):
    c = Case(8 * 40_001, 8, gdtype=gd, pdtype=pd, seed=5, scale=65536.0)
    c.run(_adam(0.01), t=3)
    ref, _, _ = c.expect(_adam(0.01), t=3)
    assert c.compare(ref) == [0, 0, 0, 0]


def test_sum_instead_of_mean_and_late_step():
    c = Case(2 * 50_000, 2, seed=6)
    c.run(_adam(), t=1000, divisor=1.0)
    ref, _, _ = c.expect(_adam(), t=1000, divisor=1.0)
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("where", ["vector", "tail", "both"])
@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_overflow_flag_bit_exact(where, dtype):
    n = 16 * 10_001                       # odd per-rank size: a ragged tail
    c = Case(n, 16, gdtype=dtype, pdtype=dtype, seed=7)
    pos = {"vector": [100, 5000], "tail": [n - 1], "both": [3, n - 2]}[where]
    rep = 11
    workloads.inject(c.G[rep], np.array(pos), np.array([True, False][:len(pos)]), dtype)
    to_dev_u16(c.G[rep], TD[dtype], buf=c.g_dev[rep])
    c.run(_adam())
    _, ovf, _ = c.expect(_adam())
    assert ovf == 1 and int(c.flag.item()) == 1


def test_overflow_flag_is_never_cleared_by_the_kernel():
    c = Case(4 * 1000, 4, seed=8)
    c.flag.fill_(1)
    c.run(_adam())
    assert int(c.flag.item()) == 1


def test_bf16_finite_inputs_overflowing_the_sum():
    c = Case(2 * 64, 2, gdtype=oracle.BF16, pdtype=oracle.BF16, seed=9)
    for k in range(2):
        c.G[k][10] = 0x7F7F
        to_dev_u16(c.G[k], torch.bfloat16, buf=c.g_dev[k])
    c.run(_adam())
    _, ovf, _ = c.expect(_adam())
    assert ovf == 1 and int(c.flag.item()) == 1


def test_grad_sqnorm_and_determinism():
    c = Case(8 * 300_007, 8, seed=10, norm=True, scale=65536.0)
    ref, _, sq = c.expect(_adam())
    vals = []
    for _ in range(3):
        c.norm.zero_()
        c.run(_adam())
        vals.append(float(c.norm.item()))
    assert abs(vals[0] - sq) <= 1e-5 * sq
    assert vals[0] == vals[1] == vals[2]
    assert c.compare(ref) == [0, 0, 0, 0]
    # the workspace is left zero-filled and a second call adds to the norm
    assert int(c.ws[:4].view(torch.int32).item()) == 0
    c.run(_adam())
    assert abs(float(c.norm.item()) - 2 * vals[0]) <= 1e-12 * vals[0]


def test_outputs_deterministic_across_runs():
    c = Case(8 * 200_001, 8, seed=11)
    outs = []
    for _ in range(3):
        c.run(_adam())
        outs.append([host_f32(b.t).copy() for b in c.out_dev] + [host_u16(c.p_dev.t).copy()])
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


# ------------------------------------------------------------------ all-gather

@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("world,part,offset", [(8, 25_001, 0), (8, 4096, 1000), (3, 7, 3), (1, 100, 5),
                                               (64, 129, 1), (16, 50_000, 8)])
def test_allgather_bit_exact(dtype, world, part, offset):
    rng = np.random.Generator(np.random.PCG64(world + part))
    es = torch.empty((), dtype=dtype).element_size()
    shard_len = offset + part + 11
    host = [rng.integers(0, 2 ** (8 * es), shard_len, dtype=np.uint64).astype(np.uint16 if es == 2 else np.uint32)
            for _ in range(world)]
    dev = [torch.from_numpy(h.view(np.int16 if es == 2 else np.int32).copy()).cuda().view(dtype) for h in host]
    dst = Guarded(world * part, dtype)
    Z.zero_allgather_params(dev, offset, part, dst.t)
    torch.cuda.synchronize()
    dst.check()
    got = dst.t.view(torch.int16 if es == 2 else torch.int32).cpu().numpy().view(host[0].dtype)
    if es == 2:
        ref = oracle.allgather(host, offset, part)
    else:  # the oracle's gather is typed on 16-bit words: gather the two halves
        halves = [h.view(np.uint16) for h in host]
        ref = oracle.allgather(halves, 2 * offset, 2 * part).view(np.uint32)
    assert np.array_equal(got, ref)


def test_flatten_bit_exact():
    rng = np.random.Generator(np.random.PCG64(12))
    numels = [80_411, 1, 0, 1600, 7_680_000 // 64, 3, 4800, 6400 * 3 + 5]
    for world, cap, dtype in [(8, 0, torch.float32), (4, 50_000, torch.float16), (3, 30_000, torch.bfloat16)]:
        lay = Z.zero_partition_layout(numels, world, cap)
        olay = oracle.partition_layout(numels, world, cap)
        es = torch.empty((), dtype=dtype).element_size()
        npdt = np.uint16 if es == 2 else np.uint32
        host = [rng.integers(0, 2 ** 16, n, dtype=np.uint64).astype(npdt) for n in numels]
        dev = [torch.from_numpy(h.view(np.int16 if es == 2 else np.int32).copy()).cuda().view(dtype) for h in host]
        for b in range(lay.n_buckets):
            buf = Guarded(lay.bucket_padded[b], dtype)
            buf.t.view(torch.uint8).fill_(0xEE)           # padding must be cleared
            Z.zero_flatten_bucket(lay, b, dev, buf.t)
            torch.cuda.synchronize()
            buf.check()
            got = buf.t.view(torch.int16 if es == 2 else torch.int32).cpu().numpy().view(npdt)
            ref = oracle.flatten_bucket(olay, b, host, npdt)
            assert np.array_equal(got, ref)


# ------------------------------------------------------------- ZeroAdam driver

def test_zeroadam_multi_bucket_matches_stage2_with_overflow_skip():
    numels = [5000, 123, 40_000, 7, 9999, 20_000]
    N, cap = 8, 30_000
    adam = workloads.AdamConfig(weight_decay=0.01)
    L = oracle.partition_layout(numels, N, cap)
    tensors = [workloads.master(n, 500 + i) for i, n in enumerate(numels)]
    init = [oracle.flatten_bucket(L, b, tensors, np.float32) for b in range(L.n_buckets)]
    orc = oracle.StageRun(2, L, init, adam, oracle.Scaler(65536.0))
    opt = Z.ZeroAdam(numels, N, cap, lr=adam.lr, betas=(adam.beta1, adam.beta2), eps=adam.eps,
                     weight_decay=adam.weight_decay, loss_scale=65536.0, track_grad_norm=True)
    params16 = [torch.from_numpy(oracle.from_f32(t, oracle.F16).view(np.int16)).cuda().view(torch.float16)
                for t in tensors]
    opt.load(params16, [torch.from_numpy(t).cuda() for t in tensors])
    for step in range(1, 6):
        G = []
        for b in range(L.n_buckets):
            per = []
            for k in range(N):
                g = workloads.grads(L.bucket_padded[b], workloads.seed_for(9, step, k) + b, 1e-3, orc.scaler.scale)
                g[L.bucket_numel[b]:] = 0
                per.append(g)
            G.append(per)
        if step == 3:
            workloads.inject(G[1][5], np.array([17, 18]), np.array([True, False]))
        for b in range(L.n_buckets):
            for k in range(N):
                opt.grad_buffers(b)[k].copy_(torch.from_numpy(G[b][k].view(np.int16)).cuda().view(torch.float16))
        before = [[x.clone() for x in opt.state(b)] for b in range(L.n_buckets)]
        applied = opt.step()
        ovf = orc.step(G)
        assert applied == (not ovf) and opt.last_overflow == ovf == (1 if step == 3 else 0)
        assert opt.scale == orc.scaler.scale and opt.t == orc.scaler.t
        for b in range(L.n_buckets):
            fs = orc.flat_state(b)
            master, m, v, p = opt.state(b)
            assert assert_f32_close(host_f32(master), fs.master, "master") == 0
            assert assert_f32_close(host_f32(m), fs.m, "m") == 0
            assert assert_f32_close(host_f32(v), fs.v, "v") == 0
            assert assert_u16_close(host_u16(p), fs.params, "params") == 0
            if ovf:
                for x, y in zip(before[b], opt.state(b)):
                    assert torch.equal(x.view(torch.uint8) if x.dtype != torch.uint8 else x,
                                       y.view(torch.uint8) if y.dtype != torch.uint8 else y)


def test_flatten_many_tensors_spans_several_launches():
    # 150 tensors in one bucket: the copy kernel takes 64 segments per launch
    rng = np.random.Generator(np.random.PCG64(13))
    numels = rng.integers(1, 3000, 150).tolist()
    lay = Z.zero_partition_layout(numels, 8, 0)
    olay = oracle.partition_layout(numels, 8, 0)
    host = [rng.integers(0, 2 ** 16, n, dtype=np.uint64).astype(np.uint16) for n in numels]
    dev = [torch.from_numpy(h.view(np.int16).copy()).cuda().view(torch.float16) for h in host]
    buf = Guarded(lay.bucket_padded[0], torch.float16)
    Z.zero_flatten_bucket(lay, 0, dev, buf.t)
    torch.cuda.synchronize()
    buf.check()
    assert np.array_equal(host_u16(buf.t), oracle.flatten_bucket(olay, 0, host))


def test_allgather_more_than_64_ranks():
    rng = np.random.Generator(np.random.PCG64(14))
    world, part = 100, 1031
    host = [rng.integers(0, 2 ** 16, part + 5, dtype=np.uint64).astype(np.uint16) for _ in range(world)]
    dev = [torch.from_numpy(h.view(np.int16).copy()).cuda().view(torch.bfloat16) for h in host]
    dst = Guarded(world * part, torch.bfloat16)
    Z.zero_allgather_params(dev, 5, part, dst.t)
    torch.cuda.synchronize()
    dst.check()
    assert np.array_equal(host_u16(dst.t), oracle.allgather(host, 5, part))


def test_step_with_128_replicas():
    c = Case(128 * 1001, 128, seed=15)
    c.run(_adam())
    ref, _, _ = c.expect(_adam())
    assert c.compare(ref) == [0, 0, 0, 0]
