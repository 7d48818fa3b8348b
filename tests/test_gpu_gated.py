"""Parity of the statistics pass, the gated step, clipping and ZeroAdam's
in-place mode against the oracle.

- zero_grad_stats: overflow flag bit-exact, squared norm within n * 2^-53
  (relative) of the oracle's fp64 sum (each term exact in double; only the
  summation order differs), N = 1 .. 64, bf16, single partitions.
- zero_reduce_scatter_adam_step_gated: a set gate leaves every output byte
  and the call's flag untouched; a clear gate equals the plain step bit for
  bit; clipping equals the oracle's clipped update.
- ZeroAdam(mode="inplace"): one bank, statistics + gated in-place update,
  exact skip on injected inf / NaN, bit-identical to the oracle's Stage 2.
- ZeroAdam(max_grad_norm=...): clipping by the step's global norm.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import assert_f32_close, assert_u16_close, host_f32, host_u16, to_dev_u16
from test_gpu_step import TD, Case, _adam, _hp

pytestmark = pytest.mark.gpu


def _stats(c: Case, scale=None, divisor=0.0):
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    norm = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = torch.zeros(Z.zero_step_workspace_bytes(), dtype=torch.uint8, device="cuda")
    Z.zero_grad_stats([g.t for g in c.g_dev], c.padded, c.partition, c.scale if scale is None else scale,
                      flag, norm, ws, divisor)
    torch.cuda.synchronize()
    return int(flag.item()), float(norm.item())


def _norm_tol(count):
    """Relative bound between two fp64 sums of `count` exact positive terms
    added in different orders: count * 2^-53 (each addition errs by at most
    half an ulp of a partial sum, and every partial sum is below the total)."""
    return max(1e-13, count * 2.0 ** -53)


def _oracle_stats(c: Case, divisor=None):
    s = oracle.reduce(c.G, c.gdtype, c.begin, c.n)
    d = float(c.world if divisor is None else divisor)
    cst = oracle.adam_constants(_adam(), 1, d, c.scale)
    return oracle.any_nonfinite(s), oracle.grad_sqnorm(s, cst[4]), s, cst


@pytest.mark.parametrize("world,per_rank", [(1, 3_000_001), (2, 7), (4, 250_001), (8, 300_007), (16, 65_537),
                                            (64, 4099)])
def test_stats_flag_and_norm(world, per_rank):
    c = Case(world * per_rank, world, seed=400 + world, scale=65536.0)
    flag, norm = _stats(c)
    ovf, sq, _, _ = _oracle_stats(c)
    assert flag == ovf == 0
    assert abs(norm - sq) <= _norm_tol(c.n) * sq


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
@pytest.mark.parametrize("r", [-1, 1])
def test_stats_bf16_partition_and_injection(dtype, r):
    c = Case(8 * 100_003, 8, gdtype=dtype, pdtype=dtype, seed=410, partition=r, goff=1)
    flag, norm = _stats(c)
    ovf, sq, _, _ = _oracle_stats(c)
    assert flag == ovf == 0 and abs(norm - sq) <= _norm_tol(c.n) * sq
    pos = np.array([c.begin + 5, c.begin + c.n - 1])
    workloads.inject(c.G[6], pos, np.array([False, True]), dtype)
    to_dev_u16(c.G[6], TD[dtype], buf=c.g_dev[6])
    flag, _ = _stats(c)
    assert flag == 1 == _oracle_stats(c)[0]


def test_gate_set_writes_nothing():
    c = Case(8 * 300_007, 8, seed=420)
    for b in c.out_dev + [c.p_dev]:
        b.t.view(torch.uint8).fill_(0xA5)
    gate = torch.ones(1, dtype=torch.int32, device="cuda")
    norm = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = torch.zeros(Z.zero_step_workspace_bytes(), dtype=torch.uint8, device="cuda")
    c.flag.fill_(0)
    workloads.inject(c.G[0], np.array([9]), np.array([True]))     # would set the flag if it ran
    to_dev_u16(c.G[0], torch.float16, buf=c.g_dev[0])
    Z.zero_reduce_scatter_adam_step_gated([g.t for g in c.g_dev], c.padded, -1, *[b.t for b in c.in_dev],
                                          *[b.t for b in c.out_dev], c.p_dev.t, _hp(_adam(), 1), c.scale, c.flag,
                                          norm, ws, gate=gate)
    torch.cuda.synchronize()
    for b in c.out_dev + [c.p_dev]:
        assert bool((b.t.view(torch.uint8) == 0xA5).all())
        b.check()
    assert int(c.flag.item()) == 0 and float(norm.item()) == 0.0


@pytest.mark.parametrize("n,world", [(8 * 300_007, 8), (4 * 1001, 4)])
def test_gate_clear_equals_plain_step(n, world):
    c = Case(n, world, seed=430)
    gate = torch.zeros(1, dtype=torch.int32, device="cuda")
    Z.zero_reduce_scatter_adam_step_gated([g.t for g in c.g_dev], c.padded, -1, *[b.t for b in c.in_dev],
                                          *[b.t for b in c.out_dev], c.p_dev.t, _hp(_adam(), 1), c.scale, c.flag,
                                          gate=gate)
    torch.cuda.synchronize()
    ref, _, _ = c.expect(_adam())
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.parametrize("n,world,dtype", [(8 * 300_007, 8, oracle.F16), (16 * 70_001, 16, oracle.BF16),
                                           (2 * 5003, 2, oracle.F16)])
def test_clipped_step_matches_oracle(n, world, dtype):
    c = Case(n, world, gdtype=dtype, pdtype=dtype, seed=440, scale=65536.0)
    flag, norm = _stats(c)
    ovf, sq, s, cst = _oracle_stats(c)
    max_norm = 0.3 * float(np.sqrt(sq))
    total = torch.tensor([norm], dtype=torch.float64, device="cuda")
    gate = torch.zeros(1, dtype=torch.int32, device="cuda")
    adam = _adam(0.01)
    Z.zero_reduce_scatter_adam_step_gated([g.t for g in c.g_dev], c.padded, -1, *[b.t for b in c.in_dev],
                                          *[b.t for b in c.out_dev], c.p_dev.t, _hp(adam, 3), c.scale, c.flag,
                                          gate=gate, clip_sqnorm=total, max_norm=max_norm)
    torch.cuda.synchronize()
    ref = c.host.copy()
    clip = oracle.clip_coefficient(sq, np.float32(max_norm))
    assert clip < 1
    cst = oracle.adam_constants(adam, 3, float(world), c.scale)
    oracle.adam_update_clipped(s, cst, clip, ref.master, ref.m, ref.v, ref.params, dtype)
    diffs = c.compare(ref)          # within tolerance (asserted inside)
    # bit-exact whenever both sides' fp64 norms give the same fp32 clip factor
    if oracle.clip_coefficient(norm, np.float32(max_norm)) == clip:
        assert diffs == [0, 0, 0, 0], diffs


def _opt_and_oracle(numels, N, cap, adam, mode, max_norm=None):
    L = oracle.partition_layout(numels, N, cap)
    tensors = [workloads.master(n, 800 + i) for i, n in enumerate(numels)]
    opt = Z.ZeroAdam(numels, N, cap, lr=adam.lr, betas=(adam.beta1, adam.beta2), eps=adam.eps,
                     weight_decay=adam.weight_decay, loss_scale=65536.0, mode=mode, max_grad_norm=max_norm)
    params16 = [torch.from_numpy(oracle.from_f32(t, oracle.F16).view(np.int16)).cuda().view(torch.float16)
                for t in tensors]
    opt.load(params16, [torch.from_numpy(t).cuda() for t in tensors])
    init = [oracle.flatten_bucket(L, b, tensors, np.float32) for b in range(L.n_buckets)]
    states = [oracle.initial_state(init[b]) for b in range(L.n_buckets)]
    return L, opt, states


def _grads_for(L, N, step, scale):
    G = []
    for b in range(L.n_buckets):
        per = []
        for k in range(N):
            g = workloads.grads(L.bucket_padded[b], workloads.seed_for(11, step, k) + 13 * b, 1e-3, scale)
            g[L.bucket_numel[b]:] = 0
            per.append(g)
        G.append(per)
    return G


def _upload(opt, G):
    for b, per in enumerate(G):
        for k, g in enumerate(per):
            opt.grad_buffers(b)[k].copy_(torch.from_numpy(g.view(np.int16)).cuda().view(torch.float16))


@pytest.mark.parametrize("mode", ["inplace", "staged"])
@pytest.mark.parametrize("max_norm", [None, 0.3])
def test_zeroadam_one_bank_modes(mode, max_norm):
    numels = [300_000, 77, 1_200_003, 5, 250_000]
    N, cap = 8, 1_000_000
    adam = workloads.AdamConfig(weight_decay=0.01)
    L, opt, states = _opt_and_oracle(numels, N, cap, adam, mode, max_norm)
    assert all(len(bank) == 1 for bank in opt.master)          # one bank: 12 Psi/N of optimizer state
    scale, good, t = 65536.0, 0, 0
    for step in range(1, 6):
        G = _grads_for(L, N, step, scale)
        if step == 3:
            workloads.inject(G[1][4], np.array([3, 1000]), np.array([True, False]))
        _upload(opt, G)
        before = [[x.clone() for x in opt.state(b)] for b in range(L.n_buckets)]
        applied = opt.step()
        sums = [oracle.reduce(G[b]) for b in range(L.n_buckets)]
        ovf = int(any(oracle.any_nonfinite(s) for s in sums))
        assert applied == (not ovf) and ovf == (step == 3)
        if not ovf:
            t += 1
            c = oracle.adam_constants(adam, t, float(N), scale)
            clip = np.float32(1.0)
            if max_norm is not None:
                total = sum(oracle.grad_sqnorm(s, c[4]) for s in sums)
                clip = oracle.clip_coefficient(total, np.float32(max_norm))
                assert clip < 1
            for b in range(L.n_buckets):
                st = states[b]
                oracle.adam_update_clipped(sums[b], c, clip, st.master, st.m, st.v, st.params)
        else:
            for b in range(L.n_buckets):
                for x, y in zip(before[b], opt.state(b)):
                    assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
        scale, good = oracle.loss_scale_update(scale, good, bool(ovf))
        assert opt.scale == scale and opt.t == t
        for b in range(L.n_buckets):
            master, m, v, p = opt.state(b)
            st = states[b]
            assert assert_f32_close(host_f32(master), st.master, "master") == 0
            assert assert_f32_close(host_f32(m), st.m, "m") == 0
            assert assert_f32_close(host_f32(v), st.v, "v") == 0
            assert assert_u16_close(host_u16(p), st.params, "params") == 0


def test_zeroadam_banks_mode_with_clipping():
    numels = [900_001, 33, 400_000]
    N = 4
    adam = workloads.AdamConfig()
    L, opt, states = _opt_and_oracle(numels, N, 0, adam, "banks", 0.05)
    for step in range(1, 4):
        G = _grads_for(L, N, step, 65536.0)
        _upload(opt, G)
        assert opt.step()
        sums = [oracle.reduce(G[b]) for b in range(L.n_buckets)]
        c = oracle.adam_constants(adam, step, float(N), 65536.0)
        total = sum(oracle.grad_sqnorm(s, c[4]) for s in sums)
        assert abs(opt.grad_sqnorm() - total) <= _norm_tol(sum(L.bucket_padded)) * total
        clip = oracle.clip_coefficient(total, np.float32(0.05))
        for b in range(L.n_buckets):
            oracle.adam_update_clipped(sums[b], c, clip, states[b].master, states[b].m, states[b].v,
                                       states[b].params)
    for b in range(L.n_buckets):
        master, m, v, p = opt.state(b)
        assert assert_f32_close(host_f32(master), states[b].master, "master") == 0
        assert assert_u16_close(host_u16(p), states[b].params, "params") == 0


@pytest.mark.parametrize("mode", ["banks", "inplace", "staged"])
def test_checkpoint_resume_bit_identical(mode):
    """Save after step 2, reload into a fresh optimizer: steps 3-5 (one with
    an injected overflow) are bit-identical to the uninterrupted run."""
    numels = [400_000, 13, 900_001]
    N = 4
    adam = workloads.AdamConfig(weight_decay=0.01)
    L, opt, _ = _opt_and_oracle(numels, N, 500_000, adam, mode)
    grads = {}
    for step in range(1, 6):
        G = _grads_for(L, N, step, 65536.0 if step < 5 else 32768.0)
        if step == 4:
            workloads.inject(G[0][1], np.array([2]), np.array([False]))
        grads[step] = G
    for step in (1, 2):
        _upload(opt, grads[step])
        opt.step()
    sd = opt.state_dict()
    for step in (3, 4, 5):
        _upload(opt, grads[step])
        opt.step()
    L2, opt2, _ = _opt_and_oracle(numels, N, 500_000, adam, mode)
    opt2.load_state_dict(sd)
    for step in (3, 4, 5):
        _upload(opt2, grads[step])
        opt2.step()
    assert (opt.t, opt.scale, opt.good_steps) == (opt2.t, opt2.scale, opt2.good_steps) == (4, 32768.0, 1)
    for b in range(L.n_buckets):
        for x, y in zip(opt.state(b), opt2.state(b)):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


@pytest.fixture
def force_pipeline():
    Z.zero_test_force_step_kernel(Z.STEP_KERNEL_PIPE)
    try:
        yield
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


def _stats_tile(world):
    return min(8192, (180 * 1024 // (2 * 2 * world)) // 512 * 512)


@pytest.mark.parametrize("world,dtype,goff", [(8, oracle.F16, 0), (8, oracle.F16, 3), (16, oracle.BF16, 0),
                                              (1, oracle.F16, 5), (3, oracle.BF16, 1)])
def test_stats_pipeline(world, dtype, goff, force_pipeline):
    """Sizes that give every SM at least two tiles, the statistics pipeline
    kernel forced (in normal use it takes the reduce-scatter at N = 3..8 from
    128 tiles per SM, and N = 17..20), with ragged tails and (goff > 0) a
    scalar head."""
    T = _stats_tile(world)
    per_rank = (2 * 148 * T + 777) // world + 3
    c = Case(world * per_rank, world, gdtype=dtype, pdtype=dtype, seed=460 + world, goff=goff, scale=65536.0)
    flag, norm = _stats(c)
    ovf, sq, _, _ = _oracle_stats(c)
    assert flag == ovf == 0 and abs(norm - sq) <= _norm_tol(c.n) * sq
    n = c.n
    for pos, is_inf in [(np.array([n // 3]), np.array([True])), (np.array([n - 2]), np.array([False])),
                        (np.array([1]), np.array([False]))]:
        g = c.G[world - 1].copy()
        workloads.inject(c.G[world - 1], pos, is_inf, dtype)
        to_dev_u16(c.G[world - 1], TD[dtype], buf=c.g_dev[world - 1])
        flag, _ = _stats(c)
        assert flag == 1 == _oracle_stats(c)[0]
        c.G[world - 1] = g
        to_dev_u16(g, TD[dtype], buf=c.g_dev[world - 1])


@pytest.mark.parametrize("kind", [Z.STEP_KERNEL_REGISTER, Z.STEP_KERNEL_PIPE, Z.STEP_KERNEL_QUAD])
@pytest.mark.parametrize("world,goff", [(1, 0), (2, 3), (3, 0), (5, 1), (8, 0), (9, 2), (16, 0), (17, 0)])
def test_stats_every_kernel_and_world(kind, world, goff):
    """Each statistics kernel forced (where it can run the call; the quad
    kernel takes N <= 16) on a ragged size, bf16 at odd N: flag and norm
    against the oracle, then one injected inf in the last replica."""
    Z.zero_test_force_step_kernel(kind)
    try:
        dtype = oracle.BF16 if world % 2 else oracle.F16
        per_rank = 61_111 + world
        c = Case(world * per_rank, world, gdtype=dtype, pdtype=dtype, seed=470 + world, goff=goff, scale=65536.0)
        flag, norm = _stats(c)
        ovf, sq, _, _ = _oracle_stats(c)
        assert flag == ovf == 0 and abs(norm - sq) <= _norm_tol(c.n) * sq
        g = c.G[world - 1].copy()
        workloads.inject(c.G[world - 1], np.array([c.n - 5]), np.array([True]), dtype)
        to_dev_u16(c.G[world - 1], TD[dtype], buf=c.g_dev[world - 1])
        flag, _ = _stats(c)
        assert flag == 1 == _oracle_stats(c)[0]
        c.G[world - 1] = g
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


@pytest.mark.parametrize("mode", ["banks", "inplace", "staged"])
def test_step_from_host_matches_device_step(mode):
    """The end-to-end entry (pinned host gradients, per-bucket copy stream)
    gives the same bits as writing the gradients on the device first."""
    numels = [700_001, 3, 900_000]
    N = 4
    adam = workloads.AdamConfig(weight_decay=0.01)
    L, a, _ = _opt_and_oracle(numels, N, 800_000, adam, mode)
    _, b, _ = _opt_and_oracle(numels, N, 800_000, adam, mode)
    for step in range(1, 4):
        G = _grads_for(L, N, step, 65536.0)
        host = [[torch.from_numpy(g.view(np.int16)).view(torch.float16).pin_memory() for g in per] for per in G]
        _upload(a, G)
        assert a.step() and b.step_from_host(host)
    for bk in range(L.n_buckets):
        for x, y in zip(a.state(bk), b.state(bk)):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_runner_protocol_and_state():
    """The native runner: launch/commit alternate, state round-trips, and a
    step through it equals a step through the per-bucket calls."""
    numels = [500_000, 11]
    N = 4
    adam = workloads.AdamConfig(weight_decay=0.01)
    L, a, _ = _opt_and_oracle(numels, N, 0, adam, "banks")
    assert a._runner is not None
    G = _grads_for(L, N, 1, 65536.0)
    _upload(a, G)
    r = a._runner
    r.launch()
    with pytest.raises(Z.ZeroError):
        r.launch()                      # the launched step is not committed yet
    assert r.commit() is True
    with pytest.raises(Z.ZeroError):
        r.commit()                      # nothing launched
    t, scale, good, bank = r.state()
    assert (t, scale, good, bank) == (1, 65536.0, 1, 1)
    r.set_state(t, scale, good, bank)
    with pytest.raises(Z.ZeroError):
        r.set_state(1, -1.0, 0, 0)
    # the same step through the per-bucket Python path on a fresh optimizer
    _, b, _ = _opt_and_oracle(numels, N, 0, adam, "banks")
    _upload(b, G)
    b.launch()
    assert b.commit()
    for bk in range(L.n_buckets):
        a_state = [x.clone() for x in (a.master[bk][bank], a.m[bk][bank], a.v[bk][bank], a.params_bank[bk][bank])]
        for x, y in zip(a_state, b.state(bk)):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_staged_runner_protocol_and_state():
    """The native runner on the staged route: one bank, bank 0 stays current,
    an injected inf skips the step (states bit-identical), and its steps
    equal the per-bucket Python path of the same mode."""
    numels = [700_001, 13]
    N = 4
    adam = workloads.AdamConfig(weight_decay=0.01)
    L, a, _ = _opt_and_oracle(numels, N, 0, adam, "staged")
    _, b, _ = _opt_and_oracle(numels, N, 0, adam, "staged")
    assert a._runner is not None
    r = a._runner
    for step in (1, 2, 3):
        G = _grads_for(L, N, step, a.scale)
        if step == 2:
            workloads.inject(G[0][3], np.array([5]), np.array([False]))
        _upload(a, G)
        _upload(b, G)
        before = [x.clone() for x in a.state(0)]
        applied = a.step()                      # runner
        b.launch()                              # per-bucket Python path
        assert b.commit() == applied == (step != 2)
        if step == 2:
            for x, y in zip(before, a.state(0)):
                assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
        for bk in range(L.n_buckets):
            for x, y in zip(a.state(bk), b.state(bk)):
                assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    assert r.state() == (2, 32768.0, 1, 0)
    with pytest.raises(Z.ZeroError):
        r.set_state(2, 32768.0, 1, 1)           # a staged runner has one bank
