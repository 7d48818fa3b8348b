"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (every rank's partition in one launch per bucket).

- GPT-2 1.5B parameter list, 4 buckets of <= 500M elements, N = 8, AdamW,
  5 steps: sampled windows (seeded windows, every partition and bucket
  boundary, first and last elements) against the oracle run on the same
  windows; the overflow flag is 0 at every step, as it must be for finite
  fp16 gradients (8 x 65504 cannot overflow fp32).
- Dynamic loss-scale workload: flat 100M elements, N = 16, 6 steps, +inf /
  NaN injected at 17 positions at steps 2 and 4: full arrays against the
  oracle, flag bit-exact, skipped steps leave every state bit-identical,
  scale 65536 -> 32768 -> 16384.
- Stage 3 layer-wise path on the 6.7B GPT shape, N = 8, fp16 and bf16, three
  steps: per unit and step an all-gather of the unit's parameters from 8
  rank-major shards into a reused layer buffer, then one fused call per rank
  writing its updated parameters into its own shard, moments carried between
  steps; windows against the oracle, whole gathered units bit-exact.
- Flat bandwidth-sweep points: windows.
- The staged route on a bucket past 2^31 elements (64-bit indexing) and on a
  bf16 N = 16 point: windows of the reduced gradients, states, parameters.
- The native runner with buckets that take different step kernels in one
  step (pipeline or register beside oct): windows over two steps, then a
  skipped step that leaves every bank bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import (assert_f32_close, assert_u16_close, device_grads as _device_grads,
                  device_master as _device_master, free_gb as _free_gb, host_f32, host_u16,
                  windows as _windows)

pytestmark = pytest.mark.gpu

TD = {oracle.F16: torch.float16, oracle.BF16: torch.bfloat16}


def _u16(t):
    return host_u16(t)


@pytest.mark.skipif(not torch.cuda.is_available() or _free_gb() < 80, reason="needs ~70 GB of HBM")
@pytest.mark.parametrize("mode", ["banks", "staged"])
def test_gpt2_1p5b_windows_five_steps(mode):
    w = workloads.gpt2_1p5b()
    opt = Z.ZeroAdam(w.numels, w.world, w.bucket_elems, lr=w.adam.lr, betas=(w.adam.beta1, w.adam.beta2),
                     eps=w.adam.eps, weight_decay=w.adam.weight_decay, loss_scale=w.loss_scale, mode=mode)
    L = opt.layout
    wins, refs = [], []
    for b in range(L.n_buckets):
        _device_master(opt.master[b][0], 700 + b)
        opt.master[b][0][L.bucket_numel[b]:].zero_()
        opt.params_bank[b][0].copy_(opt.master[b][0])
        for extra in range(1, len(opt.master[b])):
            opt.master[b][extra].copy_(opt.master[b][0])
            opt.params_bank[b][extra].copy_(opt.params_bank[b][0])
        wb = _windows(L.bucket_padded[b], w.world, n_random=16, seed=b)
        wins.append(wb)
        # the oracle's state on the windows, from the device's initial values
        refs.append([oracle.FlatState(host_f32(opt.master[b][0][lo:hi]).copy(),
                                      np.zeros(hi - lo, np.float32), np.zeros(hi - lo, np.float32),
                                      _u16(opt.params_bank[b][0][lo:hi]).copy()) for lo, hi in wb])
    for step in range(1, w.steps + 1):
        win_grads = []
        for b in range(L.n_buckets):
            for k in range(w.world):
                _device_grads(opt.grads[b][k], workloads.seed_for(w.seed, step, k) + 31 * b, w.grad_std, w.loss_scale)
                opt.grads[b][k][L.bucket_numel[b]:].zero_()
            win_grads.append([[_u16(opt.grads[b][k][lo:hi]) for k in range(w.world)] for lo, hi in wins[b]])
        assert opt.step(), f"unexpected overflow at step {step}"
        assert int(opt.flag.item()) == 0
        for b in range(L.n_buckets):
            for (lo, hi), G, st in zip(wins[b], win_grads[b], refs[b]):
                ovf, _ = oracle.flat_step(G, st, w.adam, step, w.loss_scale, float(w.world))
                assert ovf == 0
    for b in range(L.n_buckets):
        master, m, v, p = opt.state(b)
        for (lo, hi), st in zip(wins[b], refs[b]):
            assert assert_f32_close(host_f32(master[lo:hi]), st.master, "master") == 0
            assert assert_f32_close(host_f32(m[lo:hi]), st.m, "m") == 0
            assert assert_f32_close(host_f32(v[lo:hi]), st.v, "v") == 0
            assert assert_u16_close(_u16(p[lo:hi]), st.params, "params") == 0
    assert opt.t == w.steps and opt.scale == w.loss_scale


@pytest.mark.skipif(not torch.cuda.is_available() or _free_gb() < 12, reason="needs ~8 GB of HBM")
@pytest.mark.parametrize("mode", ["banks", "staged", "inplace"])
def test_overflow_workload_full_arrays(mode):
    w = workloads.overflow_flat()
    (psi,) = w.numels
    N = w.world
    opt = Z.ZeroAdam([psi], N, lr=w.adam.lr, betas=(w.adam.beta1, w.adam.beta2), eps=w.adam.eps,
                     weight_decay=w.adam.weight_decay, loss_scale=w.loss_scale, track_grad_norm=True, mode=mode)
    padded = opt.layout.bucket_padded[0]
    assert padded == psi
    _device_master(opt.master[0][0], 900)
    opt.params_bank[0][0].copy_(opt.master[0][0])
    for extra in range(1, len(opt.master[0])):
        opt.master[0][extra].copy_(opt.master[0][0])
        opt.params_bank[0][extra].copy_(opt.params_bank[0][0])
    ref = oracle.FlatState(host_f32(opt.master[0][0]).copy(), np.zeros(psi, np.float32),
                           np.zeros(psi, np.float32), _u16(opt.params_bank[0][0]).copy())
    scaler = oracle.Scaler(w.loss_scale)
    scales = []
    for step in range(1, w.steps + 1):
        G = []
        for k in range(N):
            _device_grads(opt.grads[0][k], workloads.seed_for(w.seed, step, k), w.grad_std, opt.scale)
            G.append(_u16(opt.grads[0][k]))
        injected = step in (2, 4)
        if injected:
            rep, pos, is_inf = workloads.injection_sites(psi, step, N)
            workloads.inject(G[rep], pos, is_inf)
            opt.grads[0][rep].copy_(torch.from_numpy(G[rep].view(np.int16)).cuda().view(torch.float16))
        before = [x.clone() for x in opt.state(0)]
        applied = opt.step()
        s = oracle.reduce(G)
        ovf = oracle.any_nonfinite(s)
        assert ovf == int(injected) and applied == (not ovf) and int(opt.flag.item()) == ovf
        if not ovf:
            c = oracle.adam_constants(w.adam, scaler.t + 1, float(N), scaler.scale)
            sq = oracle.grad_sqnorm(s, c[4])
            oracle.adam_update(s, c, ref.master, ref.m, ref.v, ref.params)
            scaler.t += 1
            assert abs(opt.grad_sqnorm() - sq) <= 1e-5 * sq
        else:
            for x, y in zip(before, opt.state(0)):
                assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
        scaler.scale, scaler.good_steps = oracle.loss_scale_update(scaler.scale, scaler.good_steps, bool(ovf))
        assert opt.scale == scaler.scale and opt.t == scaler.t
        scales.append(opt.scale)
        master, m, v, p = opt.state(0)
        assert assert_f32_close(host_f32(master), ref.master, "master") == 0
        assert assert_f32_close(host_f32(m), ref.m, "m") == 0
        assert assert_f32_close(host_f32(v), ref.v, "v") == 0
        assert assert_u16_close(_u16(p), ref.params, "params") == 0
    assert scales == [65536.0, 32768.0, 32768.0, 16384.0, 16384.0, 16384.0]
    assert opt.t == 4


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_stage3_layerwise_6p7b(dtype):
    """Stage 3 on the 6.7B GPT shape, three steps (t = 1, 2, 3).

    Per unit and step: the all-gather of the unit's parameters from the 8
    rank-major shards into the reused layer buffer (after step 1 these are the
    parameters the previous step wrote into the shards, so the gather is
    checked against the oracle's parameters of that step), fresh seeded
    gradients, then one fused call per rank reading the unit's fp32 state and
    writing the rotating spare bank and rank r's shard; the banks swap, so m
    and v carry over and steps 2 and 3 read non-zero moments with t > 1 bias
    corrections.  Units are independent (no overflow, the same t for every
    unit), so each unit runs its three steps before the next unit starts.

    Runs every unit when the GPU has room for the whole shard set plus one
    unit's buffers; otherwise the first, a middle and the last unit.
    """
    w = workloads.gpt_6p7b_layerwise()
    units = list(w.numels)
    N = w.world
    steps = 3
    lay = Z.zero_partition_layout(units, N, 1)
    parts = [lay.part(u) for u in range(len(units))]
    shard_off = np.concatenate([[0], np.cumsum(parts)]).astype(np.int64)
    max_pad = max(lay.bucket_padded)
    need_gb = (sum(lay.bucket_padded) * 2 + max_pad * (2 * N + 2 + 24)) / 1e9 + 6
    run_units = list(range(len(units))) if _free_gb() > need_gb else [0, 16, len(units) - 1]
    tdt = TD[dtype]
    shards = [torch.empty(int(shard_off[-1]), dtype=tdt, device="cuda") for _ in range(N)]
    layer_buf = torch.empty(max_pad, dtype=tdt, device="cuda")
    grads = [torch.empty(max_pad, dtype=tdt, device="cuda") for _ in range(N)]
    bank = [{nm: torch.empty(max_pad, dtype=torch.float32, device="cuda") for nm in ("p", "m", "v")}
            for _ in range(2)]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    adam = w.adam

    def unit_params(u, lo, hi):
        # parameters live in the shards: element i of the unit is shard i // P, slot i % P
        P = parts[u]
        pieces = []
        for r in range(lo // P, (hi - 1) // P + 1):
            a = max(lo, r * P) - r * P
            b = min(hi, (r + 1) * P) - r * P
            pieces.append(_u16(shards[r][shard_off[u] + a:shard_off[u] + b]))
        return np.concatenate(pieces)

    for u in run_units:
        pad, P = lay.bucket_padded[u], parts[u]
        st, spare = bank[0], bank[1]
        # unit u's fp32 state (flat, rank-major) and its parameter slices in the shards
        _device_master(st["p"][:pad], 1200 + u)
        st["p"][lay.bucket_numel[u]:pad].zero_()
        st["m"][:pad].zero_()
        st["v"][:pad].zero_()
        for r in range(N):
            shards[r][shard_off[u]:shard_off[u] + P].copy_(st["p"][r * P:(r + 1) * P])
        wins = _windows(pad, N, n_random=8, seed=u)
        p0 = [host_f32(st["p"][lo:hi]).copy() for lo, hi in wins]
        refs = [oracle.initial_state(x, dtype) for x in p0]
        for t in range(1, steps + 1):
            # forward/backward reconstruct: all-gather the unit into the layer buffer
            Z.zero_allgather_params(shards, int(shard_off[u]), P, layer_buf[:pad], status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            if u in (0, len(units) - 1) and t == 1:
                ref_full = oracle.allgather([_u16(s[shard_off[u]:shard_off[u] + P]) for s in shards], 0, P)
                assert np.array_equal(_u16(layer_buf[:pad]), ref_full)
            for (lo, hi), ref in zip(wins, refs):
                # the gathered layer holds the previous step's parameters (at t = 1
                # the initial ones, written into the shards above)
                assert np.array_equal(_u16(layer_buf[lo:hi]), unit_params(u, lo, hi))
                if t > 1:
                    assert assert_u16_close(_u16(layer_buf[lo:hi]), ref.params, "gathered params") == 0
            for k in range(N):
                _device_grads(grads[k][:pad], workloads.seed_for(w.seed, t, k) + 17 * u, w.grad_std, w.loss_scale)
                grads[k][lay.bucket_numel[u]:pad].zero_()
            flag.zero_()
            hp = Z.hparams(adam.lr, adam.beta1, adam.beta2, adam.eps, adam.weight_decay, t)
            # one fused call per rank: reduce-scatter slice r, update, write rank r's shard
            for r in range(N):
                sl = slice(r * P, (r + 1) * P)
                Z.zero_reduce_scatter_adam_step([g[:pad] for g in grads], pad, r,
                                                st["p"][sl], st["m"][sl], st["v"][sl],
                                                spare["p"][sl], spare["m"][sl], spare["v"][sl],
                                                shards[r][shard_off[u]:shard_off[u] + P], hp, w.loss_scale, flag)
            torch.cuda.synchronize()
            assert int(flag.item()) == 0
            for (lo, hi), ref in zip(wins, refs):
                G = [_u16(g[lo:hi]) for g in grads]
                ovf, _ = oracle.flat_step(G, ref, adam, t, w.loss_scale, float(N), dtype, dtype)
                assert ovf == 0
                what = f"unit {u} t={t}"
                assert assert_f32_close(host_f32(spare["p"][lo:hi]), ref.master, what + " master") == 0
                assert assert_f32_close(host_f32(spare["m"][lo:hi]), ref.m, what + " m") == 0
                assert assert_f32_close(host_f32(spare["v"][lo:hi]), ref.v, what + " v") == 0
                assert assert_u16_close(unit_params(u, lo, hi), ref.params, what + " params") == 0
            st, spare = spare, st


@pytest.mark.parametrize("psi,world,dtype", [(1 << 20, 64, oracle.F16), (16 << 20, 16, oracle.BF16),
                                             (256 << 20, 8, oracle.F16), (256 << 20, 2, oracle.BF16),
                                             (1 << 30, 16, oracle.BF16), (2 << 30, 4, oracle.F16)])
def test_sweep_points_windows(psi, world, dtype):
    need = psi * (2 * world + 30) / 1e9 + 2
    if _free_gb() < need:
        pytest.skip(f"needs {need:.0f} GB of HBM")
    tdt = TD[dtype]
    grads = [torch.empty(psi, dtype=tdt, device="cuda") for _ in range(world)]
    for k in range(world):
        _device_grads(grads[k], 5000 + k, 1e-3, 65536.0)
    st_in = {nm: torch.empty(psi, dtype=torch.float32, device="cuda") for nm in ("p", "m", "v")}
    _device_master(st_in["p"], 77)
    st_in["m"].zero_()
    st_in["v"].zero_()
    st_out = {nm: torch.empty_like(st_in["p"]) for nm in ("p", "m", "v")}
    params = torch.empty(psi, dtype=tdt, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    adam = workloads.AdamConfig(weight_decay=0.01)
    Z.zero_reduce_scatter_adam_step(grads, psi, Z.ZERO_ALL_PARTITIONS, st_in["p"], st_in["m"], st_in["v"],
                                    st_out["p"], st_out["m"], st_out["v"], params,
                                    Z.hparams(adam.lr, adam.beta1, adam.beta2, adam.eps, adam.weight_decay, 1),
                                    65536.0, flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    for lo, hi in _windows(psi, world, n_random=8, seed=psi + world):
        G = [_u16(g[lo:hi]) for g in grads]
        ref = oracle.initial_state(host_f32(st_in["p"][lo:hi]).copy(), dtype)
        oracle.flat_step(G, ref, adam, 1, 65536.0, float(world), dtype, dtype)
        assert assert_f32_close(host_f32(st_out["p"][lo:hi]), ref.master, "master") == 0
        assert assert_f32_close(host_f32(st_out["m"][lo:hi]), ref.m, "m") == 0
        assert assert_f32_close(host_f32(st_out["v"][lo:hi]), ref.v, "v") == 0
        assert assert_u16_close(_u16(params[lo:hi]), ref.params, "params") == 0


@pytest.mark.parametrize("psi,world,dtype", [((2 << 30) + 4 * 1001, 4, oracle.F16), (256 << 20, 16, oracle.BF16)])
def test_staged_windows_beyond_int32(psi, world, dtype):
    """The staged route (reduce-scatter to fp32, then the in-place update from
    it) on a bucket of more than 2^31 elements, as one all-partition call of
    each: windows of the reduced gradients, states and parameters against the
    oracle, including the windows past element 2^31 and the ragged end."""
    need = psi * (2 * world + 22) / 1e9 + 2
    if _free_gb() < need:
        pytest.skip(f"needs {need:.0f} GB of HBM")
    tdt = TD[dtype]
    grads = [torch.empty(psi, dtype=tdt, device="cuda") for _ in range(world)]
    for k in range(world):
        _device_grads(grads[k], 6000 + k, 1e-3, 65536.0)
    st = {nm: torch.empty(psi, dtype=torch.float32, device="cuda") for nm in ("p", "m", "v")}
    _device_master(st["p"], 78)
    st["m"].zero_()
    st["v"].zero_()
    wins = _windows(psi, world, n_random=8, seed=psi + world) + [(2 ** 31 - 8, 2 ** 31 + 8)] * (psi > 2 ** 31)
    wins = sorted(set(wins))
    start = [host_f32(st["p"][lo:hi]).copy() for lo, hi in wins]
    reduced = torch.empty(psi, dtype=torch.float32, device="cuda")
    params = torch.empty(psi, dtype=tdt, device="cuda")
    flags = torch.zeros(2, dtype=torch.int32, device="cuda")
    adam = workloads.AdamConfig(weight_decay=0.01)
    hp = Z.hparams(adam.lr, adam.beta1, adam.beta2, adam.eps, adam.weight_decay, 1)
    Z.zero_reduce_scatter_grads(grads, psi, Z.ZERO_ALL_PARTITIONS, 65536.0, reduced, flags[0:1])
    Z.zero_adam_step_reduced(reduced, psi, st["p"], st["m"], st["v"], st["p"], st["m"], st["v"], params, hp,
                             flags[1:2], gate=flags[0:1])
    torch.cuda.synchronize()
    assert flags.cpu().tolist() == [0, 0]
    inv = oracle.adam_constants(adam, 1, float(world), 65536.0)[4]
    for (lo, hi), p0 in zip(wins, start):
        G = [_u16(g[lo:hi]) for g in grads]
        s = oracle.reduce(G, dtype)
        assert np.array_equal(host_f32(reduced[lo:hi]).view(np.uint32), oracle.unscale(s, inv).view(np.uint32))
        ref = oracle.initial_state(p0, dtype)
        oracle.flat_step(G, ref, adam, 1, 65536.0, float(world), dtype, dtype)
        assert assert_f32_close(host_f32(st["p"][lo:hi]), ref.master, "master") == 0
        assert assert_f32_close(host_f32(st["m"][lo:hi]), ref.m, "m") == 0
        assert assert_f32_close(host_f32(st["v"][lo:hi]), ref.v, "v") == 0
        assert assert_u16_close(_u16(params[lo:hi]), ref.params, "params") == 0


@pytest.mark.skipif(not torch.cuda.is_available() or _free_gb() < 12, reason="needs ~6 GB of HBM")
@pytest.mark.parametrize("numels,world,kinds", [
    ([64 << 20, 1 << 20, 240_007], 8, [Z.STEP_KERNEL_PIPE, Z.STEP_KERNEL_OCT]),
    ([88 << 20, 1 << 20], 4, [Z.STEP_KERNEL_REGISTER, Z.STEP_KERNEL_OCT]),
])
def test_runner_step_with_mixed_kernels(numels, world, kinds):
    """One native-runner step whose buckets take different kernels (the
    pipeline or the register kernel on a large bucket, the oct kernel on a
    small one), sharing one overflow flag: windows against the oracle over two
    steps; then an inf in the small bucket skips the whole step, every bank
    bit-identical."""
    adam = workloads.AdamConfig(weight_decay=0.01)
    opt = Z.ZeroAdam(numels, world, 64 << 20 if world == 8 else 88 << 20, lr=adam.lr, weight_decay=adam.weight_decay,
                     loss_scale=65536.0)
    L = opt.layout
    assert opt.bucket_kernels() == kinds
    wins, refs = [], []
    for b in range(L.n_buckets):
        _device_master(opt.master[b][0], 900 + b)
        opt.master[b][0][L.bucket_numel[b]:].zero_()
        opt.params_bank[b][0].copy_(opt.master[b][0])
        opt.master[b][1].copy_(opt.master[b][0])
        opt.params_bank[b][1].copy_(opt.params_bank[b][0])
        wb = _windows(L.bucket_padded[b], world, n_random=8, seed=50 + b)
        wins.append(wb)
        refs.append([oracle.FlatState(host_f32(opt.master[b][0][lo:hi]).copy(), np.zeros(hi - lo, np.float32),
                                      np.zeros(hi - lo, np.float32), _u16(opt.params_bank[b][0][lo:hi]).copy())
                     for lo, hi in wb])
    for step in (1, 2):
        win_grads = []
        for b in range(L.n_buckets):
            for k in range(world):
                _device_grads(opt.grads[b][k], 7000 + 100 * step + 10 * b + k, 1e-3, 65536.0)
                opt.grads[b][k][L.bucket_numel[b]:].zero_()
            win_grads.append([[_u16(opt.grads[b][k][lo:hi]) for k in range(world)] for lo, hi in wins[b]])
        assert opt.step()
        for b in range(L.n_buckets):
            for G, st in zip(win_grads[b], refs[b]):
                assert oracle.flat_step(G, st, adam, step, 65536.0, float(world))[0] == 0
    for b in range(L.n_buckets):
        master, m, v, p = opt.state(b)
        for (lo, hi), st in zip(wins[b], refs[b]):
            assert assert_f32_close(host_f32(master[lo:hi]), st.master, "master") == 0
            assert assert_f32_close(host_f32(m[lo:hi]), st.m, "m") == 0
            assert assert_f32_close(host_f32(v[lo:hi]), st.v, "v") == 0
            assert assert_u16_close(_u16(p[lo:hi]), st.params, "params") == 0
    # an inf in the last bucket's last replica: nothing in any bucket changes
    before = [[x.clone() for x in opt.state(b)] for b in range(L.n_buckets)]
    small = L.n_buckets - 1
    opt.grads[small][world - 1][12345] = float("inf")
    assert not opt.step()
    assert opt.t == 2 and opt.scale == 32768.0
    for b in range(L.n_buckets):
        for x, y in zip(opt.state(b), before[b]):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
