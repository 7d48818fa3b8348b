"""Pins: ZeRO-DP stages compute exactly what plain data parallelism computes.

The pages call ZeRO a drop-in replacement for data parallelism that keeps its
execution pattern [ZeRO explainer, results paragraph; ZeRO method record,
description].  Partitioning only moves who computes which element, so Stage
1, 2 and 3 must give bit-identical states to plain all-reduce + full Adam on
every replica, after every step.  A wrong partition index, a wrong shard
offset or a missing all-gather breaks this equality.
"""
import numpy as np
import pytest

import oracle
import workloads


def _runs(numels, world, cap, adam, scale, gdtype, pdtype, seed, stages=(0, 1, 2, 3)):
    L = oracle.partition_layout(numels, world, cap)
    tensors = [workloads.master(n, seed + i) for i, n in enumerate(numels)]
    init = [oracle.flatten_bucket(L, b, tensors, np.float32) for b in range(L.n_buckets)]
    runs = {st: oracle.StageRun(st, L, init, adam, oracle.Scaler(scale), gdtype, pdtype)
            for st in stages}
    return L, runs


def _grads(L, step, seed, scale, gdtype, numels):
    out = []
    for b in range(L.n_buckets):
        per = []
        for k in range(L.world):
            g = workloads.grads(L.bucket_padded[b], workloads.seed_for(seed, step, k) + 7 * b,
                                1e-3, scale, gdtype)
            g[L.bucket_numel[b]:] = 0          # padding carries no gradient
            per.append(g)
        out.append(per)
    return out


def _assert_equal_states(a, b):
    for name in ("master", "m", "v"):
        assert np.array_equal(getattr(a, name).view(np.uint32), getattr(b, name).view(np.uint32)), name
    assert np.array_equal(a.params, b.params)


@pytest.mark.parametrize("world,numels,cap", [
    (4, [10_007], 0),                         # odd size, padding
    (3, [5, 1000, 17, 333, 2, 4096], 1500),   # several buckets, N not a power of two
    (8, [64, 64, 8], 0),
    (1, [999], 0),
])
@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_stages_equal_plain_dp_bit_exact(world, numels, cap, dtype):
    adam = workloads.AdamConfig(weight_decay=0.01)
    L, runs = _runs(numels, world, cap, adam, 1024.0, dtype, dtype, 50)
    for step in range(1, 4):
        G = _grads(L, step, 50, 1024.0, dtype, numels)
        flags = {st: r.step(G) for st, r in runs.items()}
        assert set(flags.values()) == {0}
        for st in (1, 2, 3):
            for b in range(L.n_buckets):
                _assert_equal_states(runs[0].flat_state(b), runs[st].flat_state(b))
        for r in runs.values():
            assert r.replicas_identical()
    assert runs[3].gathers == 2 * world * L.n_buckets * 3


def test_tiny_flat_workload_three_steps_all_stages():
    w = workloads.tiny_flat()
    L, runs = _runs(list(w.numels), w.world, w.bucket_elems, w.adam, w.loss_scale,
                    oracle.F16, oracle.F16, w.seed)
    assert L.bucket_padded == [1_000_004]
    for step in range(1, w.steps + 1):
        G = _grads(L, step, w.seed, w.loss_scale, oracle.F16, list(w.numels))
        for r in runs.values():
            assert r.step(G) == 0
        for st in (1, 2, 3):
            _assert_equal_states(runs[0].flat_state(0), runs[st].flat_state(0))
    # padding element stays zero
    fs = runs[2].flat_state(0)
    assert fs.master[-1] == 0 and fs.m[-1] == 0 and fs.v[-1] == 0 and fs.params[-1] == 0


def test_flat_step_equals_stage2():
    w = workloads.tiny_flat()
    n = 40_000
    L, runs = _runs([n], 4, 0, w.adam, 1024.0, oracle.F16, oracle.F16, 77, stages=(2,))
    st = oracle.initial_state(workloads.master(n, 77))
    for step in range(1, 3):
        G = _grads(L, step, 77, 1024.0, oracle.F16, [n])
        runs[2].step(G)
        ovf, _ = oracle.flat_step(G[0], st, w.adam, step, 1024.0, 4.0)
        assert ovf == 0
    _assert_equal_states(runs[2].flat_state(0), st)
    # the same on a window of elements
    st2 = oracle.initial_state(workloads.master(n, 77))
    lo, cnt = 12_345, 777
    win = oracle.FlatState(st2.master[lo:lo + cnt].copy(), st2.m[lo:lo + cnt].copy(),
                           st2.v[lo:lo + cnt].copy(), st2.params[lo:lo + cnt].copy())
    for step in range(1, 3):
        G = _grads(L, step, 77, 1024.0, oracle.F16, [n])
        oracle.flat_step(G[0], win, w.adam, step, 1024.0, 4.0, begin=lo, count=cnt)
    assert np.array_equal(win.master, st.master[lo:lo + cnt])
    assert np.array_equal(win.params, st.params[lo:lo + cnt])


def test_overflow_skips_update_and_halves_scale():
    # the dynamic loss-scale workload at a small size: N = 16, injections at
    # steps 2 and 4, six steps, scale from 65536
    N, n = 16, 20_000
    adam = workloads.AdamConfig()
    L, runs = _runs([n], N, 0, adam, 65536.0, oracle.F16, oracle.F16, 3, stages=(0, 2, 3))
    scales = []
    for step in range(1, 7):
        scale = runs[2].scaler.scale
        G = _grads(L, step, 3, scale, oracle.F16, [n])
        injected = step in (2, 4)
        if injected:
            rep, pos, is_inf = workloads.injection_sites(n, step, N)
            workloads.inject(G[0][rep], pos, is_inf)
        before = runs[2].flat_state(0)
        t_before = runs[2].scaler.t
        flags = {st: r.step(G) for st, r in runs.items()}
        assert set(flags.values()) == {int(injected)}
        after = runs[2].flat_state(0)
        if injected:
            _assert_equal_states(before, after)
            assert runs[2].scaler.t == t_before
        else:
            assert not np.array_equal(before.master, after.master)
            assert runs[2].scaler.t == t_before + 1
        _assert_equal_states(runs[0].flat_state(0), after)
        _assert_equal_states(runs[3].flat_state(0), after)
        scales.append(runs[2].scaler.scale)
    assert scales == [65536.0, 32768.0, 32768.0, 16384.0, 16384.0, 16384.0]
    assert runs[2].scaler.t == 4


def test_loss_scale_rule():
    s, g = 8.0, 0
    s, g = oracle.loss_scale_update(s, g, True)
    assert (s, g) == (4.0, 0)
    s, g = oracle.loss_scale_update(1.0, 5, True)
    assert (s, g) == (1.0, 0)
    s, g = 2.0, 0
    for _ in range(2):
        s, g = oracle.loss_scale_update(s, g, False, growth_interval=3)
    assert (s, g) == (2.0, 2)
    s, g = oracle.loss_scale_update(s, g, False, growth_interval=3)
    assert (s, g) == (4.0, 0)
