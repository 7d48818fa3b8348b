"""ZeroStage3 (layer-wise ZeRO-3 with gather prefetch) against the oracle.

Per unit the update is the Stage-2 update of that unit's partitions (staged
reduce-scatter + update from the reduced gradients, or statistics pass +
fused gated update), so the
oracle runs flat_step per unit; the parameters read back through the
all-gather of the shards must equal the oracle's bit for bit.  Prefetch on
and off give identical bits.  An overflow injected into one unit skips that
unit's update only, keeps t and halves the loss scale.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import host_f32, host_u16

pytestmark = pytest.mark.gpu

UNITS = [50_000, 70_001, 3, 120_000]
N = 4


def _unit_grads(L, u, step, scale, inject=False):
    out = []
    for k in range(N):
        g = workloads.grads(L.bucket_padded[u], workloads.seed_for(31, step, k) + 101 * u, 1e-3, scale)
        g[L.bucket_numel[u]:] = 0
        if inject and k == 2:
            workloads.inject(g, np.array([1, 7]), np.array([True, False]))
        out.append(g)
    return out


def _run(prefetch, inject_unit=None, update="staged"):
    adam = workloads.AdamConfig(weight_decay=0.01)
    s3 = Z.ZeroStage3(UNITS, N, lr=adam.lr, betas=(adam.beta1, adam.beta2), eps=adam.eps,
                      weight_decay=adam.weight_decay, loss_scale=65536.0, prefetch=prefetch, update=update)
    L = oracle.partition_layout(UNITS, N, 1, 8)
    init = [np.concatenate([workloads.master(n, 950 + u), np.zeros(L.bucket_padded[u] - n, np.float32)])
            for u, n in enumerate(UNITS)]
    s3.load([torch.from_numpy(x).cuda() for x in init])
    results = []
    for step in (1, 2):
        scale = s3.scale

        def fill(u, bufs, step=step, scale=scale):
            for k, g in enumerate(_unit_grads(L, u, step, scale, inject=(step == 2 and u == inject_unit))):
                bufs[k][:g.size].copy_(torch.from_numpy(g.view(np.int16)).cuda().view(torch.float16))
        applied = s3.step(fill)
        results.append(applied)
    params = [host_u16(s3.unit_params(u)) for u in range(len(UNITS))]
    states = [(host_f32(s3.master[u]), host_f32(s3.m[u]), host_f32(s3.v[u])) for u in range(len(UNITS))]
    assert s3.gathers == 2 * 2 * len(UNITS)
    return s3, L, init, results, params, states


@pytest.mark.parametrize("update", ["staged", "stats"])
@pytest.mark.parametrize("inject_unit", [None, 1])
def test_stage3_matches_oracle_and_prefetch_is_exact(inject_unit, update):
    s3a, L, init, res_a, par_a, st_a = _run(True, inject_unit, update)
    s3b, _, _, res_b, par_b, st_b = _run(False, inject_unit, update)
    assert res_a == res_b
    for x, y in zip(par_a, par_b):
        assert np.array_equal(x, y)
    for xs, ys in zip(st_a, st_b):
        for x, y in zip(xs, ys):
            assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
    # oracle, unit by unit
    adam = workloads.AdamConfig(weight_decay=0.01)
    for u in range(len(UNITS)):
        st = oracle.initial_state(init[u])
        scale, t = 65536.0, 0
        for step in (1, 2):
            G = _unit_grads(L, u, step, scale, inject=(step == 2 and u == inject_unit))
            ovf, _ = oracle.flat_step(G, st, adam, t + 1, scale, float(N))
            all_ok = not (step == 2 and inject_unit is not None)
            if all_ok:
                t += 1
            scale = scale if all_ok else scale / 2
        assert np.array_equal(st_a[u][0].view(np.uint32), st.master.view(np.uint32)), u
        assert np.array_equal(st_a[u][1].view(np.uint32), st.m.view(np.uint32)), u
        assert np.array_equal(st_a[u][2].view(np.uint32), st.v.view(np.uint32)), u
        assert np.array_equal(par_a[u], st.params), u
    if inject_unit is None:
        assert res_a == [True, True] and s3a.t == 2 and s3a.scale == 65536.0
    else:
        assert res_a == [True, False] and s3a.t == 1 and s3a.scale == 32768.0
