"""Pins of the oracle's global-norm gradient clipping.

Not on the pages: the usual rule g <- g * min(1, max_norm / (||g|| + 1e-6)).
Pinned to its closed form, to the identity clip = 1, to the norm of the
clipped gradient, and to torch.nn.utils.clip_grad_norm_ followed by
torch.optim.AdamW on the CPU (library routines).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from _brute import f32_ulp_distance


@pytest.mark.parametrize("total,mx", [(4.0, 1.0), (0.25, 1.0), (1e-12, 1e-3), (7.3e5, 12.5), (1.0, 1.0)])
def test_coefficient_closed_form(total, mx):
    coef = mx / (math.sqrt(total) + 1e-6)
    assert oracle.clip_coefficient(total, mx) == np.float32(min(1.0, coef))


def test_clip_one_is_the_unclipped_update():
    n = 20_000
    G = [workloads.grads(n, 40 + k, 1e-3, 1024.0) for k in range(4)]
    s = oracle.reduce(G)
    cfg = workloads.AdamConfig(weight_decay=0.01)
    c = oracle.adam_constants(cfg, 2, 4.0, 1024.0)
    a = oracle.initial_state(workloads.master(n, 41))
    b = a.copy()
    oracle.adam_update(s, c, a.master, a.m, a.v, a.params)
    oracle.adam_update_clipped(s, c, np.float32(1.0), b.master, b.m, b.v, b.params)
    for x, y in ((a.master, b.master), (a.m, b.m), (a.v, b.v)):
        assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
    assert np.array_equal(a.params, b.params)


def test_clipped_gradient_has_the_target_norm():
    n = 50_000
    G = [workloads.grads(n, 50 + k, 1e-3, 1.0) for k in range(2)]
    s = oracle.reduce(G)
    inv = np.float32(0.5)
    total = oracle.grad_sqnorm(s, inv)
    mx = 0.25 * math.sqrt(total)
    clip = oracle.clip_coefficient(total, mx)
    g = (s * inv).astype(np.float32) * clip
    assert abs(math.sqrt(float(np.sum(g.astype(np.float64) ** 2))) - mx) <= 1e-5 * mx


def test_matches_torch_clip_then_adamw():
    n, steps, mx = 30_000, 3, 0.02
    cfg = workloads.AdamConfig(weight_decay=0.01)
    m0 = workloads.master(n, 60)
    st = oracle.initial_state(m0)
    p = torch.nn.Parameter(torch.from_numpy(m0.copy()))
    f32 = lambda x: float(np.float32(x))
    opt = torch.optim.AdamW([p], lr=f32(cfg.lr), betas=(f32(cfg.beta1), f32(cfg.beta2)), eps=f32(cfg.eps),
                            weight_decay=f32(cfg.weight_decay), foreach=False, fused=False)
    for t in range(1, steps + 1):
        s = oracle.reduce([workloads.grads(n, 70 + t, 1e-3, 1.0)])
        total = oracle.grad_sqnorm(s, np.float32(1.0))
        assert math.sqrt(total) > mx                      # clipping is active
        c = oracle.adam_constants(cfg, t, 1.0, 1.0)
        oracle.adam_update_clipped(s, c, oracle.clip_coefficient(total, mx), st.master, st.m, st.v, st.params)
        p.grad = torch.from_numpy(s.copy())
        torch.nn.utils.clip_grad_norm_([p], mx)
        opt.step()
    u = 2.0 ** -24
    lr = f32(cfg.lr)
    ref = p.detach().numpy().astype(np.float64)
    assert (np.abs(st.master - ref) <= steps * (8 * u * lr + 2 * u * np.abs(ref))).all()
    # m differs only by the rounding of the clip factor and the op order
    ref_m = opt.state[p]["exp_avg"].numpy()
    assert np.allclose(st.m, ref_m, rtol=1e-5, atol=1e-6 * np.abs(ref_m).max())
    assert np.median(f32_ulp_distance(st.master, p.detach().numpy())) <= 1
