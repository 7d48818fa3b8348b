"""Pins of the oracle's Adam / AdamW update.

The pages name Adam and its fp32 states but print no formula, so the oracle
takes Adam with bias correction and epsilon outside the square root (Kingma &
Ba) with decoupled weight decay.  Pins:
  - the step-1 closed form m_hat / (sqrt(v_hat) + eps) = g / (|g| + eps);
  - a constant gradient gives the same update at every step;
  - torch.optim.AdamW (a library routine) on the CPU, fp32;
  - an fp64 textbook restatement, element by element, on tiny inputs;
  - special cases: zero gradient, zero learning rate, padding stays zero.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from _brute import adamw_textbook, f32_ulp_distance, u16_ulp_distance


def _cfg(wd=0.0, lr=1e-3):
    return workloads.AdamConfig(lr=lr, weight_decay=wd)


def _step(s, state, cfg, t, divisor, scale, pdtype=oracle.F16):
    c = oracle.adam_constants(cfg, t, divisor, scale)
    oracle.adam_update(s, c, state.master, state.m, state.v, state.params, pdtype)
    return c


def test_constants_are_rounded_from_double():
    cfg = workloads.AdamConfig(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    c = oracle.adam_constants(cfg, 3, 8.0, 65536.0)
    b1, b2 = float(np.float32(0.9)), float(np.float32(0.999))
    lr = float(np.float32(1e-3))
    assert c[4] == np.float32(1.0 / (8 * 65536.0))
    assert c[5] == np.float32(1.0 - b1) and c[6] == np.float32(1.0 - b2)
    assert c[7] == np.float32(1.0 / (1.0 - b1 ** 3))
    assert c[8] == np.float32(1.0 / math.sqrt(1.0 - b2 ** 3))
    assert c[9] == np.float32(1.0 - lr * float(np.float32(0.01)))


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_step1_closed_form(wd):
    n = 50_000
    G = [workloads.grads(n, 100 + k, 1e-3, 1024.0) for k in range(4)]
    st = oracle.initial_state(workloads.master(n, 7))
    p0 = st.master.astype(np.float64).copy()
    s = oracle.reduce(G)
    cfg = _cfg(wd)
    c = _step(s, st, cfg, 1, 4.0, 1024.0)
    g = s.astype(np.float64) * float(c[4])
    lr = float(np.float32(cfg.lr))
    decay = 1.0 - lr * float(np.float32(wd))
    eps = float(np.float32(cfg.eps))
    expect = p0 * decay - lr * g / (np.abs(g) + eps)
    # error budget in units u = 2^-24: u = m_hat/(sqrt(v_hat)+eps) carries
    # about eight fp32 roundings (ops and the rounded constants 1-b1,
    # 1/(1-b1^t), 1/sqrt(1-b2^t)), p*decay two, the final fma one
    u = 2.0 ** -24
    err = np.abs(st.master.astype(np.float64) - expect)
    bound = 2 * u * np.abs(p0) + 8 * u * lr + u * np.abs(expect)
    assert (err <= bound).all()
    # m and v after one step from zero
    b1, b2 = float(np.float32(cfg.beta1)), float(np.float32(cfg.beta2))
    assert (f32_ulp_distance(st.m, (1 - b1) * g) <= 2).all()
    assert (f32_ulp_distance(st.v, (1 - b2) * g * g) <= 4).all()


def test_constant_gradient_gives_constant_update():
    n = 4096
    g16 = workloads.grads(n, 150, 1e-3, 1.0)
    st = oracle.initial_state(np.zeros(n, np.float32))
    cfg = _cfg(0.0, lr=1e-3)
    prev = st.master.astype(np.float64).copy()
    g = g16.view(np.float16).astype(np.float64)
    expect_u = g / (np.abs(g) + float(np.float32(1e-8)))
    for t in range(1, 6):
        _step(oracle.reduce([g16]), st, cfg, t, 1.0, 1.0)
        du = (prev - st.master.astype(np.float64)) / float(np.float32(1e-3))
        assert np.allclose(du, expect_u, rtol=2e-5, atol=1e-6), t
        prev = st.master.astype(np.float64).copy()


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_matches_torch_adamw_cpu(wd):
    n = 20_000
    steps = 4
    cfg = _cfg(wd)
    m0 = workloads.master(n, 8)
    st = oracle.initial_state(m0)
    p = torch.nn.Parameter(torch.from_numpy(m0.copy()))
    f32 = lambda x: float(np.float32(x))      # the oracle's hyper-parameters are fp32
    opt = torch.optim.AdamW([p], lr=f32(cfg.lr), betas=(f32(cfg.beta1), f32(cfg.beta2)),
                            eps=f32(cfg.eps), weight_decay=f32(wd), foreach=False, fused=False)
    mag = np.zeros(n)          # running sum of |terms| of m: the scale of its rounding error
    for t in range(1, steps + 1):
        g16 = workloads.grads(n, 200 + t, 1e-3, 1.0)
        s = oracle.reduce([g16])
        _step(s, st, cfg, t, 1.0, 1.0)
        p.grad = torch.from_numpy(s.copy())
        opt.step()
        mag = 0.9 * mag + 0.1 * np.abs(s)
    state = opt.state[p]
    ref_p = p.detach().numpy()
    ref_m = state["exp_avg"].numpy()
    ref_v = state["exp_avg_sq"].numpy()
    # Same mathematics, different rounding order (lerp, division by the bias
    # corrections).  Master weights agree to a few ulp; m and v to a few ulp
    # except where b1*m and (1-b1)*g nearly cancel, where the bound is the
    # size of the terms.
    # Each step the two differ by a few roundings of lr*u plus the rounding of
    # p; near zero the ulp is tiny, so the bound is absolute in lr*u.
    u = 2.0 ** -24
    lr = float(np.float32(cfg.lr))
    diff = np.abs(st.master.astype(np.float64) - ref_p)
    assert (diff <= steps * (8 * u * lr + 2 * u * np.abs(ref_p))).all()
    assert np.median(f32_ulp_distance(st.master, ref_p)) <= 1
    assert (np.abs(st.m - ref_m) <= 4 * u * mag * steps).all()
    assert (f32_ulp_distance(st.v, ref_v) <= 8).all()


def test_fp64_textbook_brute_force():
    # tiny buckets, several replicas, several steps, AdamW
    rng = np.random.Generator(np.random.PCG64(9))
    for N, n, wd in [(1, 17, 0.0), (3, 29, 0.01), (5, 64, 0.01)]:
        cfg = _cfg(wd)
        m0 = workloads.master(n, 300 + N)
        st = oracle.initial_state(m0)
        bp = [float(x) for x in m0]
        bm = [0.0] * n
        bv = [0.0] * n
        scale = 1024.0
        f = lambda x: float(np.float32(x))
        for t in range(1, 4):
            G = [workloads.grads(n, 400 + 10 * t + k, 1e-3, scale) for k in range(N)]
            s = oracle.reduce(G)
            _step(s, st, cfg, t, float(N), scale)
            for j in range(n):
                gj = sum(float(np.float16(G[k].view(np.float16)[j])) for k in range(N)) / (N * scale)
                bp[j], bm[j], bv[j] = adamw_textbook(bp[j], bm[j], bv[j], gj, t, f(cfg.lr),
                                                     f(cfg.beta1), f(cfg.beta2), f(cfg.eps), f(wd))
        bp, bm, bv = map(np.array, (bp, bm, bv))
        assert np.allclose(st.master, bp, rtol=2e-6, atol=1e-9), N
        assert np.allclose(st.m, bm, rtol=1e-4, atol=1e-6 * np.abs(bm).max()), N
        assert np.allclose(st.v, bv, rtol=1e-5, atol=1e-6 * np.abs(bv).max()), N
        # parameters: the rounding of the master copy
        ref16 = bp.astype(np.float32).astype(np.float16).view(np.uint16)
        assert u16_ulp_distance(st.params, ref16).max() <= 1


def test_zero_gradient_keeps_moments_and_decays_weights():
    n = 1000
    m0 = workloads.master(n, 10)
    st = oracle.initial_state(m0)
    cfg = _cfg(0.01)
    c = _step(np.zeros(n, np.float32), st, cfg, 1, 1.0, 1.0)
    assert (st.m == 0).all() and (st.v == 0).all()
    assert np.array_equal(st.master, (m0 * c[9]).astype(np.float32))


def test_zero_lr_changes_no_weight():
    n = 1000
    m0 = workloads.master(n, 11)
    st = oracle.initial_state(m0)
    _step(oracle.reduce([workloads.grads(n, 12, 1e-3, 1.0)]), st, _cfg(0.0, lr=0.0), 1, 1.0, 1.0)
    assert np.array_equal(st.master, m0)


def test_padding_stays_zero():
    n = 64
    st = oracle.initial_state(np.zeros(n, np.float32))
    for t in range(1, 4):
        _step(np.zeros(n, np.float32), st, _cfg(0.01), t, 4.0, 65536.0)
    assert not st.master.any() and not st.m.any() and not st.v.any() and not st.params.any()


def test_bf16_parameters_are_rounded_master():
    n = 5000
    st = oracle.initial_state(workloads.master(n, 13), oracle.BF16)
    G = [workloads.grads(n, 14 + k, 1e-3, 1024.0, oracle.BF16) for k in range(2)]
    _step(oracle.reduce(G, oracle.BF16), st, _cfg(), 1, 2.0, 1024.0, oracle.BF16)
    ref = torch.from_numpy(st.master.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(st.params, ref)
