"""Pins of the oracle's gradient reduction and overflow test."""
import numpy as np
import pytest

import oracle
import workloads
from _brute import f16_bits_to_float


def test_single_replica_is_exact_conversion():
    g = workloads.grads(10_001, 1, 1e-3, 1024.0)
    s = oracle.reduce([g])
    assert np.array_equal(s, g.view(np.float16).astype(np.float32))


def test_integer_gradients_sum_exactly():
    # integer-valued binary16 inputs: every partial sum is an integer far below
    # 2^24, so fp32 adds are exact and any order gives the integer sum
    N = 7
    G = [workloads.integer_grads(4099, 20 + k) for k in range(N)]
    s = oracle.reduce(G)
    exact = sum(g.view(np.float16).astype(np.int64) for g in G)
    assert np.array_equal(s.astype(np.int64), exact)


def test_rank_order_is_left_to_right():
    # 1 + 2^-24 is a tie in fp32 and rounds to 1; adding replicas left to right
    # from replica 0 therefore gives exactly 1, whereas adding the two small
    # terms first would give 1 + 2^-23.
    one = np.array([0x3C00], np.uint16)
    tiny = np.array([0x0001], np.uint16)        # 2^-24
    assert f16_bits_to_float(0x0001) == 2.0 ** -24
    assert oracle.reduce([one, tiny, tiny])[0] == np.float32(1.0)
    assert oracle.reduce([tiny, tiny, one])[0] == np.float32(1.0 + 2.0 ** -23)


def test_reduce_scatter_slices_concatenate_to_allreduce():
    N = 5
    G = [workloads.grads(5 * 301, 40 + k, 1e-3, 65536.0) for k in range(N)]
    full = oracle.reduce(G)
    P = 301
    parts = [oracle.reduce(G, oracle.F16, r * P, P) for r in range(N)]
    assert np.array_equal(np.concatenate(parts).view(np.uint32), full.view(np.uint32))


def test_reduce_within_fp32_error_bound_of_exact_sum():
    N = 16
    G = [workloads.grads(20_000, 60 + k, 1e-3, 65536.0) for k in range(N)]
    s = oracle.reduce(G).astype(np.float64)
    xs = [g.view(np.float16).astype(np.float64) for g in G]
    exact = sum(xs)
    bound = (N - 1) * 2.0 ** -24 * sum(np.abs(x) for x in xs) * 1.0001
    assert (np.abs(s - exact) <= bound).all()


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_overflow_flag(dtype):
    G = [workloads.grads(1000, 80 + k, 1e-3, 65536.0, dtype) for k in range(4)]
    assert oracle.any_nonfinite(oracle.reduce(G, dtype)) == 0
    replica, pos, is_inf = workloads.injection_sites(1000, 2, 4)
    workloads.inject(G[replica], pos, is_inf, dtype)
    s = oracle.reduce(G, dtype)
    assert oracle.any_nonfinite(s) == 1
    bad = np.flatnonzero(~np.isfinite(s))
    assert np.array_equal(bad, pos)
    assert (np.isnan(s[pos[~is_inf]])).all()
    assert (s[pos[is_inf]] == np.inf).all()


def test_bf16_finite_inputs_can_overflow_the_sum():
    big = np.array([0x7F7F], np.uint16)         # largest finite bfloat16
    s = oracle.reduce([big, big], oracle.BF16)
    assert oracle.any_nonfinite(s) == 1 and s[0] == np.inf


def test_grad_sqnorm_matches_fp64_sum():
    G = [workloads.grads(30_000, 90 + k, 1e-3, 1024.0) for k in range(4)]
    s = oracle.reduce(G)
    inv = np.float32(1.0 / 4096.0)
    ref = float(np.sum((s.astype(np.float64) * float(inv)) ** 2))
    assert abs(oracle.grad_sqnorm(s, inv) - ref) <= 1e-12 * ref


def test_nan_alone_sets_the_flag():
    G = [workloads.grads(64, 95 + k, 1e-3, 1024.0) for k in range(3)]
    G[1][17] = workloads.F16_NAN
    s = oracle.reduce(G)
    assert np.isnan(s[17]) and oracle.any_nonfinite(s) == 1
    G[1][17] = workloads.F16_POS_INF
    G[2][17] = 0xFC00                          # -inf: inf + (-inf) is NaN
    s = oracle.reduce(G)
    assert np.isnan(s[17]) and oracle.any_nonfinite(s) == 1


@pytest.mark.parametrize("N,S", [(8, 65536.0), (16, 1024.0), (1, 1.0)])
def test_unscale_by_power_of_two_is_exact(N, S):
    # 1/(N*S) is a power of two: the unscaled gradient is s * 2^-k exactly
    G = [workloads.grads(5_003, 40 + k, 1e-3, S) for k in range(N)]
    s = oracle.reduce(G)
    k = int(np.log2(N * S))
    g = oracle.unscale(s, 2.0 ** -k)
    assert np.array_equal(g, np.ldexp(s, -k).astype(np.float32))


def test_unscale_is_the_correctly_rounded_product():
    # inv = 1/(3 * 1000) is not a power of two; the product of two fp32
    # values is exact in fp64 (48 significant bits), so the fp32 result must
    # be that exact product rounded once to nearest
    s = oracle.reduce([workloads.grads(20_011, 60 + k, 1e-3, 1000.0) for k in range(3)])
    inv = np.float32(1.0 / 3000.0)
    g = oracle.unscale(s, float(inv))
    exact = s.astype(np.float64) * np.float64(inv)
    assert np.array_equal(g, exact.astype(np.float32))
    assert not np.array_equal(g, s)
