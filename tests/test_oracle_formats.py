"""Pins of the oracle's storage-format conversions (binary16 / bfloat16).

The oracle writes both conversions from the IEEE 754 definition; they are
pinned here to brute force over every binary16 pattern and to library
round-to-nearest-even conversions (numpy float16, torch bfloat16 on the CPU).
"""
import math

import numpy as np
import torch

import oracle
from _brute import f16_bits_to_float, bf16_bits_to_float

pytestmark = []


def test_f16_to_f32_every_pattern_brute_force():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.to_f32(bits, oracle.F16)
    for h in range(0, 65536, 1):
        ref = f16_bits_to_float(h)
        g = float(got[h])
        if math.isnan(ref):
            assert math.isnan(g), hex(h)
        else:
            assert g == ref and math.copysign(1, g) == math.copysign(1, ref), hex(h)


def test_f16_to_f32_matches_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.to_f32(bits, oracle.F16)
    ref = bits.view(np.float16).astype(np.float32)
    same = (got.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def _f32_edge_values():
    vals = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.996, 65520.0, 65536.0, 1e9, -1e9,
            2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -26, 2.0 ** -14,
            2.0 ** -14 * (1 - 2.0 ** -11), 2.0 ** -15, 3 * 2.0 ** -25, 5 * 2.0 ** -25,
            1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 1.0 + 2.0 ** -11 + 2.0 ** -20,
            float(np.finfo(np.float32).tiny), 1e-45, 3.4e38, math.inf, -math.inf]
    return np.array(vals, dtype=np.float32)


def test_f32_to_f16_rne_matches_numpy():
    rng = np.random.Generator(np.random.PCG64(11))
    # random bit patterns cover every exponent, plus values near the f16 range
    x = rng.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    x = np.concatenate([x, _f32_edge_values(),
                        rng.standard_normal(500_000).astype(np.float32) * 1e-5,
                        rng.standard_normal(500_000).astype(np.float32) * 3e4])
    finite = np.isfinite(x) | np.isinf(x)
    x = x[finite]
    got = oracle.from_f32(x, oracle.F16)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_f32_to_f16_nan_stays_nan():
    x = np.array([np.nan, -np.nan], dtype=np.float32)
    got = oracle.from_f32(x, oracle.F16).view(np.float16)
    assert np.isnan(got).all()


def test_f32_to_f16_ties_to_even():
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: even significand wins (1.0)
    # 1 + 3*2^-11 lies halfway between 1+2^-10 and 1+2^-9: even wins (1 + 2^-9)
    x = np.array([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -25, 3 * 2.0 ** -25], np.float32)
    got = oracle.from_f32(x, oracle.F16)
    assert got.tolist() == [0x3C00, 0x3C02, 0x0000, 0x0002]


def test_f32_to_bf16_rne_matches_torch():
    rng = np.random.Generator(np.random.PCG64(12))
    x = rng.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    x = np.concatenate([x, _f32_edge_values(), np.array([3.3895314e38, 3.4028235e38], np.float32)])
    x = x[~np.isnan(x)]
    got = oracle.from_f32(x, oracle.BF16)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_to_f32_every_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.to_f32(bits, oracle.BF16)
    for h in range(0, 65536, 97):
        ref = bf16_bits_to_float(h)
        g = float(got[h])
        assert (math.isnan(ref) and math.isnan(g)) or g == ref
    ref_all = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    same = (got.view(np.uint32) == ref_all.view(np.uint32)) | (np.isnan(got) & np.isnan(ref_all))
    assert same.all()
