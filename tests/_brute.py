"""Brute-force restatements used to pin the oracle (test helpers, not product).

Everything here is written independently of `oracle/`: textbook formulas in
Python float (fp64) scalars, element by element, for tiny inputs only.
"""
from __future__ import annotations

import math
import struct


def f16_bits_to_float(h: int) -> float:
    """binary16 bits -> Python float, from the IEEE 754 field definition."""
    sign = -1.0 if (h >> 15) & 1 else 1.0
    e = (h >> 10) & 0x1F
    f = h & 0x3FF
    if e == 0x1F:
        return sign * math.inf if f == 0 else math.nan
    if e == 0:
        return sign * f * 2.0 ** -24
    return sign * (1.0 + f / 1024.0) * 2.0 ** (e - 15)


def bf16_bits_to_float(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (b & 0xFFFF) << 16))[0]


def adamw_textbook(p: float, m: float, v: float, g: float, t: int, lr: float, b1: float,
                   b2: float, eps: float, wd: float):
    """Kingma & Ba Adam with bias correction, decoupled weight decay, in fp64.

    m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
    m_hat = m / (1 - b1^t) ;  v_hat = v / (1 - b2^t)
    p <- p (1 - lr wd) - lr m_hat / (sqrt(v_hat) + eps)
    """
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    m_hat = m / (1.0 - b1 ** t)
    v_hat = v / (1.0 - b2 ** t)
    p = p * (1.0 - lr * wd) - lr * m_hat / (math.sqrt(v_hat) + eps)
    return p, m, v


def f32_ulp_distance(a, b):
    """Integer ulp distance between float32 arrays (+0 and -0 are equal)."""
    import numpy as np
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    # map sign-magnitude to a monotone integer line
    a = np.where(a < 0, -(a & 0x7FFFFFFF), a)
    b = np.where(b < 0, -(b & 0x7FFFFFFF), b)
    return np.abs(a - b)


def u16_ulp_distance(a, b):
    """ulp distance between binary16 (or bfloat16) bit arrays of finite values."""
    import numpy as np
    a = np.asarray(a, np.uint16).astype(np.int64)
    b = np.asarray(b, np.uint16).astype(np.int64)
    a = np.where(a & 0x8000, -(a & 0x7FFF), a)
    b = np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(a - b)
