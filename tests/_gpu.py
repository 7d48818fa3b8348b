"""GPU test helpers: guarded device buffers and parity assertions.

Parity bar for the fused step: partition indexing, padding, gathered layout
and the overflow flag bit-exact; fp32 master / m / v within 4 ulp or 1e-6
relative; fp16 / bf16 parameters within 1 ulp.
"""
from __future__ import annotations

import numpy as np
import torch

from _brute import f32_ulp_distance, u16_ulp_distance

GUARD = 4096            # bytes of sentinel before and after each guarded buffer
SENTINEL = 0x5A


class Guarded:
    """A device buffer with sentinel bytes on both sides.

    `elem_offset` shifts the buffer start by whole elements (to exercise the
    unaligned paths); the sentinels must be intact after every call.
    """

    def __init__(self, n: int, dtype: torch.dtype, elem_offset: int = 0, device="cuda"):
        es = torch.empty((), dtype=dtype).element_size()
        self.n, self.dtype, self.es = n, dtype, es
        self.pre = GUARD + elem_offset * es
        total = self.pre + n * es + GUARD
        self.raw = torch.full((total,), SENTINEL, dtype=torch.uint8, device=device)
        self.t = self.raw[self.pre:self.pre + n * es].view(dtype)

    def check(self) -> None:
        torch.cuda.synchronize()
        pre = self.raw[:self.pre]
        post = self.raw[self.pre + self.n * self.es:]
        assert bool((pre == SENTINEL).all()) and bool((post == SENTINEL).all()), "guard bytes overwritten"


def to_dev_u16(bits: np.ndarray, dtype: torch.dtype, buf: Guarded | None = None, elem_offset: int = 0):
    if buf is None:
        buf = Guarded(bits.size, dtype, elem_offset)
    buf.t.copy_(torch.from_numpy(bits.view(np.int16).copy()).view(dtype))
    return buf


def to_dev_f32(x: np.ndarray, buf: Guarded | None = None, elem_offset: int = 0):
    if buf is None:
        buf = Guarded(x.size, torch.float32, elem_offset)
    buf.t.copy_(torch.from_numpy(np.ascontiguousarray(x, np.float32)))
    return buf


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float32, copy=False)


def assert_f32_close(got: np.ndarray, ref: np.ndarray, what: str = "") -> int:
    """fp32 parity: ulp <= 4 or relative <= 1e-6.  Returns #elements not bit-equal."""
    assert got.shape == ref.shape, what
    got = np.ascontiguousarray(got, np.float32)
    ref = np.ascontiguousarray(ref, np.float32)
    if np.array_equal(got.view(np.uint32), ref.view(np.uint32)):
        return 0                    # bit-equal: within any tolerance (fast path for large arrays)
    ulp = f32_ulp_distance(got, ref)
    rel = np.abs(got.astype(np.float64) - ref) / np.maximum(np.abs(ref.astype(np.float64)), 1e-38)
    ok = (ulp <= 4) | (rel <= 1e-6)
    if not ok.all():
        i = int(np.flatnonzero(~ok)[0])
        raise AssertionError(f"{what}: element {i}: got {got[i]!r} ref {ref[i]!r} ulp {ulp[i]}")
    return int((got.view(np.uint32) != ref.view(np.uint32)).sum())


def assert_u16_close(got: np.ndarray, ref: np.ndarray, what: str = "") -> int:
    """fp16 / bf16 parity: <= 1 ulp.  Returns #elements not bit-equal."""
    assert got.shape == ref.shape, what
    if np.array_equal(got, ref):
        return 0                    # bit-equal (fast path for large arrays)
    d = u16_ulp_distance(got, ref)
    if not (d <= 1).all():
        i = int(np.flatnonzero(d > 1)[0])
        raise AssertionError(f"{what}: element {i}: got {got[i]:#06x} ref {ref[i]:#06x}")
    return int((got != ref).sum())


# --------------------------------------------------- full-size workload helpers

def device_grads(buf, seed, std, scale):
    """Seeded N(0, std) x scale draws on the device, rounded to buf's dtype."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    n = buf.numel()
    chunk = 1 << 27
    for o in range(0, n, chunk):
        e = min(n, o + chunk)
        buf[o:e].copy_(torch.randn(e - o, generator=gen, device="cuda").mul_(std * scale))


def device_master(buf, seed, std=0.02):
    """Seeded fp32 N(0, std) draws on the device."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    n = buf.numel()
    for o in range(0, n, 1 << 27):
        e = min(n, o + (1 << 27))
        buf[o:e].copy_(torch.randn(e - o, generator=gen, device="cuda").mul_(std))


def windows(padded, world, n_random=64, width=65_536, seed=0):
    """Sorted, disjoint [lo, hi) windows: random, partition boundaries, ends."""
    rng = np.random.Generator(np.random.PCG64(seed))
    P = padded // world
    spans = [(0, 4096), (padded - 4096, padded)]
    for r in range(1, world):
        spans.append((r * P - 4, r * P + 4))
    for lo in rng.integers(0, max(1, padded - width), n_random):
        spans.append((int(lo), int(lo) + width))
    spans = sorted((max(0, a), min(padded, b)) for a, b in spans)
    merged = []
    for a, b in spans:
        if merged and a <= merged[-1][1]:
            merged[-1] = (merged[-1][0], max(merged[-1][1], b))
        else:
            merged.append((a, b))
    return merged


def free_gb():
    """Free device memory in GB (blocks cached by earlier tests count as free)."""
    torch.cuda.empty_cache()
    free, _ = torch.cuda.mem_get_info()
    return free / 1e9
