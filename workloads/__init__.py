"""Seeded synthetic inputs and model shapes for the partitioned Adam step.

This module is shared by the CPU oracle, the tests and the benchmark.  It holds
no arithmetic of the method itself: only parameter-list shapes, the
hyper-parameters of the five workloads, and seeded random draws of gradients
and master weights (already rounded to the storage dtype, as a training step
would hand them over).

Shapes follow the models the ZeRO pages name: GPT-2 1.5B (ZeRO explainer
(azimuth.plus), model-states paragraph: "1.5B parameter model like GPT-2") and
a 13B-class transformer that ZeRO-DP trains without model parallelism (same
page, results paragraph), represented by a 6.7B GPT shape.  No dataset is
involved; every value is drawn from a seeded generator.
"""
from __future__ import annotations

import dataclasses
import numpy as np

F16 = "f16"
BF16 = "bf16"


# ---------------------------------------------------------------------------
# Model shapes
# ---------------------------------------------------------------------------

def gpt2_1p5b_tensor_numels(layers: int = 48, d: int = 1600, ffn: int = 6400,
                            vocab: int = 50257, ctx: int = 1024) -> list[int]:
    """Parameter tensors of a GPT-2 1.5B-shaped model, in module order.

    Order: token embedding, position embedding, then per layer
    [ln1.w, ln1.b, qkv.W (d x 3d), qkv.b, proj.W (d x d), proj.b, ln2.w,
    ln2.b, fc.W (d x ffn), fc.b, fcproj.W (ffn x d), fcproj.b], then the final
    LayerNorm weight and bias.  The LM head is tied to the token embedding.
    With the defaults this is 580 tensors and 1,557,611,200 elements.
    """
    out = [vocab * d, ctx * d]
    for _ in range(layers):
        out += [d, d, d * 3 * d, 3 * d, d * d, d, d, d, d * ffn, ffn, ffn * d, d]
    out += [d, d]
    return out


def gpt_6p7b_unit_numels(layers: int = 32, d: int = 4096, ffn: int = 16384,
                         vocab: int = 50257) -> list[int]:
    """Per-unit element counts of a 6.7B GPT shape for layer-wise (Stage 3) use.

    Unit k < layers is transformer layer k (two LayerNorms with bias, fused
    qkv with bias, output projection with bias, two MLP matrices with bias):
    201,379,840 elements with the defaults.  The last unit is the token
    embedding plus the final LayerNorm (205,860,864 elements).  No position
    embedding table is counted.
    """
    layer = (2 * d) + (d * 3 * d + 3 * d) + (d * d + d) + (2 * d) \
        + (d * ffn + ffn) + (ffn * d + d)
    return [layer] * layers + [vocab * d + 2 * d]


# ---------------------------------------------------------------------------
# Workload configurations
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class AdamConfig:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    numels: tuple            # parameter tensors (or units) in order
    world: int               # N simulated data-parallel replicas
    loss_scale: float
    steps: int
    adam: AdamConfig
    bucket_elems: int = 0    # 0 = one bucket holding every tensor
    grad_std: float = 1e-3
    master_std: float = 0.02
    seed: int = 0


def tiny_flat() -> Workload:
    """Flat model of 1,000,003 elements (odd), 4 replicas, loss scale 1024."""
    return Workload("tiny_flat_1000003_n4", (1_000_003,), 4, 1024.0, 3,
                    AdamConfig(), seed=1)


def gpt2_1p5b() -> Workload:
    """GPT-2 1.5B parameter list, 500M-element buckets, 8 replicas, AdamW."""
    return Workload("gpt2_1.5b_n8_bucket500m", tuple(gpt2_1p5b_tensor_numels()), 8,
                    65536.0, 5, AdamConfig(weight_decay=0.01),
                    bucket_elems=500_000_000, seed=2)


def overflow_flat() -> Workload:
    """Flat 100M-element model, 16 replicas, dynamic loss scale from 65536."""
    return Workload("overflow_flat_100m_n16", (100_000_000,), 16, 65536.0, 6,
                    AdamConfig(), seed=3)


def gpt_6p7b_layerwise() -> Workload:
    """6.7B GPT shape, one unit per layer plus the embedding unit, 8 replicas."""
    return Workload("gpt_6.7b_layerwise_n8", tuple(gpt_6p7b_unit_numels()), 8,
                    65536.0, 1, AdamConfig(), seed=4)


SWEEP_PSI = (1 << 20, 16 << 20, 256 << 20, 1 << 30, 2 << 30)
SWEEP_N = (1, 2, 4, 8, 16, 64)


def sweep_points(max_grad_bytes: int = 96 * 10**9):
    """(psi, N) points of the flat bandwidth sweep with N*2*psi <= 96 GB."""
    return [(p, n) for p in SWEEP_PSI for n in SWEEP_N if n * 2 * p <= max_grad_bytes]


# ---------------------------------------------------------------------------
# Seeded draws (host, numpy PCG64)
# ---------------------------------------------------------------------------

def seed_for(config_seed: int, step: int, replica: int) -> int:
    """Seed of one replica's gradients at one step."""
    return 1000 * config_seed + 100 * step + replica


def _round_f32_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage rounding of drawn values (library conversion), as uint16 bits."""
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    if dtype == BF16:
        import torch
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dtype)


def grads(numel: int, seed: int, std: float, loss_scale: float, dtype: str = F16) -> np.ndarray:
    """One replica's scaled gradient buffer: round(N(0, std) * loss_scale) as uint16 bits."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(numel, dtype=np.float32) * np.float32(std) * np.float32(loss_scale)
    return _round_f32_to(x, dtype)


def master(numel: int, seed: int, std: float = 0.02) -> np.ndarray:
    """fp32 master weights ~ N(0, std)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal(numel, dtype=np.float32) * np.float32(std)


def params_from_master(m: np.ndarray, dtype: str = F16) -> np.ndarray:
    """Initial low-precision parameters: the storage rounding of the master copy."""
    return _round_f32_to(m, dtype)


def integer_grads(numel: int, seed: int, bound: int = 2048) -> np.ndarray:
    """fp16 bits of integers in [-bound, bound]; sums of a few are exact in fp32."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(-bound, bound + 1, numel).astype(np.float16).view(np.uint16)


F16_POS_INF = 0x7C00
F16_NAN = 0x7E00
BF16_POS_INF = 0x7F80
BF16_NAN = 0x7FC0


def injection_sites(psi: int, step: int, world: int, count: int = 17):
    """Overflow injection for the dynamic loss-scale workload.

    Returns (replica, positions, values_are_inf): `count` distinct positions in
    [0, psi) drawn with seed 3000 + step, in replica (5 * step) mod world; the
    sorted draw index decides +inf (even) or NaN (odd).
    """
    rng = np.random.Generator(np.random.PCG64(3000 + step))
    pos = np.sort(rng.choice(psi, size=count, replace=False)).astype(np.int64)
    is_inf = (np.arange(count) % 2) == 0
    return (5 * step) % world, pos, is_inf


def inject(buf: np.ndarray, positions: np.ndarray, is_inf: np.ndarray, dtype: str = F16) -> None:
    """Overwrite positions of a uint16 gradient buffer with +inf / NaN bits."""
    inf_bits = F16_POS_INF if dtype == F16 else BF16_POS_INF
    nan_bits = F16_NAN if dtype == F16 else BF16_NAN
    buf[positions] = np.where(is_inf, inf_bits, nan_bits).astype(np.uint16)
