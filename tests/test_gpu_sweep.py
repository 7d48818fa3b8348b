"""Parity at every point of the flat bandwidth sweep.

The sweep is Psi in {1M, 16M, 256M, 1B, 2B} elements x N in {1, 2, 4, 8, 16,
64} replicas with N x 2 x Psi <= 96 GB: 28 points, run here in fp16 and in
bf16 (56 cases).  Each point is one flat bucket processed by one
all-partition call, the launch the sweep times (same sizes, same 256-byte
aligned buffers, so the same kernel, tile and grid).

Per point:
- seeded gradients N(0, 1e-3) x 65536 and fp32 master N(0, 0.02) drawn on the
  device, m = v = 0;
- two steps (t = 1 from zero moments, t = 2 from the first step's moments,
  banks swapped between them);
- sampled windows (first and last 4096 elements, every partition boundary
  +-4, 8 seeded windows of 16,384) of every input, taken before the steps,
  run through the oracle for both steps; master / m / v / parameters compared
  bit for bit after each step;
- the overflow flag over the whole array: 0 at both steps, which is what the
  rank-order sum must give when every input is finite and |x| <= 65504
  (checked on the inputs), since 64 such values cannot sum past fp32's range;
- a third call with +inf planted at one seeded position of one replica: the
  flag must be 1 (an infinite input makes its sum non-finite whatever the
  other replicas hold).

All points share one device pool sized for the largest point that fits.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import assert_f32_close, assert_u16_close, device_grads, device_master, free_gb, host_f32, windows

pytestmark = pytest.mark.gpu

TD = {oracle.F16: torch.float16, oracle.BF16: torch.bfloat16}
INF_BITS = {oracle.F16: 0x7C00, oracle.BF16: 0x7F80}
ALIGN = 256
ADAM = workloads.AdamConfig(weight_decay=0.01)
SCALE = 65536.0


def _bytes_needed(psi, world):
    # N gradient buffers, two fp32 banks of master/m/v, one parameter buffer
    return psi * (2 * world + 24 + 2) + 16 * ALIGN


class _Pool:
    """Carves 256-byte aligned typed views out of one device allocation."""

    def __init__(self, nbytes):
        self.raw = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        self.off = 0

    def reset(self):
        self.off = 0

    def take(self, n, dtype):
        es = torch.empty((), dtype=dtype).element_size()
        nb = n * es
        assert self.off + nb <= self.raw.numel()
        v = self.raw[self.off:self.off + nb].view(dtype)
        self.off += (nb + ALIGN - 1) // ALIGN * ALIGN
        return v


def _max_abs(t):
    m = 0.0
    for o in range(0, t.numel(), 1 << 27):
        m = max(m, float(t[o:o + (1 << 27)].abs().max()))
    return m


def _u16_at(t, idx):
    return t.view(torch.int16)[idx].cpu().numpy().view(np.uint16)


def _f32_at(t, idx):
    return host_f32(t[idx])


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_every_sweep_point(dtype):
    points = workloads.sweep_points()
    assert len(points) == 28
    free = free_gb() * 1e9 - 4e9          # headroom for the draws' temporaries
    total = torch.cuda.get_device_properties(0).total_memory
    fits = [pt for pt in points if _bytes_needed(*pt) <= free]
    if total >= 150e9:                     # a B200-class GPU holds every point
        assert fits == points, f"only {len(fits)} of {len(points)} sweep points fit in {free / 1e9:.0f} GB"
    if not fits:
        pytest.skip("no sweep point fits in the free device memory")
    pool = _Pool(max(_bytes_needed(*pt) for pt in fits))
    tdt = TD[dtype]
    checked = 0
    for idx, (psi, N) in enumerate(points):
        if (psi, N) not in fits:
            continue
        pool.reset()
        grads = [pool.take(psi, tdt) for _ in range(N)]
        bank = [[pool.take(psi, torch.float32) for _ in range(3)] for _ in range(2)]
        params = pool.take(psi, tdt)
        for k in range(N):
            device_grads(grads[k], 50_000 + 100 * idx + k, 1e-3, SCALE)
            assert _max_abs(grads[k]) <= 65504.0       # finite, and small enough that no sum overflows
        device_master(bank[0][0], 60_000 + idx)
        bank[0][1].zero_()
        bank[0][2].zero_()
        wins = windows(psi, N, n_random=8, width=16_384, seed=idx)
        sel = torch.cat([torch.arange(lo, hi, device="cuda") for lo, hi in wins])
        G = [_u16_at(g, sel) for g in grads]
        ref = oracle.initial_state(_f32_at(bank[0][0], sel), dtype)
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        for t in (1, 2):
            src, dst = bank[(t - 1) % 2], bank[t % 2]
            flag.zero_()
            Z.zero_reduce_scatter_adam_step(grads, psi, Z.ZERO_ALL_PARTITIONS, *src, *dst, params,
                                            Z.hparams(ADAM.lr, ADAM.beta1, ADAM.beta2, ADAM.eps, ADAM.weight_decay, t),
                                            SCALE, flag)
            torch.cuda.synchronize()
            assert int(flag.item()) == 0, f"psi={psi} N={N} t={t}: flag"
            ovf, _ = oracle.flat_step(G, ref, ADAM, t, SCALE, float(N), dtype, dtype)
            assert ovf == 0
            what = f"psi={psi} N={N} {dtype} t={t}"
            assert assert_f32_close(_f32_at(dst[0], sel), ref.master, what + " master") == 0
            assert assert_f32_close(_f32_at(dst[1], sel), ref.m, what + " m") == 0
            assert assert_f32_close(_f32_at(dst[2], sel), ref.v, what + " v") == 0
            assert assert_u16_close(_u16_at(params, sel), ref.params, what + " params") == 0
        # one infinite input anywhere in the array must raise the flag
        rng = np.random.Generator(np.random.PCG64(70_000 + idx))
        k, pos = int(rng.integers(0, N)), int(rng.integers(0, psi))
        grads[k].view(torch.int16)[pos] = INF_BITS[dtype]
        flag.zero_()
        Z.zero_reduce_scatter_adam_step(grads, psi, Z.ZERO_ALL_PARTITIONS, *bank[0], *bank[1], params,
                                        Z.hparams(ADAM.lr, ADAM.beta1, ADAM.beta2, ADAM.eps, ADAM.weight_decay, 3),
                                        SCALE, flag)
        torch.cuda.synchronize()
        assert int(flag.item()) == 1, f"psi={psi} N={N}: +inf at replica {k}, element {pos} not flagged"
        checked += 1
    assert checked == len(fits)


@pytest.mark.parametrize("psi,world", [(1 << 20, 4), (8 * 1_000_003, 8), (24 * 43_691, 24)])
def test_bench_kernel_ab_mode(psi, world):
    """bench.py --kernel-ab: one JSON line with every kernel's timing; the
    forced kernels that can run the call report themselves (the others the
    automatic choice), and every kernel's sampled outputs equal the automatic
    choice's."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--kernel-ab", str(psi), "--world", str(world), "--steps", "3"],
                       cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    res = d["results"]
    assert set(res) == {"auto", "register", "pipeline", "quad", "oct"}
    assert res["register"]["kernel_ran"] == "register"
    if world <= 16:
        assert res["quad"]["kernel_ran"] == "quad" and res["oct"]["kernel_ran"] == "oct"
        assert res["pipeline"]["kernel_ran"] == "pipeline"
    else:
        assert res["quad"]["kernel_ran"] == res["oct"]["kernel_ran"] == res["auto"]["kernel_ran"]
    for name, v in res.items():
        assert v["gbs"] > 0
        if name != "auto":
            assert v["sample_bit_identical_to_auto"] is True, name


@pytest.mark.parametrize("world", [2, 8])
def test_bench_kernel_ab_passes_mode(world):
    """bench.py --kernel-ab --mode staged: the reduce-scatter, statistics and
    update passes timed under every kernel; every kernel's reduce-scatter
    output, flag and norm agree with the automatic choice's."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--kernel-ab", str(world * 131_072), "--world", str(world),
                        "--mode", "staged", "--steps", "3"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert set(d["passes_timed"]) == {"reduce_scatter", "statistics", "update"}
    for p in d["passes_timed"].values():
        assert set(p["results"]) == {"auto", "register", "pipeline", "quad", "oct"}
        assert all(v["gbs"] > 0 for v in p["results"].values())
    assert set(d["reduce_scatter_agrees_with_auto"]) == {"register", "pipeline", "quad", "oct"}
    assert all(d["reduce_scatter_agrees_with_auto"].values())
