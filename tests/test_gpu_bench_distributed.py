"""bench.py --distributed: the one-process-per-GPU routes under torchrun.

Two ranks share the one GPU of the test box (gloo host barriers; no kernel
waits on another rank, so sharing a GPU is safe): the run must finish, rank 0
alone prints one JSON line, every timed step applies, and the per-rank peer
bytes equal the layout's 2 (N - 1) P per bucket (3 (N - 1) P per unit for
Stage 3).  This checks the mode's host logic; NVLink bandwidth needs several
GPUs.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("mode", ["banks", "staged", "stage3"])
def test_bench_distributed_two_ranks(mode):
    import oracle
    flat, world, steps = 3_000_011, 2, 3
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={world}",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--distributed", "staged" if mode == "stage3" else mode, "--dist-backend", "gloo",
           "--flat", str(flat), "--steps", str(steps), "--warmup", "3"] + (["--stage3"] if mode == "stage3" else [])
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-3000:]
    d = json.loads(lines[0])
    assert d["n_gpus"] == world and d["steps"] == steps and d["applied_steps"] == steps
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["config"]["world"] == world
    units = [flat] * (4 if mode == "stage3" else 1)
    L = oracle.partition_layout(units, world, 1 if mode == "stage3" else 0, 8)
    parts = [L.bucket_padded[b] // world for b in range(L.n_buckets)]
    assert d["config"]["psi_padded"] == sum(L.bucket_padded)
    per = sum((world - 1) * P for P in parts)
    assert d["p2p"]["pull_bytes"] == 2 * per
    assert d["p2p"]["gather_bytes"] == 2 * per * (2 if mode == "stage3" else 1)
    assert d["p2p"]["elements_moved"] == per * (3 if mode == "stage3" else 2)
