"""Multi-process ZeRO-2: one process per rank, peers' buffers through CUDA IPC.

Layouts: 2 ranks with buckets padded to a multiple of 8N (every partition
16-byte aligned: the quad kernel at these sizes; gradient buffers on another
GPU always take plain loads, since the pipeline kernel's bulk copies read only
this GPU's memory), 3 ranks padded to a multiple of N only (partitions off the
16-byte phase: register and scalar paths).

2 and 3 ranks run as separate processes (on the one GPU of this machine, each
with its own context; host barriers over gloo order them, no kernel waits on
another rank).  Rank k writes replica k's gradients; the fused kernel of rank
r reads slice r of every peer's buffer in rank order.  After every step each
rank's partition of the fp32 states and its full gathered parameter buffer
must equal the oracle's Stage 2 bit for bit, including a step where one rank
injects inf / NaN and every rank skips.  Both the fused route (two banks) and
the staged route (one bank plus the reduced gradients; the update runs only
after the group's verdict) are run.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NUMELS = [300_001, 17, 650_000, 5, 3_100_000]
CAP = 400_000
STEPS = 4
INJECT_STEP, INJECT_RANK = 3, 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _grads(L, step, k):
    out = []
    for b in range(L.n_buckets):
        g = workloads.grads(L.bucket_padded[b], workloads.seed_for(21, step, k) + 17 * b, 1e-3, 65536.0)
        g[L.bucket_numel[b]:] = 0
        if step == INJECT_STEP and k == INJECT_RANK and b == 0:
            workloads.inject(g, np.array([4, 1000]), np.array([True, False]))
        out.append(g)
    return out


def _initial(L):
    tensors = [workloads.master(n, 900 + i) for i, n in enumerate(NUMELS)]
    return [oracle.flatten_bucket(L, b, tensors, np.float32) for b in range(L.n_buckets)]


def _rank_main(rank, world, align, port, outdir, mode="banks"):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import zero_sharded_optimizer_reduce_b200 as Z
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        adam = workloads.AdamConfig(weight_decay=0.01)
        opt = Z.DistributedZeroAdam(NUMELS, CAP, align, lr=adam.lr, betas=(adam.beta1, adam.beta2), eps=adam.eps,
                                    weight_decay=adam.weight_decay, loss_scale=65536.0, mode=mode)
        L = oracle.partition_layout(NUMELS, world, CAP, align)
        init = _initial(L)
        opt.load([torch.from_numpy(x).cuda() for x in init],
                 [torch.from_numpy(oracle.from_f32(x, oracle.F16).view(np.int16)).cuda().view(torch.float16)
                  for x in init])
        applied = []
        for step in range(1, STEPS + 1):
            scale = opt.scale
            for b, g in enumerate(_grads(L, step, rank)):
                if scale != 65536.0:          # regenerate at the current scale
                    g = workloads.grads(L.bucket_padded[b], workloads.seed_for(21, step, rank) + 17 * b, 1e-3,
                                        scale)
                    g[L.bucket_numel[b]:] = 0
                opt.grads[b].copy_(torch.from_numpy(g.view(np.int16)).cuda().view(torch.float16))
            applied.append(opt.step())
        res = {"applied": applied, "t": opt.t, "scale": opt.scale}
        for b in range(L.n_buckets):
            ms, m, v = opt.partition_state(b)
            res[f"master{b}"] = ms.cpu().numpy()
            res[f"m{b}"] = m.cpu().numpy()
            res[f"v{b}"] = v.cpu().numpy()
            res[f"params{b}"] = opt.params[b].view(torch.int16).cpu().numpy().view(np.uint16)
        np.save(os.path.join(outdir, f"rank{rank}.npy"), res, allow_pickle=True)
        opt.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,align,mode", [(2, 8, "banks"), (3, 1, "banks"), (2, 8, "staged"), (3, 1, "staged")])
def test_multiprocess_zero2_matches_oracle(world, align, mode, tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, align, port, str(tmp_path), mode))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]

    # the oracle: Stage 2 on `world` simulated ranks with the same inputs
    L = oracle.partition_layout(NUMELS, world, CAP, align)
    adam = workloads.AdamConfig(weight_decay=0.01)
    run = oracle.StageRun(2, L, _initial(L), adam, oracle.Scaler(65536.0))
    applied = []
    for step in range(1, STEPS + 1):
        scale = run.scaler.scale
        G = [[None] * world for _ in range(L.n_buckets)]
        for k in range(world):
            for b, g in enumerate(_grads(L, step, k)):
                if scale != 65536.0:
                    g = workloads.grads(L.bucket_padded[b], workloads.seed_for(21, step, k) + 17 * b, 1e-3, scale)
                    g[L.bucket_numel[b]:] = 0
                G[b][k] = g
        applied.append(run.step(G) == 0)
    assert applied == [True, True, False, True]
    for r in range(world):
        res = np.load(os.path.join(str(tmp_path), f"rank{r}.npy"), allow_pickle=True).item()
        assert res["applied"] == applied and res["t"] == run.scaler.t and res["scale"] == run.scaler.scale
        for b in range(L.n_buckets):
            P = L.part(b)
            fs = run.flat_state(b)
            own = slice(r * P, (r + 1) * P)
            for name in ("master", "m", "v"):
                assert np.array_equal(res[f"{name}{b}"].view(np.uint32), getattr(fs, name)[own].view(np.uint32)), name
            assert np.array_equal(res[f"params{b}"], fs.params), f"params of bucket {b} on rank {r}"
