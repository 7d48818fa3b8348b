"""Multi-process ZeRO-3: one process per rank, peers' shards and gradients
through CUDA IPC (DistributedZeroStage3).

2 ranks with units padded to a multiple of 8N (16-byte aligned slices) and 3
ranks padded to a multiple of N (slices off the 16-byte phase) run as
separate processes on the one GPU of this machine (own contexts, gloo host
barriers, no kernel waits on another rank).  Rank k supplies replica k's
gradients of each unit.  After two steps (one unit of the second step gets
an injected inf / NaN from rank 1) every rank's slices of the fp32 states
and every unit gathered from the shards must equal the oracle's step unit by
unit, bit for bit; the overflowing unit is left unchanged, t and the loss
scale follow the skip.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
import workloads

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
UNITS = [50_000, 70_001, 3, 120_000]
INJECT_STEP, INJECT_UNIT, INJECT_RANK = 2, 1, 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _unit_grads(L, u, step, k, scale):
    g = workloads.grads(L.bucket_padded[u], workloads.seed_for(41, step, k) + 101 * u, 1e-3, scale)
    g[L.bucket_numel[u]:] = 0
    if step == INJECT_STEP and u == INJECT_UNIT and k == INJECT_RANK:
        workloads.inject(g, np.array([1, 7]), np.array([True, False]))
    return g


def _initial(L):
    return [np.concatenate([workloads.master(n, 960 + u), np.zeros(L.bucket_padded[u] - n, np.float32)])
            for u, n in enumerate(UNITS)]


def _rank_main(rank, world, align, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import zero_sharded_optimizer_reduce_b200 as Z
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        adam = workloads.AdamConfig(weight_decay=0.01)
        s3 = Z.DistributedZeroStage3(UNITS, align_elems=align, lr=adam.lr, betas=(adam.beta1, adam.beta2),
                                     eps=adam.eps, weight_decay=adam.weight_decay, loss_scale=65536.0)
        L = oracle.partition_layout(UNITS, world, 1, align)
        s3.load([torch.from_numpy(x).cuda() for x in _initial(L)])
        applied = []
        for step in (1, 2):
            scale = s3.scale

            def fill(u, buf, step=step, scale=scale):
                g = _unit_grads(L, u, step, rank, scale)
                buf.copy_(torch.from_numpy(g.view(np.int16)).cuda().view(torch.float16))
            applied.append(s3.step(fill))
        res = {"applied": applied, "t": s3.t, "scale": s3.scale, "gathers": s3.gathers}
        for u in range(len(UNITS)):
            res[f"master{u}"] = s3.master[u].cpu().numpy()
            res[f"m{u}"] = s3.m[u].cpu().numpy()
            res[f"v{u}"] = s3.v[u].cpu().numpy()
            res[f"params{u}"] = s3.gather(u).clone().view(torch.int16).cpu().numpy().view(np.uint16)
        np.save(os.path.join(outdir, f"rank{rank}.npy"), res, allow_pickle=True)
        s3.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,align", [(2, 8), (3, 1)])
def test_multiprocess_zero3_matches_oracle(world, align, tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, align, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]

    L = oracle.partition_layout(UNITS, world, 1, align)
    adam = workloads.AdamConfig(weight_decay=0.01)
    init = _initial(L)
    states = [oracle.initial_state(x) for x in init]
    scale, t = 65536.0, 0
    for step in (1, 2):
        all_ok = True
        for u in range(len(UNITS)):
            G = [_unit_grads(L, u, step, k, scale) for k in range(world)]
            ovf, _ = oracle.flat_step(G, states[u], adam, t + 1, scale, float(world))   # skips on overflow
            all_ok = all_ok and not ovf
        if all_ok:
            t += 1
        scale = scale if all_ok else scale / 2
    for r in range(world):
        res = np.load(os.path.join(str(tmp_path), f"rank{r}.npy"), allow_pickle=True).item()
        assert res["applied"] == [True, False] and res["t"] == t == 1 and res["scale"] == scale == 32768.0
        assert res["gathers"] == 2 * 2 * len(UNITS)          # forward + backward gathers, 2 steps
        for u in range(len(UNITS)):
            P = L.part(u)
            own = slice(r * P, (r + 1) * P)
            for name in ("master", "m", "v"):
                assert np.array_equal(res[f"{name}{u}"].view(np.uint32),
                                      getattr(states[u], name)[own].view(np.uint32)), (name, u)
            assert np.array_equal(res[f"params{u}"], states[u].params), f"unit {u} gathered on rank {r}"
