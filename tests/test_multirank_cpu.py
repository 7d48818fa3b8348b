"""The benchmark's multi-rank path on the CPU: world_size 2 over gloo.

Under torchrun every GPU runs its own instance of the workload (the N data-
parallel replicas are simulated inside each GPU, so no data crosses GPUs);
the ranks only agree on the timing: the step time is the maximum over ranks
and the whole-job value sums every rank's elements.  These tests run that
host logic in two gloo processes, and the reference arm's rank rule (rank 0
alone prints, the others exit 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = [12.5, 10.0][rank]               # rank 0 is the slow one
        got = bench.max_over_ranks(ms, "cpu")
        value = bench.whole_job_gparams(1_000_000_000, world, got)
        q.put((rank, got, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [12.5, 12.5]
    assert all(abs(r[2] - 2 * 1e9 / 12.5e-3 / 1e9) < 1e-9 for r in res)


def test_helpers_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, "cpu") == 3.0
    assert bench.whole_job_gparams(1_557_611_200, 1, 9.72) == pytest.approx(160.25, rel=1e-3)


def test_reference_arm_two_ranks_only_rank0_prints():
    env = dict(os.environ, PYTHONPATH=ROOT)
    outs = []
    for rank in (0, 1):
        e = dict(env, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                            "--steps", "1", "--warmup", "0", "--ref-sample", "65536"],
                           env=e, capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr
        outs.append(r.stdout.strip())
    assert outs[1] == ""
    line = json.loads(outs[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def _verdict_worker(rank, world, port, flags, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from zero_sharded_optimizer_reduce_b200.distributed import DistributedZeroAdam
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        from zero_sharded_optimizer_reduce_b200.distributed_stage3 import DistributedZeroStage3
        got = []
        for cls in (DistributedZeroAdam, DistributedZeroStage3):
            opt = object.__new__(cls)                  # only the group-verdict logic, no device state
            opt.group, opt.device = None, "cpu"
            got.append([opt._or_over_ranks(f[rank]) for f in flags])
        q.put((rank, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_distributed_step_verdict_is_shared_by_every_rank():
    """The multi-process steps' skip decision (DistributedZeroAdam per step,
    DistributedZeroStage3 per unit): every rank's local flag word is OR-ed
    (max) over the group, so one rank's overflow (1) or pipeline timeout (2)
    makes every rank skip."""
    world, port = 3, _free_port()
    flags = [(0, 0, 0), (0, 1, 0), (2, 0, 0), (1, 1, 1)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_verdict_worker, args=(r, world, port, flags, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(r[1] == [[0, 1, 2, 1], [0, 1, 2, 1]] for r in res)


def test_bench_byte_models():
    """The bytes per element the benchmark divides by: the fused single pass
    2N + 26, statistics + gated update 4N + 26, staged 2N + 34 (reduce-scatter
    2N + 4, update 30); the update kernel alone in the staged mode is 30."""
    sys.path.insert(0, ROOT)
    import bench
    for n in (1, 8, 64):
        assert bench.bytes_per_elem(n) == 2 * n + 26
        assert bench.step_bytes_per_elem(n, "banks", False) == 2 * n + 26
        assert bench.step_bytes_per_elem(n, "banks", True) == 4 * n + 26
        assert bench.step_bytes_per_elem(n, "inplace", False) == 4 * n + 26
        assert bench.step_bytes_per_elem(n, "staged", False) == (2 * n + 4) + 30
        assert bench.update_bytes_per_elem(n, "staged") == 30
        assert bench.update_bytes_per_elem(n, "banks") == 2 * n + 26


def test_bench_traffic_records_scale_with_elements():
    sys.path.insert(0, ROOT)
    import bench
    for kind in bench.TRAFFIC_RECORDS:
        a, b = bench.profiled_traffic(1e6, kind), bench.profiled_traffic(3e6, kind)
        if a is None:                  # the record predates the current kernel source
            assert b is None
            continue
        assert abs(b - 3 * a) < 1e-6 * b
        # DRAM bytes never exceed the algorithmic bytes by more than a few percent
        per = a / 1e6
        bound = {"fused": 42, "staged": 30, "staged_step": 50}[kind]
        assert 0.9 * bound <= per <= 1.05 * bound


def test_p2p_byte_model_matches_the_pages_volumes():
    """Bytes one rank moves between GPUs per step of the one-process-per-GPU
    routes (bench.p2p_bytes_per_rank), against the pages' communication
    volumes (ZeRO explainer, communication-volume paragraphs): Stage 1/2 move
    2 Psi (N - 1) / N elements per rank (reduce-scatter + all-gather, the same
    as data parallelism's all-reduce), Stage 3 moves 1.5 x that."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import workloads
    for numels, world, cap in [(workloads.gpt2_1p5b_tensor_numels(), 8, 500_000_000), ([1_000_003], 4, 0),
                               ([100_000_000], 16, 0), ([7, 5000, 123], 3, 4000)]:
        L = oracle.partition_layout(numels, world, cap)
        parts = [L.bucket_padded[b] // world for b in range(L.n_buckets)]
        psi_p = sum(L.bucket_padded)
        for mode in ("banks", "staged"):
            m = bench.p2p_bytes_per_rank(parts, world, 2, 2, mode)
            assert m["elements_moved"] == 2 * (world - 1) * psi_p // world
            assert m["pull_bytes"] == m["gather_bytes"] == 2 * (world - 1) * psi_p // world
            # the oracle's own ring count for the same layout
            assert m["elements_moved"] == oracle.comm_elements(2, L)
        s3 = bench.p2p_bytes_per_rank(parts, world, 2, 2, "stage3")
        assert s3["elements_moved"] == 3 * (world - 1) * psi_p // world == oracle.comm_elements(3, L)
        assert s3["gather_bytes"] == 2 * s3["pull_bytes"]
        assert s3["elements_moved"] * 2 == 3 * bench.p2p_bytes_per_rank(parts, world, 2, 2, "banks")["elements_moved"]
    # fp32 gradients, bf16 parameters: bytes follow the element sizes
    m = bench.p2p_bytes_per_rank([10], 3, 4, 2, "banks")
    assert (m["pull_bytes"], m["gather_bytes"]) == (80, 40)
    assert bench.p2p_bytes_per_rank([10], 1, 2, 2, "staged")["elements_moved"] == 0


def test_clock_csv_parsing():
    """bench.parse_clock_csv: median SM clock under load, max clock, the
    throttle reasons seen, timestamps kept per sample; idle samples below half
    the top clock left out of the median; malformed lines skipped."""
    import bench
    lines = [
        "0, 1965, 1965, 900.1, 0x0, Not Active, Not Active, Not Active, Not Active, 2026/12/03 10:00:00.000\n",
        "0, 1650, 1965, 1000.0, 0x4, Not Active, Not Active, Not Active, Active, 2026/12/03 10:00:00.100\n",
        "0, 1700, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active, 2026/12/03 10:00:00.200\n",
        "0, 345, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active, 2026/12/03 10:00:00.300\n",
        "garbage line\n",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active, 2026/12/03 10:00:00.400\n",
    ]
    summary, samples = bench.parse_clock_csv(lines)
    assert summary == {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 4}
    assert [s[1] for s in samples] == [1965.0, 1650.0, 1700.0, 345.0]
    assert samples[1][2] == ["sw_power_cap"] and samples[0][2] == []
    assert abs((samples[3][0] - samples[0][0]) - 0.3) < 1e-6
    assert bench.parse_clock_csv([]) == (None, [])
