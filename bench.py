"""Benchmark of the fused ZeRO-2 step (reduce-scatter + Adam) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload: a GPT-2 1.5B-shaped parameter list (48 layers, d=1600, ffn=6400,
vocab 50257, ctx 1024; 580 tensors, 1,557,611,200 elements) packed into
constant-size buffers of at most 500M elements (4 buckets), N = 8 simulated
data-parallel replicas whose fp16 gradients (N(0, 1e-3) x 65536) are resident
in HBM, fp32 master ~ N(0, 0.02), AdamW (lr 1e-3, betas 0.9/0.999, eps 1e-8,
wd 0.01), dynamic loss scale 65536.  Synthetic, seeded data.

A step = the fused kernel over the 4 buckets (every rank's partition), the
overflow flag read back to the host, the bank commit and the loss-scale
update.  `value` is Gparams/s (padded elements updated per second, all
ranks); the roofline object rates the fused kernel's algorithmic HBM bytes,
(2N + 26) per element, against the measured B200 copy bandwidth.

Under torchrun with N > 1, every GPU runs its own instance of the workload
(no exchange between GPUs: the replicas are simulated inside each GPU), the
step time is the max over ranks, and `value` sums all ranks' elements.

--impl reference times the CPU oracle (C, OpenMP) on the host cores, each
step a bounded slice of the same workload.

Other modes (each prints JSON lines of its own):
  --mode {inplace,staged}, --max-grad-norm X   the one-bank step routes, clipping
  --flat PSI --world N                         a flat workload instead of GPT-2
  --sweep                                      the flat bandwidth sweep (kernel calls alone)
  --kernel-ab PSI --world N [--mode staged]    one flat point with each step kernel forced in turn
                                               (--mode staged: the one-bank routes' passes)
  --allgather P --world N                      the all-gather of N slices of P elements
  --stage3                                     the layer-wise ZeRO-3 step, 6.7B shape
  --distributed {banks,staged} [--stage3]      one process per GPU under torchrun (real ranks)
  --cpu-configs                                the CPU oracle on every workload (no GPU)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "fused ZeRO step: Gparams/s and achieved HBM GB/s vs B200 peak (1 GPU)"
UNIT = "Gparams/s"
FALLBACK_HBM_GBS = 6650.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def bytes_per_elem(world: int) -> int:
    """Algorithmic HBM bytes per partition element of the fused step."""
    return 2 * world + 26


def step_bytes_per_elem(world: int, mode: str, clipped: bool) -> int:
    """Algorithmic HBM bytes per element of a whole step: the fused single
    pass (2N + 26), statistics + gated update (4N + 26), or the staged
    reduce-scatter (2N + 4) + update from the reduced gradients (30)."""
    if mode == "staged":
        return 2 * world + 34
    if mode == "inplace" or clipped:
        return 4 * world + 26
    return 2 * world + 26


def update_bytes_per_elem(world: int, mode: str) -> int:
    """Algorithmic bytes per element of the kernel the roofline times (the
    step's update kernel)."""
    return 30 if mode == "staged" else 2 * world + 26


PASSES = {"banks": "single fused pass", "inplace": "statistics pass (2N B/elem) + gated update (2N + 26)",
          "staged": "reduce-scatter to fp32 (2N + 4 B/elem) + gated update from it (30)"}


# ----------------------------------------------------------------- helpers

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region.
    With keep_samples, stop() also returns every sample as (unix time, SM MHz,
    reasons), for attributing clocks to sub-intervals."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,timestamp")

    def __init__(self, device_index: int, keep_samples: bool = False):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.keep = keep_samples
        self.samples = []

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.dev), "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        summary, samples = parse_clock_csv(lines)
        if self.keep:
            self.samples = samples
        return summary


def parse_clock_csv(lines):
    """nvidia-smi lines of ClockSampler.Q -> (summary, samples): the median SM
    clock under load, the largest max clock, the throttle reasons seen; and
    every sample as (unix time, SM MHz, reasons) when it has a timestamp."""
    import datetime
    sm, mx, reasons, samples = [], 0.0, set(), []
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            clk = float(parts[1])
            mx = max(mx, float(parts[2]))
        except ValueError:
            continue
        sm.append(clk)
        here = [n for n, v in zip(names, parts[5:9]) if v.lower() == "active"]
        reasons.update(here)
        if len(parts) >= 10:
            try:
                ts = datetime.datetime.strptime(parts[9], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                samples.append((ts, clk, here))
            except ValueError:
                pass
    if not sm:
        return None, samples
    under_load = [x for x in sm if x >= 0.5 * max(sm)] or sm
    return ({"sm_mhz": statistics.median(under_load), "sm_max_mhz": mx, "reasons": sorted(reasons),
             "samples": len(sm)}, samples)


def source_digest(files=("fused_step.cuh",)) -> str:
    """Hash of kernel sources, comments and whitespace removed, so that the
    recorded ncu traffic is dropped only when the code changes."""
    import re
    text = ""
    for name in files:
        with open(os.path.join(ROOT, "zero_sharded_optimizer_reduce_b200", "csrc", name)) as f:
            text += f.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()[:16]


# timed kernel -> (committed ncu traffic record, the sources it was taken on)
TRAFFIC_RECORDS = {"fused": ("fused_step_traffic.json", ("bulk.cuh", "fused_step.cuh")),
                   "staged": ("adam_reduced_traffic.json", ("bulk.cuh", "fused_step.cuh", "staged.cuh")),
                   "staged_step": ("staged_step_traffic.json",
                                   ("bulk.cuh", "fused_step.cuh", "grad_stats.cuh", "staged.cuh"))}


def profiled_traffic(elems_per_launch: float, kernel: str = "fused"):
    """DRAM bytes per launch of the timed kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    name, files = TRAFFIC_RECORDS[kernel]
    p = os.path.join(ROOT, "profiles", name)
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_source_sha256_16") != source_digest(files):
        return None
    return float(d["dram_bytes_per_elem"]) * elems_per_launch


# --------------------------------------------------------------- CPU side

def _oracle_rate(G, master, adam, loss_scale, divisor, min_seconds, max_steps=None):
    """Elements per second of the oracle's flat step (reduce-scatter, overflow
    test, Adam) over the given replicas: whole steps until min_seconds have
    passed (at least one).  Returns (Gparams/s, steps, seconds)."""
    import oracle
    n = G[0].size
    st = oracle.initial_state(master)
    done, t0, t = 0, time.perf_counter(), 0
    while True:
        t += 1
        oracle.flat_step(G, st, adam, t, loss_scale, divisor)
        done += n
        el = time.perf_counter() - t0
        if el >= min_seconds or (max_steps is not None and t >= max_steps):
            return done / el / 1e9, t, el


def cpu_baseline(w: workloads.Workload, sample_elems: int, min_seconds: float = 8.0):
    """The oracle on this host's cores (OpenMP over every core, and one
    thread): on a contiguous slice of the benchmark workload (its unit), plus
    the full arrays of the tiny and the dynamic-loss-scale workloads."""
    import oracle
    cores = oracle.threads()

    def both(G, master, loss_scale, divisor, adam, secs, single_steps=1):
        v, steps, el = _oracle_rate(G, master, adam, loss_scale, divisor, secs)
        oracle.set_threads(1)
        try:
            v1, steps1, el1 = _oracle_rate(G, master, adam, loss_scale, divisor, float("inf"),
                                              max_steps=single_steps)
        finally:
            oracle.set_threads(cores)
        return {"value": v, "single_thread_value": v1, "steps": steps, "seconds": el,
                "single_thread_steps": steps1, "single_thread_seconds": el1}

    N = w.world
    G = [workloads.grads(sample_elems, workloads.seed_for(w.seed, 1, k), w.grad_std, w.loss_scale)
         for k in range(N)]
    head = both(G, workloads.master(sample_elems, 7 * w.seed), w.loss_scale, float(N), w.adam, min_seconds)
    del G
    configs = {}
    tiny = workloads.tiny_flat()
    padded = -(-tiny.numels[0] // tiny.world) * tiny.world
    G = [workloads.grads(padded, workloads.seed_for(tiny.seed, 1, k), tiny.grad_std, tiny.loss_scale)
         for k in range(tiny.world)]
    r = both(G, workloads.master(padded, 7 * tiny.seed), tiny.loss_scale, float(tiny.world), tiny.adam, 2.0,
             single_steps=3)
    configs[tiny.name] = dict(r, elements=padded, world=tiny.world, sample="full arrays")
    ovf = workloads.overflow_flat()
    psi = ovf.numels[0]
    # two seeded draws; the other replicas are seeded rotations of them (the
    # same distribution; the oracle's time does not depend on the values)
    base = [workloads.grads(psi, workloads.seed_for(ovf.seed, 1, k), ovf.grad_std, ovf.loss_scale) for k in range(2)]
    G = [np.roll(base[k % 2], 7919 * k) for k in range(ovf.world)]
    r = both(G, workloads.master(psi, 7 * ovf.seed), ovf.loss_scale, float(ovf.world), ovf.adam, 2.0)
    configs[ovf.name] = dict(r, elements=psi, world=ovf.world,
                             sample="full arrays (replicas 2-15 are seeded rotations of two draws)")
    del G, base
    return {"value": head["value"], "unit": UNIT, "cores": cores, "kind": "oracle",
            "single_thread_value": head["single_thread_value"],
            "sample": f"{head['steps']} oracle steps (reduce-scatter, overflow test, AdamW) over a "
                      f"{sample_elems:,}-element contiguous slice of bucket 0 of {w.name} with N={N} replicas, "
                      f"{head['seconds']:.1f} s on {cores} threads; single_thread_value: "
                      f"{head['single_thread_steps']} step(s) of the same slice on 1 thread; configs: the full "
                      f"arrays of the tiny and the dynamic-loss-scale workloads, same protocol",
            "configs": configs}


def run_cpu_configs(args):
    """The oracle timed on every workload: the full arrays of the tiny and the dynamic-loss-scale
    workloads, 64M-element slices of the GPT-2 1.5B bucket, of one 6.7B unit
    and of the sweep's flat buffers (N = 1, 8, 16 and 64), each on every host
    core and on one thread.  One JSON line; no GPU is used."""
    import oracle
    cores = oracle.threads()
    S = args.cpu_sample

    def rate(G, master, adam, loss_scale, divisor, secs=4.0):
        v, steps, el = _oracle_rate(G, master, adam, loss_scale, divisor, secs)
        oracle.set_threads(1)
        try:
            v1, _, el1 = _oracle_rate(G, master, adam, loss_scale, divisor, float("inf"), max_steps=1)
        finally:
            oracle.set_threads(cores)
        return {"value": v, "single_thread_value": v1, "steps": steps, "seconds": round(el, 2),
                "single_thread_seconds": round(el1, 2)}

    def draws(n, world, seed, std, scale, distinct=2):
        # `distinct` seeded draws; further replicas are seeded rotations of them
        base = [workloads.grads(n, workloads.seed_for(seed, 1, k), std, scale) for k in range(min(distinct, world))]
        return [base[k] if k < len(base) else np.roll(base[k % len(base)], 7919 * k) for k in range(world)]

    out = {}
    tiny = workloads.tiny_flat()
    padded = -(-tiny.numels[0] // tiny.world) * tiny.world
    out[tiny.name] = dict(rate(draws(padded, tiny.world, tiny.seed, tiny.grad_std, tiny.loss_scale, tiny.world),
                               workloads.master(padded, 7), tiny.adam, tiny.loss_scale, float(tiny.world)),
                          elements=padded, world=tiny.world, sample="full arrays")
    g2 = workloads.gpt2_1p5b()
    out[g2.name] = dict(rate(draws(S, g2.world, g2.seed, g2.grad_std, g2.loss_scale), workloads.master(S, 14),
                             g2.adam, g2.loss_scale, float(g2.world)),
                        elements=S, world=g2.world, sample=f"{S:,}-element slice of bucket 0")
    ov = workloads.overflow_flat()
    out[ov.name] = dict(rate(draws(ov.numels[0], ov.world, ov.seed, ov.grad_std, ov.loss_scale),
                             workloads.master(ov.numels[0], 21), ov.adam, ov.loss_scale, float(ov.world)),
                        elements=ov.numels[0], world=ov.world, sample="full arrays")
    g3 = workloads.gpt_6p7b_layerwise()
    out[g3.name] = dict(rate(draws(S, g3.world, g3.seed, g3.grad_std, g3.loss_scale), workloads.master(S, 28),
                             g3.adam, g3.loss_scale, float(g3.world)),
                        elements=S, world=g3.world, sample=f"{S:,}-element slice of unit 0")
    for N in (1, 8, 16, 64):
        adam = workloads.AdamConfig(weight_decay=0.01)
        out[f"sweep_flat_n{N}"] = dict(rate(draws(S, N, 5, 1e-3, 65536.0), workloads.master(S, 35), adam, 65536.0,
                                            float(N)),
                                       elements=S, world=N, sample=f"{S:,}-element slice of a flat buffer")
    print(json.dumps({"metric": "CPU oracle: Gparams/s per workload (reduce-scatter, overflow test, Adam)",
                      "unit": UNIT, "cores": cores, "kind": "oracle",
                      "note": "replicas past the first two of each workload are seeded rotations of those "
                              "draws (the same distribution; the oracle's time does not depend on the values)",
                      "configs": out}), flush=True)
    return 0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = workloads.gpt2_1p5b()
    N = w.world
    sample = args.ref_sample
    G = [workloads.grads(sample, workloads.seed_for(w.seed, 1, k), w.grad_std, w.loss_scale) for k in range(N)]
    st = oracle.initial_state(workloads.master(sample, 7 * w.seed))
    for t in range(1, args.warmup + 1):
        oracle.flat_step(G, st, w.adam, t, w.loss_scale, float(N))
    t0 = time.perf_counter()
    for t in range(args.warmup + 1, args.warmup + args.steps + 1):
        oracle.flat_step(G, st, w.adam, t, w.loss_scale, float(N))
    el = time.perf_counter() - t0
    value = sample * args.steps / el / 1e9
    sample_desc = f"{sample:,}-element slice of the {w.name} workload per step (N={N})"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": w.name, "world": N, "elems_per_step": sample,
                                            "note": "CPU oracle on a bounded slice"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                             "sample": sample_desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------- multi-rank helpers

def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gparams(elems_per_rank: int, n_ranks: int, ms_per_step: float) -> float:
    """Elements updated per second by all ranks together (weak scaling: every
    rank runs the same workload), in Gparams/s, from the slowest rank's time."""
    return n_ranks * elems_per_rank / (ms_per_step * 1e-3) / 1e9


# --------------------------------------------------------------- GPU side

def fill_workload(opt, w, seed_base: int):
    """Seeded device-side draws: gradients, master weights, parameters."""
    import torch
    gen = torch.Generator(device="cuda")
    L = opt.layout
    for b in range(L.n_buckets):
        n = L.bucket_padded[b]
        for k in range(w.world):
            gen.manual_seed(workloads.seed_for(seed_base, 1, k) + 7919 * b)
            buf = opt.grads[b][k]
            chunk = 1 << 27
            for o in range(0, n, chunk):
                e = min(n, o + chunk)
                x = torch.randn(e - o, generator=gen, device="cuda", dtype=torch.float32)
                buf[o:e].copy_(x.mul_(w.grad_std * w.loss_scale))
            buf[L.bucket_numel[b]:].zero_()
        gen.manual_seed(7 * seed_base + b)
        for o in range(0, n, 1 << 27):
            e = min(n, o + (1 << 27))
            x = torch.randn(e - o, generator=gen, device="cuda", dtype=torch.float32).mul_(w.master_std)
            opt.master[b][0][o:e].copy_(x)
        opt.master[b][0][L.bucket_numel[b]:].zero_()
        opt.params_bank[b][0].copy_(opt.master[b][0])
        for bank in (opt.m, opt.v):
            bank[b][0].zero_()
        for extra in opt.master[b][1:]:
            extra.copy_(opt.master[b][0])
        for extra in opt.params_bank[b][1:]:
            extra.copy_(opt.params_bank[b][0])
    torch.cuda.synchronize()


def select_workload(args) -> workloads.Workload:
    if args.flat:
        return workloads.Workload(f"flat_{args.flat}_n{args.world}_{args.grad_dtype}", (args.flat,), args.world,
                                  65536.0, 1, workloads.AdamConfig(weight_decay=0.01), seed=5)
    return workloads.gpt2_1p5b()


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import zero_sharded_optimizer_reduce_b200 as Z

    world_gpus = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world_gpus > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world_gpus > 1:
            dist.barrier()
        torch.cuda.synchronize()

    w = select_workload(args)
    gdt = torch.bfloat16 if args.grad_dtype == "bf16" else torch.float16
    opt = Z.ZeroAdam(w.numels, w.world, w.bucket_elems, lr=w.adam.lr, betas=(w.adam.beta1, w.adam.beta2),
                     eps=w.adam.eps, weight_decay=w.adam.weight_decay, loss_scale=w.loss_scale,
                     grad_dtype=gdt, param_dtype=gdt, mode=args.mode, max_grad_norm=args.max_grad_norm)
    L = opt.layout
    psi_p = sum(L.bucket_padded)
    fill_workload(opt, w, w.seed + 100 * rank)
    stream = torch.cuda.current_stream()

    # ---- device-timed steps
    ev = {}

    def on_launch(b, phase):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        ev.setdefault(b, []).append(e)

    for _ in range(args.warmup):
        opt.step()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev.clear()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.profiler.start()      # ncu --profile-from-start off captures only the timed steps
    t_start.record(stream)
    applied = 0
    step_ev = [t_start]              # an event at every step boundary: per-step device times
    for i in range(args.steps):
        applied += bool(opt.step(on_launch=on_launch))
        if i + 1 < args.steps:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            step_ev.append(e)
    t_end.record(stream)
    step_ev.append(t_end)
    barrier()
    torch.cuda.profiler.stop()
    clock = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    step_ms = [a.elapsed_time(b) for a, b in zip(step_ev[:-1], step_ev[1:])]
    # per-launch durations of the fused kernel
    launch_ms, launch_elems = [], []
    for b, es in ev.items():
        for i in range(0, len(es), 2):
            launch_ms.append(es[i].elapsed_time(es[i + 1]))
            # b = -1: the runner's whole step (every bucket's kernel, the flag
            # clear and its 4-byte read-back) between one pair of events
            launch_elems.append(psi_p if b < 0 else L.bucket_padded[b])
    ms = max_over_ranks(ms, "cuda")
    ms_per_step = ms / args.steps
    ms_median = max_over_ranks(statistics.median(step_ms), "cuda")
    value = whole_job_gparams(psi_p, world_gpus, ms_per_step)
    bpe = step_bytes_per_elem(w.world, args.mode, args.max_grad_norm is not None)
    # the runner's whole step (b = -1) is timed as one unit: every byte of the step
    kbpe = bpe if -1 in ev else update_bytes_per_elem(w.world, args.mode)
    peak, peak_kind = peaks()
    kern_bytes = sum(launch_elems) * kbpe
    kern_s = sum(launch_ms) * 1e-3
    achieved = kern_bytes / kern_s / 1e9
    avg_elems = sum(launch_elems) / len(launch_elems)
    # the fused-step kernel each bucket ran (single-pass banks mode): the
    # committed traffic record is the pipeline kernel's
    kinds = opt.bucket_kernels()
    if args.mode == "staged":
        traffic = profiled_traffic(avg_elems, "staged_step" if -1 in ev else "staged")
    else:
        traffic = (profiled_traffic(avg_elems) if kinds and all(k == Z.STEP_KERNEL_PIPE for k in kinds)
                   else None)
    if kinds:
        names = {Z.STEP_KERNEL_REGISTER: "register-streaming", Z.STEP_KERNEL_PIPE: "shared-memory pipeline",
                 Z.STEP_KERNEL_QUAD: "quad-streaming", Z.STEP_KERNEL_OCT: "oct-streaming"}
        fused_label = "fused_step per bucket: " + ", ".join(
            f"{kinds.count(k)} x {names[k]} kernel" for k in sorted(set(kinds)))
    else:
        fused_label = "statistics pass + gated update kernels"

    # ---- end to end through the public API: host gradients in, flag out
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(opt, args, stream, barrier, world_gpus)

    # ---- CPU baseline (oracle) on rank 0, single-GPU runs only
    cpu = None
    if rank == 0 and world_gpus == 1 and not args.no_cpu:
        cpu = cpu_baseline(w, args.cpu_sample)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world_gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "ms_per_step_median": ms_median,
                "ms_per_step_min_max": [min(step_ms), max(step_ms)],
                "value_from_median": whole_job_gparams(psi_p, world_gpus, ms_median),
                "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded N(0,1e-3)x65536 fp16 gradients, N(0,0.02) fp32 master)",
                "config": {"workload": w.name, "psi": sum(w.numels), "psi_padded": psi_p, "world": w.world,
                           "buckets": L.n_buckets, "bucket_elems": w.bucket_elems, "grad_dtype": args.grad_dtype,
                           "param_dtype": args.grad_dtype, "optimizer": "AdamW wd=0.01", "stage": 2,
                           "mode": args.mode, "max_grad_norm": args.max_grad_norm,
                           "passes": (PASSES[args.mode] if args.mode != "banks" or not opt.two_pass
                                      else "statistics pass (2N B/elem) + clipped update (2N + 26)"),
                           "parallelism": f"{world_gpus} GPU(s) x {w.world} simulated replicas",
                           "l2": (f"inputs larger than L2: {psi_p * bpe / 1e9:.1f} GB of HBM traffic per step"
                                  if psi_p * bpe > 4 * 126e6 else "L2-influenced (footprint < 4x L2)")},
                "hbm_gbs": value * 1e9 * bpe / world_gpus / 1e9,
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                             "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                             "kernel": ("staged step (reduce-scatter to fp32 + update from it); "
                                        "timed per step over all buckets" if args.mode == "staged" and -1 in ev else
                                        fused_label + "; timed per step over all buckets" if -1 in ev else
                                        "adam_reduced kernels (update from the fp32 reduced gradients)"
                                        if args.mode == "staged" else fused_label),
                             "bytes_per_elem": kbpe,
                             "elems_per_launch": avg_elems, "launches_timed": len(launch_ms),
                             "timed_unit": ("one step: all buckets' kernels + flag clear + flag read-back"
                                            if -1 in ev else "one bucket's kernel")},
                "gpu_launches": args.steps * L.n_buckets * (2 if opt.two_pass else 1),
                "applied_steps": applied,
                "clocks": clock,
                "e2e": e2e,
                "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if world_gpus > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_kernel_ab_passes(args):
    """--kernel-ab PSI --world N with --mode staged or inplace: the passes of
    the one-bank routes with each kernel forced in turn -- the staged
    reduce-scatter (gradients in, fp32 reduced gradients out, 2N + 4 B/elem),
    the statistics pass (gradients in, flag and norm out, 2N) and the staged
    update (reduced gradients and states in, states and parameters out, 30).
    Each call timed alone as in --kernel-ab; each kernel's reduced gradients,
    flag and norm compared with the automatic choice's (the norm within two
    fp64 summation orders).  One JSON line."""
    import torch
    import zero_sharded_optimizer_reduce_b200 as Z
    torch.cuda.set_device(0)
    peak, peak_kind = peaks()
    psi, N = args.kernel_ab, args.world
    if psi % N:
        raise SystemExit("--kernel-ab needs PSI to be a multiple of --world")
    gdt = torch.bfloat16 if args.grad_dtype == "bf16" else torch.float16
    gen = torch.Generator(device="cuda")
    grads = []
    for k in range(N):
        gen.manual_seed(workloads.seed_for(5, 1, k))
        g = torch.empty(psi, dtype=gdt, device="cuda")
        for o in range(0, psi, 1 << 27):
            e = min(psi, o + (1 << 27))
            g[o:e].copy_(torch.randn(e - o, generator=gen, device="cuda").mul_(1e-3 * 65536.0))
        grads.append(g)
    red = torch.empty(psi, device="cuda")
    st = [torch.randn(psi, device="cuda", generator=gen).mul_(0.02), torch.zeros(psi, device="cuda"),
          torch.zeros(psi, device="cuda")]
    par = torch.empty(psi, dtype=gdt, device="cuda")
    flags = torch.zeros(2, dtype=torch.int32, device="cuda")
    sq = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = torch.zeros(Z.zero_step_workspace_bytes(), dtype=torch.uint8, device="cuda")
    hp = Z.hparams(1e-3, 0.9, 0.999, 1e-8, 0.01, 1)
    small = psi * (2 * N + 4) < 4 * 126e6
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda") if small else None
    names = {Z.STEP_KERNEL_AUTO: "auto", Z.STEP_KERNEL_REGISTER: "register", Z.STEP_KERNEL_PIPE: "pipeline",
             Z.STEP_KERNEL_QUAD: "quad", Z.STEP_KERNEL_OCT: "oct"}
    passes = {
        "reduce_scatter": (2 * N + 4, lambda: Z.zero_reduce_scatter_grads(grads, psi, -1, 65536.0, red, flags[0:1],
                                                                          sq, ws)),
        "statistics": (2 * N, lambda: Z.zero_grad_stats(grads, psi, -1, 65536.0, flags[0:1], sq, ws)),
        "update": (30, lambda: Z.zero_adam_step_reduced(red, psi, *st, *st, par, hp, flags[1:2])),
    }
    reps = args.steps if psi * (2 * N + 4) > 20e9 else max(20, args.steps)
    out = {}
    try:
        # agreement: the reduced gradients, flag and norm of each kernel's
        # reduce-scatter against the automatic choice's
        ref = None
        agree = {}
        for kind, name in names.items():
            Z.zero_test_force_step_kernel(kind)
            flags.zero_()
            sq.zero_()
            passes["reduce_scatter"][1]()
            torch.cuda.synchronize()
            got = (red[::997].clone(), red[-65536:].clone(), int(flags[0].item()), float(sq.item()))
            if ref is None:
                ref = got
            else:
                agree[name] = (torch.equal(got[0].view(torch.int32), ref[0].view(torch.int32)) and
                               torch.equal(got[1].view(torch.int32), ref[1].view(torch.int32)) and
                               got[2] == ref[2] and abs(got[3] - ref[3]) <= 2.0 * psi * 2.0 ** -53 * ref[3])
        for pname, (bpe, fn) in passes.items():
            res = {}
            for kind, name in names.items():
                Z.zero_test_force_step_kernel(kind)
                for _ in range(3):
                    fn()
                times = []
                for _ in range(reps):
                    flags.zero_()
                    if small:
                        flush.fill_(1)
                    torch.cuda._sleep(200_000)
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    fn()
                    e1.record()
                    torch.cuda.synchronize()
                    times.append(e0.elapsed_time(e1))
                assert int(flags[0].item()) == 0 and int(flags[1].item()) == 0
                ms = statistics.median(times)
                gbs = psi * bpe / (ms * 1e-3) / 1e9
                res[name] = {"ms_median": ms, "gbs": gbs, "frac_measured": gbs / peak}
            out[pname] = {"bytes_per_elem": bpe, "results": res}
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)
    print(json.dumps({"kernel_ab": True, "passes": True, "psi": psi, "world": N, "grad_dtype": args.grad_dtype,
                      "reps": reps, "peak": peak, "peak_kind": peak_kind,
                      "reduce_scatter_agrees_with_auto": agree,
                      "note": "a forced kernel that cannot run a call leaves that call's automatic choice; the "
                              "staged update has register and pipeline versions only",
                      "l2": "L2-influenced (512 MB written between calls)" if small else "footprint > 4x L2",
                      "passes_timed": out}), flush=True)
    return 0


def run_kernel_ab(args):
    """The fused step at one flat point (--kernel-ab PSI --world N) with each
    step kernel forced in turn through zero_test_force_step_kernel: automatic
    choice, register, pipeline, quad, oct.  Each call timed alone as in the
    sweep (median of >= 20 calls, >= 5 above 20 GB, banks alternating, a
    sleep kernel before each, L2 written over between calls below 4x L2);
    the kernel that ran is named by zero_runner_bucket_kernel (a forced
    kernel that cannot run the call leaves the automatic choice); each
    kernel's outputs of one call from the same inputs are compared with the
    automatic choice's on a strided sample.  One JSON line."""
    import torch
    import zero_sharded_optimizer_reduce_b200 as Z
    torch.cuda.set_device(0)
    peak, peak_kind = peaks()
    psi, N = args.kernel_ab, args.world
    if psi % N:
        raise SystemExit("--kernel-ab needs PSI to be a multiple of --world")
    gdt = torch.bfloat16 if args.grad_dtype == "bf16" else torch.float16
    w = workloads.Workload(f"flat_{psi}_n{N}_{args.grad_dtype}", (psi,), N, 65536.0, 1,
                           workloads.AdamConfig(weight_decay=0.01), seed=5)
    opt = Z.ZeroAdam(w.numels, N, 0, lr=w.adam.lr, weight_decay=0.01, loss_scale=65536.0, grad_dtype=gdt,
                     param_dtype=gdt)
    fill_workload(opt, w, w.seed)
    bpe = bytes_per_elem(N)
    small = psi * bpe < 4 * 126e6
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda") if small else None
    banks = [[opt.master[0][i], opt.m[0][i], opt.v[0][i]] for i in (0, 1)]
    names = {Z.STEP_KERNEL_AUTO: "auto", Z.STEP_KERNEL_REGISTER: "register", Z.STEP_KERNEL_PIPE: "pipeline",
             Z.STEP_KERNEL_QUAD: "quad", Z.STEP_KERNEL_OCT: "oct"}

    def call(i, hp_t):
        hp = Z.hparams(w.adam.lr, w.adam.beta1, w.adam.beta2, w.adam.eps, w.adam.weight_decay, hp_t)
        Z.zero_reduce_scatter_adam_step(opt.grads[0], psi, Z.ZERO_ALL_PARTITIONS, *banks[i % 2], *banks[(i + 1) % 2],
                                        opt.params_bank[0][(i + 1) % 2], hp, 65536.0, opt.flag)

    def sample(x):
        # every 997th element and the last 65,536: a cheap comparison of two
        # kernels' outputs (the parity tests compare every element)
        return torch.cat([x[::997].contiguous().view(torch.uint8), x[-65536:].contiguous().view(torch.uint8)])

    results, ran, same = {}, {}, {}
    reps = args.steps if psi * bpe > 20e9 else max(20, args.steps)
    try:
        # first one call per kernel from the same inputs (bank 0, untouched
        # until the timing below), outputs sampled and compared with the
        # automatic choice's
        ref = None
        for kind, name in names.items():
            Z.zero_test_force_step_kernel(kind)
            ran[name] = names[opt.bucket_kernels()[0]]
            opt.flag.zero_()
            call(0, 1)
            out = [sample(x) for x in banks[1] + [opt.params_bank[0][1]]]
            if ref is None:
                ref = out
            else:
                same[name] = all(torch.equal(a, b) for a, b in zip(out, ref))
            assert int(opt.flag.item()) == 0
        for kind, name in names.items():
            Z.zero_test_force_step_kernel(kind)
            for i in range(3):
                call(i, i + 1)
            times = []
            for i in range(reps):
                opt.flag.zero_()
                if small:
                    flush.fill_(1)
                torch.cuda._sleep(200_000)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                call(i, i + 1)
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            assert int(opt.flag.item()) == 0
            ms = statistics.median(times)
            gbs = psi * bpe / (ms * 1e-3) / 1e9
            results[name] = {"kernel_ran": ran[name], "ms_median": ms, "gbs": gbs, "frac_measured": gbs / peak,
                             "sample_bit_identical_to_auto": same.get(name)}
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)
    print(json.dumps({"kernel_ab": True, "psi": psi, "world": N, "grad_dtype": args.grad_dtype,
                      "bytes_per_elem": bpe, "reps": reps, "peak": peak, "peak_kind": peak_kind,
                      "l2": "L2-influenced (512 MB written between calls)" if small else "footprint > 4x L2",
                      "results": results}), flush=True)
    return 0


def run_sweep(args):
    """Flat bandwidth sweep: psi in {1M, 16M, 256M, 1B, 2B} x N in {1..64}
    (N x 2 x psi <= 96 GB), fp16 and bf16; one JSON line per point.  Each
    step is timed on its own with CUDA events, the median of at least 20
    steps (at least --steps when a step moves more than 20 GB); when a
    point's footprint is below 4x L2 an L2-sized buffer is written between
    steps (untimed).  Each timed unit is the fused kernel call alone
    (zero_reduce_scatter_adam_step over the bucket, banks alternating); a
    short sleep kernel is queued before it so that the host's launch latency
    falls outside the events."""
    import torch
    import zero_sharded_optimizer_reduce_b200 as Z
    torch.cuda.set_device(0)
    peak, peak_kind = peaks()
    # this box's own copy rate, for reference beside the fixed peak: a
    # device-to-device copy of 4 GiB (8 GiB moved), timed like the points
    src = torch.empty(4 << 30, dtype=torch.uint8, device="cuda").fill_(1)
    dst = torch.empty_like(src)
    ctimes = []
    for i in range(23):
        torch.cuda._sleep(200_000)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src)
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            ctimes.append(e0.elapsed_time(e1))
    copy_gbs = 2 * src.numel() / (statistics.median(ctimes) * 1e-3) / 1e9
    del src, dst
    torch.cuda.empty_cache()
    print(json.dumps({"sweep": True, "copy_reference": True, "bytes_moved": 2 * (4 << 30), "reps": 20,
                      "gbs": copy_gbs, "what": "torch copy_ of a 4 GiB device buffer (a device-to-device "
                                               "cudaMemcpy): this box's copy rate, median of 20"}), flush=True)
    names = {Z.STEP_KERNEL_REGISTER: "register", Z.STEP_KERNEL_PIPE: "pipeline", Z.STEP_KERNEL_QUAD: "quad",
             Z.STEP_KERNEL_OCT: "oct"}
    # SM clocks beside every point: one sampler for the whole sweep (many
    # points time less than one sampling interval), each point given the
    # samples taken during its timed calls or, failing that, the nearest one
    clocks = ClockSampler(0, keep_samples=True)
    clocks.start()
    time.sleep(0.3)
    windows = []
    free_gb = torch.cuda.mem_get_info()[0] / 1e9
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    dtypes = [args.grad_dtype] if args.sweep_dtype_only else ["f16", "bf16"]
    for dt in dtypes:
        gdt = torch.bfloat16 if dt == "bf16" else torch.float16
        for psi, N in workloads.sweep_points():
            need = psi * (2 * N + 28) / 1e9 + 1
            if need > 0.92 * free_gb:
                print(json.dumps({"sweep": True, "psi": psi, "world": N, "grad_dtype": dt,
                                  "skipped": f"needs {need:.0f} GB"}), flush=True)
                continue
            w = workloads.Workload(f"flat_{psi}_n{N}_{dt}", (psi,), N, 65536.0, 1,
                                   workloads.AdamConfig(weight_decay=0.01), seed=5)
            opt = Z.ZeroAdam(w.numels, N, 0, lr=w.adam.lr, weight_decay=0.01, loss_scale=65536.0,
                             grad_dtype=gdt, param_dtype=gdt)
            fill_workload(opt, w, w.seed)
            bpe = bytes_per_elem(N)
            small = psi * bpe < 4 * 126e6
            banks = [[opt.master[0][i], opt.m[0][i], opt.v[0][i]] for i in (0, 1)]
            ncall = [0]

            def call():
                # the fused kernel call alone, banks alternating (the step's
                # flag clear and read-back stay outside the timed region)
                i = ncall[0]
                ncall[0] += 1
                hp = Z.hparams(w.adam.lr, w.adam.beta1, w.adam.beta2, w.adam.eps, w.adam.weight_decay, i + 1)
                Z.zero_reduce_scatter_adam_step(opt.grads[0], psi, Z.ZERO_ALL_PARTITIONS, *banks[i % 2],
                                                *banks[(i + 1) % 2], opt.params_bank[0][(i + 1) % 2], hp, 65536.0,
                                                opt.flag)
            for _ in range(3):
                call()
            times = []
            # median of >= 20 timed calls, >= 5 when a call moves more than 20 GB
            reps = args.steps if psi * bpe > 20e9 else max(20, args.steps)
            w0 = time.time()
            for _ in range(reps):
                opt.flag.zero_()
                if small:
                    flush.fill_(1)
                # keep the device busy (untimed) while the host enqueues the
                # call, so that the events bracket device time, not launch latency
                torch.cuda._sleep(200_000)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                call()
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            windows.append(((psi, N, dt), w0, time.time()))
            assert int(opt.flag.item()) == 0
            ms = statistics.median(times)
            gbs = psi * bpe / (ms * 1e-3) / 1e9
            # the runner of this one-bucket optimizer prepares the same call
            # (bank 0 -> 1), so it names the kernel the timed calls ran
            kind = opt.bucket_kernels()[0]
            print(json.dumps({"sweep": True, "psi": psi, "world": N, "grad_dtype": dt, "kernel": names[kind],
                              "kernel_ms_median": ms, "reps": reps, "gparams_s": psi / (ms * 1e-3) / 1e9, "gbs": gbs,
                              "frac_measured": gbs / peak, "frac_copy_this_run": gbs / copy_gbs,
                              "frac_nominal_8tbs": gbs / 8000.0,
                              "l2": "L2-influenced (footprint < 4x L2, flushed between steps)" if small
                              else "footprint > 4x L2"}), flush=True)
            del opt
            torch.cuda.empty_cache()
    summary = clocks.stop()
    per_point = {}
    for (psi, N, dt), w0, w1 in windows:
        inside = [x for x in clocks.samples if w0 <= x[0] <= w1]
        if not inside and clocks.samples:
            inside = [min(clocks.samples, key=lambda x: min(abs(x[0] - w0), abs(x[0] - w1)))]
        if inside:
            per_point[f"{dt}/{psi}/{N}"] = {"sm_mhz": statistics.median(x[1] for x in inside),
                                            "reasons": sorted({r for x in inside for r in x[2]}),
                                            "samples": len(inside)}
    print(json.dumps({"sweep": True, "clocks": summary, "clocks_by_point": per_point,
                      "note": "SM clock per point: the samples taken during its timed calls, else the nearest"}),
          flush=True)
    return 0


def run_stage3(args):
    """Layer-wise ZeRO-3 step on the 6.7B GPT shape (32 layers + embedding
    unit, N = 8): two gathers per unit plus the per-unit staged reduce-scatter
    and gated in-place update, timed without gather prefetch (the value) and
    with it, and with the statistics-pass update for comparison.  One JSON
    line."""
    import torch
    import zero_sharded_optimizer_reduce_b200 as Z
    torch.cuda.set_device(0)
    w = workloads.gpt_6p7b_layerwise()
    out = {}
    for prefetch, update in ((False, "staged"), (False, "stats"), (True, "staged")):
        s3 = Z.ZeroStage3(w.numels, w.world, lr=w.adam.lr, betas=(w.adam.beta1, w.adam.beta2), eps=w.adam.eps,
                          weight_decay=w.adam.weight_decay, loss_scale=w.loss_scale, prefetch=prefetch,
                          update=update)
        gen = torch.Generator(device="cuda")
        for u in range(s3.U):
            gen.manual_seed(4000 + u)
            s3.master[u].normal_(0.0, w.master_std, generator=gen)
            s3.master[u][s3.layout.bucket_numel[u]:].zero_()
        for k, g in enumerate(s3.grads):
            gen.manual_seed(5000 + k)
            g.copy_(torch.randn(g.numel(), generator=gen, device="cuda").mul_(w.grad_std * w.loss_scale))
        s3.load(list(s3.master))
        for _ in range(args.warmup):
            s3.step()
        torch.cuda.synchronize()
        # ncu --profile-from-start off captures the timed steps of the value's
        # configuration (no prefetch, staged update) only
        headline = not prefetch and update == "staged"
        if headline:
            torch.cuda.profiler.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            s3.step()
        e1.record()
        torch.cuda.synchronize()
        if headline:
            torch.cuda.profiler.stop()
        out[(prefetch, update)] = e0.elapsed_time(e1) / args.steps
        if prefetch and update == "staged":
            # the all-gather alone: unit 0 from the 8 shards into a layer buffer
            for _ in range(3):
                s3.unit_params(0, s3.layer[0][:s3.layout.bucket_padded[0]])
            torch.cuda.synchronize()
            e0.record()
            for _ in range(20):
                s3.unit_params(0, s3.layer[0][:s3.layout.bucket_padded[0]])
            e1.record()
            torch.cuda.synchronize()
            gather_ms = e0.elapsed_time(e1) / 20
            gather_elems = s3.layout.bucket_padded[0]
        del s3
        torch.cuda.empty_cache()
    psi = sum(Z.zero_partition_layout(w.numels, w.world, 1, 8).bucket_padded)
    N = w.world
    bpe = 8 + 2 * N + 34          # 2 gathers x (2 read + 2 write) + reduce-scatter to fp32 + update
    bpe_stats = 8 + 4 * N + 26    # 2 gathers + statistics pass + fused gated update
    # the default configuration (no prefetch: on one GPU the side stream only
    # competes for the same HBM) is the line's value; prefetch is reported beside it
    best = out[(False, "staged")]
    peak, peak_kind = peaks()
    line = {"metric": "ZeRO-3 layer-wise step (gathers + staged reduce-scatter + gated in-place update)",
            "unit": "Gparams/s", "value": psi / (best * 1e-3) / 1e9, "ms_per_step": best,
            "ms_per_step_prefetch": out[(True, "staged")],
            "prefetch_gain": best / out[(True, "staged")] - 1.0, "steps": args.steps, "warmup": args.warmup,
            "config": {"workload": w.name, "psi_padded": psi, "world": N, "units": len(w.numels)},
            "hbm_gbs": psi * bpe / (best * 1e-3) / 1e9, "bytes_per_elem": bpe,
            "frac_measured": psi * bpe / (best * 1e-3) / 1e9 / peak, "peak_kind": peak_kind,
            "stats_update": {"ms_per_step": out[(False, "stats")], "bytes_per_elem": bpe_stats,
                             "value": psi / (out[(False, "stats")] * 1e-3) / 1e9,
                             "frac_measured": psi * bpe_stats / (out[(False, "stats")] * 1e-3) / 1e9 / peak},
            "allgather": {"elements": gather_elems, "ms": gather_ms, "bytes_per_elem": 4,
                          "gbs": gather_elems * 4 / (gather_ms * 1e-3) / 1e9,
                          "frac_measured": gather_elems * 4 / (gather_ms * 1e-3) / 1e9 / peak,
                          "note": "2 B read + 2 B write per element; one unit (201M elements) from 8 shards"}}
    print(json.dumps(line), flush=True)
    return 0


def p2p_bytes_per_rank(parts, world: int, grad_esize: int, param_esize: int, mode: str) -> dict:
    """Bytes one rank moves between GPUs per step of the one-process-per-GPU
    routes, from its partition (or unit slice) sizes `parts`:

    - ZeRO-2 (mode "banks" / "staged"): the reduce-scatter reads slice r of
      every peer's gradient buffer, (N - 1) P gradient elements per bucket;
      the all-gather moves every peer's slot of P parameters, (N - 1) P
      elements (the banks mode reads the peers' slots, the staged update
      stores its own slot into every peer's buffer).  Together 2 (N - 1) P
      elements, which sums to 2 Psi (N - 1) / N per rank: the pages' "2 Psi
      per GPU" of data parallelism (ZeRO explainer, communication-volume
      paragraphs).
    - Stage 3 (mode "stage3"): two gathers of every unit (forward and
      backward) plus its reduce-scatter: 3 (N - 1) P elements, 1.5 x the
      above.
    """
    peers = world - 1
    pull = sum(peers * P * grad_esize for P in parts)
    gather = sum(peers * P * param_esize for P in parts) * (2 if mode == "stage3" else 1)
    elems = sum(peers * P for P in parts) * (3 if mode == "stage3" else 2)
    kind = {"banks": "peer reads after the commit", "staged": "the update's own stores into every peer's buffer",
            "stage3": "peer reads, forward and backward"}[mode]
    return {"pull_bytes": pull, "gather_bytes": gather, "gather_kind": kind, "elements_moved": elems}


def run_distributed(args):
    """The ZeRO-2 step (or, with --stage3, the layer-wise ZeRO-3 step) with one
    process per GPU: each process is one data-parallel rank of the real
    method, holding its own replica's gradients, its 1/N of the fp32 states
    and (ZeRO-2) the full parameter buckets or (ZeRO-3) its parameter shard;
    the reduce-scatter pulls the peers' gradient slices through CUDA IPC
    mappings inside the kernel, the all-gather moves the updated slots.
    World size = number of processes (the data-parallel degree).  Each step
    is timed with CUDA events on every rank; the slowest rank's time is
    reported.  Host barriers order the ranks (no kernel waits on another
    rank), so several ranks may share one GPU for a functional run
    (--dist-backend gloo)."""
    import datetime
    import torch
    import torch.distributed as dist
    import zero_sharded_optimizer_reduce_b200 as Z

    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29531")
    os.environ.setdefault("RANK", "0")
    os.environ.setdefault("WORLD_SIZE", "1")
    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local % torch.cuda.device_count())
    torch.cuda.set_device(dev)
    kw = {"device_id": dev} if args.dist_backend == "nccl" else {}
    dist.init_process_group(args.dist_backend, timeout=datetime.timedelta(seconds=300), **kw)
    red_dev = "cuda" if args.dist_backend == "nccl" else "cpu"
    gdt = torch.bfloat16 if args.grad_dtype == "bf16" else torch.float16
    chunk = 1 << 27

    def randn_into(buf, seed, std):
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        for o in range(0, buf.numel(), chunk):
            e = min(buf.numel(), o + chunk)
            buf[o:e].copy_(torch.randn(e - o, generator=g, device=dev).mul_(std))

    if args.stage3:
        w = workloads.gpt_6p7b_layerwise()
        if args.flat:       # a small stand-in shape: 4 units of --flat elements
            w = workloads.Workload(f"flat_4x{args.flat}_layerwise", (args.flat,) * 4, w.world, w.loss_scale, 1,
                                   w.adam, seed=w.seed)
        opt = Z.DistributedZeroStage3(w.numels, lr=w.adam.lr, betas=(w.adam.beta1, w.adam.beta2), eps=w.adam.eps,
                                      weight_decay=w.adam.weight_decay, loss_scale=w.loss_scale, grad_dtype=gdt,
                                      param_dtype=gdt)
        L = opt.layout
        masters = []
        for u in range(opt.U):
            m = torch.empty(L.bucket_padded[u], dtype=torch.float32, device=dev)
            randn_into(m, 4000 + u, w.master_std)
            m[L.bucket_numel[u]:].zero_()
            masters.append(m)
        opt.load(masters)
        del masters
        # this rank's replica gradients: one seeded buffer the size of the
        # largest unit; each unit's backward copies its prefix in (the copy
        # stands in for the backward pass writing the unit's gradients)
        src = torch.empty(max(L.bucket_padded), dtype=gdt, device=dev)
        randn_into(src, workloads.seed_for(w.seed + 100, 1, rank), w.grad_std * w.loss_scale)

        def grad_fill(u, buf):
            buf.copy_(src[:buf.numel()])
            buf[L.bucket_numel[u]:].zero_()

        step = lambda: opt.step(grad_fill)
        parts = opt.parts
        mode = "stage3"
        metric = "ZeRO-3 layer-wise step, one process per GPU: Gparams/s"
    else:
        w = select_workload(args)
        opt = Z.DistributedZeroAdam(w.numels, w.bucket_elems, 8, lr=w.adam.lr, betas=(w.adam.beta1, w.adam.beta2),
                                    eps=w.adam.eps, weight_decay=w.adam.weight_decay, loss_scale=w.loss_scale,
                                    grad_dtype=gdt, param_dtype=gdt, mode=args.distributed)
        L = opt.layout
        masters, params = [], []
        for b in range(L.n_buckets):
            randn_into(opt.grads[b], workloads.seed_for(w.seed + 100, 1, rank) + 7919 * b, w.grad_std * w.loss_scale)
            opt.grads[b][L.bucket_numel[b]:].zero_()
            m = torch.empty(L.bucket_padded[b], dtype=torch.float32, device=dev)
            randn_into(m, 7 * w.seed + b, w.master_std)        # the same on every rank
            m[L.bucket_numel[b]:].zero_()
            masters.append(m)
            params.append(m.to(gdt))
        opt.load(masters, params)
        del masters, params
        step = opt.step
        parts = [L.part(b) for b in range(L.n_buckets)]
        mode = args.distributed
        metric = "ZeRO-2 step, one process per GPU (P2P reduce-scatter + update + all-gather): Gparams/s"
    psi_p = sum(L.bucket_padded)
    torch.cuda.synchronize()

    def barrier():
        torch.cuda.synchronize()
        dist.barrier()

    for _ in range(args.warmup):
        step()
    barrier()
    stream = torch.cuda.current_stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    applied = 0
    evs[0].record(stream)
    for i in range(args.steps):
        applied += bool(step())
        evs[i + 1].record(stream)
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in zip(evs[:-1], evs[1:])]
    ms = max_over_ranks(sum(step_ms) / args.steps, red_dev)
    ms_median = max_over_ranks(statistics.median(step_ms), red_dev)
    esize = torch.empty((), dtype=gdt).element_size()
    moved = p2p_bytes_per_rank(parts, world, esize, esize, mode)
    per_rank_gbs = (moved["pull_bytes"] + moved["gather_bytes"]) / (ms * 1e-3) / 1e9
    if rank == 0:
        line = {"metric": metric, "value": psi_p / (ms * 1e-3) / 1e9, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_median": ms_median,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded, per-rank gradients)",
                "config": {"workload": w.name, "psi_padded": psi_p, "world": world, "mode": f"distributed-{mode}",
                           "units_or_buckets": L.n_buckets, "backend": args.dist_backend,
                           "gpus_visible": torch.cuda.device_count(),
                           "parallelism": f"dp{world}: one process per rank, P2P through CUDA IPC"},
                "p2p": dict(moved, per_rank_gbs=per_rank_gbs,
                            note="bytes each rank moves between GPUs per step; GB/s over the whole step time "
                                 "(host barriers and the local HBM passes included)"),
                "applied_steps": applied}
        print(json.dumps(line), flush=True)
    opt.close()
    del opt
    dist.destroy_process_group()
    return 0


def run_allgather(args):
    """The all-gather reconstruct alone (zero_allgather_params): --world
    slices of --allgather elements (fp16 or bf16) gathered into one buffer,
    the L2 written over between calls (untimed) and a short sleep kernel
    queued before each, CUDA events around the call, median of at least 20.
    An odd slice size puts every rank but the first off its destination's
    16-byte phase (the realigning kernel).  torch.cat of the same slices is
    timed the same way, for comparison.  4 bytes per element (2 read, 2
    written).  One JSON line."""
    import torch
    import zero_sharded_optimizer_reduce_b200 as Z
    torch.cuda.set_device(0)
    N, P = args.world, args.allgather
    dt = torch.bfloat16 if args.grad_dtype == "bf16" else torch.float16
    gen = torch.Generator(device="cuda")
    shards = []
    for r in range(N):
        gen.manual_seed(8000 + r)
        shards.append(torch.randn(P, generator=gen, device="cuda").to(dt))
    dst = torch.empty(N * P, dtype=dt, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    Z.zero_allgather_params(shards, 0, P, dst, status=status)
    torch.cuda.synchronize()
    assert torch.equal(dst.view(torch.int16), torch.cat(shards).view(torch.int16)) and int(status.item()) == 0

    def timed(fn, reps):
        for _ in range(3):
            fn()
        t = []
        for _ in range(reps):
            flush.fill_(1)
            torch.cuda._sleep(200_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            t.append(e0.elapsed_time(e1))
        return statistics.median(t)

    reps = max(20, args.steps)
    torch.cuda.profiler.start()
    ms = timed(lambda: Z.zero_allgather_params(shards, 0, P, dst, status=status), reps)
    torch.cuda.profiler.stop()
    ms_cat = timed(lambda: torch.cat(shards, out=dst), reps)
    peak, peak_kind = peaks()
    gbs = 4.0 * N * P / (ms * 1e-3) / 1e9
    gbs_cat = 4.0 * N * P / (ms_cat * 1e-3) / 1e9
    phases = sorted({(2 * r * P) % 16 for r in range(N)})
    print(json.dumps({"metric": "all-gather reconstruct (zero_allgather_params): achieved HBM GB/s",
                      "value": gbs, "unit": "GB/s", "ms_median": ms, "reps": reps, "world": N, "part_numel": P,
                      "dtype": args.grad_dtype, "bytes_per_elem": 4, "frac_measured": gbs / peak, "peak": peak,
                      "peak_kind": peak_kind, "dst_phases_bytes": phases,
                      "l2": "512 MB written between calls (untimed)",
                      "torch_cat": {"ms_median": ms_cat, "gbs": gbs_cat, "frac_measured": gbs_cat / peak}}),
          flush=True)
    return 0


def run_e2e(opt, args, stream, barrier, world_gpus):
    """Same step through ZeroAdam.step_from_host: every step copies the N
    replicas' gradients from pinned host memory and reads the flag back."""
    import torch
    short = 0.0
    try:
        import psutil
        need = sum(g.numel() * g.element_size() for per in opt.grads for g in per)
        if psutil.virtual_memory().available < 1.5 * need * max(1, world_gpus):
            short = 1.0
    except Exception:
        pass
    # every rank takes the same branch (the timed part below has collectives)
    if max_over_ranks(short, "cuda") > 0:
        return {"value": None, "unit": UNIT, "skipped": "not enough host memory for pinned gradients"}
    host = [[torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in per] for per in opt.grads]
    for b, per in enumerate(opt.grads):
        for k, g in enumerate(per):
            host[b][k].copy_(g)
    h2d = sum(h.numel() * h.element_size() for per in host for h in per)
    steps = max(1, min(args.steps, args.e2e_steps))
    opt.step_from_host(host)
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        opt.step_from_host(host)
    t1.record(stream)
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), "cuda")
    psi_p = sum(opt.layout.bucket_padded)
    del host
    return {"value": whole_job_gparams(psi_p, world_gpus, ms / steps), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4, "steps": steps,
            "ms_per_step": ms / steps}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=1 << 26)
    ap.add_argument("--ref-sample", type=int, default=1 << 26)
    ap.add_argument("--flat", type=int, default=0, help="flat workload of this many elements instead of GPT-2")
    ap.add_argument("--world", type=int, default=8, help="simulated replicas of the flat workload")
    ap.add_argument("--grad-dtype", choices=["f16", "bf16"], default="f16")
    ap.add_argument("--sweep", action="store_true", help="flat bandwidth sweep, one JSON line per point")
    ap.add_argument("--stage3", action="store_true", help="layer-wise ZeRO-3 step on the 6.7B shape, prefetch on/off")
    ap.add_argument("--mode", choices=["banks", "inplace", "staged"], default="banks",
                    help="banks: two state banks, one pass; inplace: one bank, statistics pass + gated update; "
                         "staged: one bank, reduce-scatter to fp32 + gated update")
    ap.add_argument("--max-grad-norm", type=float, default=None, help="clip gradients to this global norm")
    ap.add_argument("--sweep-dtype-only", action="store_true", help="sweep only --grad-dtype")
    ap.add_argument("--cpu-configs", action="store_true",
                    help="time the CPU oracle on every workload (full arrays or 64M slices), one JSON line")
    ap.add_argument("--kernel-ab", type=int, default=0,
                    help="time the fused step on a flat bucket of this many elements (--world N) with each "
                         "step kernel forced in turn, one JSON line")
    ap.add_argument("--allgather", type=int, default=0,
                    help="time the all-gather of --world slices of this many elements, one JSON line")
    ap.add_argument("--distributed", choices=["banks", "staged"], default=None,
                    help="one process per GPU (under torchrun): the multi-process ZeRO-2 route in this mode; "
                         "with --stage3 the multi-process layer-wise ZeRO-3 route")
    ap.add_argument("--dist-backend", choices=["nccl", "gloo"], default="nccl",
                    help="process-group backend of the --distributed host barriers (gloo lets ranks share a GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    if args.cpu_configs:
        return run_cpu_configs(args)
    if args.sweep:
        return run_sweep(args)
    if args.kernel_ab:
        return run_kernel_ab_passes(args) if args.mode != "banks" else run_kernel_ab(args)
    if args.allgather:
        return run_allgather(args)
    if args.distributed is not None:
        return run_distributed(args)
    if args.stage3:
        return run_stage3(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
