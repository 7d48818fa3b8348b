"""ZeroStage3: the ZeRO-3 layer-wise step on one GPU, optional gather prefetch.

ZeRO explainer, "Stage 3 - Parameter Partitioning (P_os+g+p)": each rank
keeps only its 1/N slice of every parameter; a layer's full parameters are
rebuilt by all-gather before its forward and again before its backward, then
dropped; the communication paragraph counts these two extra all-gathers.

Simulation on one GPU, per unit u (a transformer layer or the embedding):
  - parameters live only as N rank-major shards (shard r = concatenation
    over units of unit slice r); `gather(u)` rebuilds unit u in one of two
    reused layer buffers (zero_allgather_params);
  - fp32 master / m / v per unit in flat (rank-major) order, one bank;
  - N replica gradient buffers, reused by every unit; `grad_fill(u, bufs)`
    stands for the backward pass that produces unit u's gradients;
  - the update of unit u, update="staged" (default): the reduce-scatter of
    the unit stores every rank's reduced fp32 gradients (and the unit's
    overflow flag) in a reused buffer, then one gated call per rank r updates
    slice r in place from them and writes the new parameters into shard r's
    slot of unit u: 2N + 34 bytes per element.  update="stats": a
    statistics pass over the unit, then one gated fused call per rank that
    re-reads the N replicas: 4N + 26 bytes per element.
Step: forward gathers u = 0 .. U-1, then for u = U-1 .. 0: gather, gradients,
update.  With prefetch, the gather of the next unit runs on a side stream
into the other layer buffer while the current unit's work runs; events order
the buffers.  On one GPU both streams share HBM, so prefetch can only fill
the gaps between kernels: measured on B200 (6.7B shape) it cost 3 % (62.5
against 60.6 ms per step), so it is off by default here; it pays where the
gathers come over NVLink.

Skip scope: each unit's update is gated by that unit's own statistics (the
units' gradients never coexist in memory); the host reads the per-unit flags
at the end of the step for the loss scale.  t advances when no unit
overflowed.
"""
from __future__ import annotations

import torch

from . import (hparams, zero_adam_step_reduced, zero_allgather_params, zero_grad_stats, zero_loss_scale_update,
               zero_partition_layout, zero_reduce_scatter_adam_step_gated, zero_reduce_scatter_grads)


class ZeroStage3:
    def __init__(self, unit_numels, world: int, *, align_elems: int = 8, lr: float = 1e-3, betas=(0.9, 0.999),
                 eps: float = 1e-8, weight_decay: float = 0.0, grad_dtype=torch.float16,
                 param_dtype=torch.float16, loss_scale: float = 65536.0, growth_interval: int = 1000,
                 min_scale: float = 1.0, prefetch: bool = False, update: str = "staged", device="cuda"):
        if update not in ("staged", "stats"):
            raise ValueError("update must be 'staged' or 'stats'")
        self.update_mode = update
        self.world = world
        self.layout = L = zero_partition_layout(list(unit_numels), world, 1, align_elems)   # one unit per bucket
        self.U = L.n_buckets
        self.parts = [L.part(u) for u in range(self.U)]
        self.shard_off = [0]
        for p in self.parts:
            self.shard_off.append(self.shard_off[-1] + p)
        dev = self.device = torch.device(device)
        self.lr, self.betas, self.eps, self.weight_decay = lr, betas, eps, weight_decay
        self.scale, self.good_steps, self.t = float(loss_scale), 0, 0
        self.growth_interval, self.min_scale = growth_interval, min_scale
        self.prefetch = prefetch
        self.grad_dtype, self.param_dtype = grad_dtype, param_dtype
        self.shards = [torch.zeros(self.shard_off[-1], dtype=param_dtype, device=dev) for _ in range(world)]
        f32 = dict(dtype=torch.float32, device=dev)
        self.master = [torch.zeros(L.bucket_padded[u], **f32) for u in range(self.U)]
        self.m = [torch.zeros(L.bucket_padded[u], **f32) for u in range(self.U)]
        self.v = [torch.zeros(L.bucket_padded[u], **f32) for u in range(self.U)]
        mx = max(L.bucket_padded)
        self.grads = [torch.zeros(mx, dtype=grad_dtype, device=dev) for _ in range(world)]
        self.reduced = torch.zeros(mx, **f32) if update == "staged" else None
        self.layer = [torch.zeros(mx, dtype=param_dtype, device=dev) for _ in range(2)]
        self.unit_flags = torch.zeros(self.U, dtype=torch.int32, device=dev)
        self.step_flag = torch.zeros(1, dtype=torch.int32, device=dev)
        self.side = torch.cuda.Stream(device=dev)
        self.gathers = 0

    # ---------------------------------------------------------------- state
    def load(self, unit_master) -> None:
        """unit_master[u]: fp32 master of unit u (padded, flat).  The shards
        get the low-precision copy; m = v = 0."""
        for u in range(self.U):
            self.master[u].copy_(unit_master[u])
            self.m[u].zero_()
            self.v[u].zero_()
            P = self.parts[u]
            for r in range(self.world):
                self.shards[r][self.shard_off[u]:self.shard_off[u] + P].copy_(self.master[u][r * P:(r + 1) * P])
        torch.cuda.synchronize()
        self.t = 0

    def unit_params(self, u: int, out=None):
        """Gather unit u's full parameters (synchronously) into `out` or a new tensor."""
        P = self.parts[u]
        out = torch.empty(self.layout.bucket_padded[u], dtype=self.param_dtype, device=self.device) \
            if out is None else out
        zero_allgather_params(self.shards, self.shard_off[u], P, out)
        return out

    # ----------------------------------------------------------------- step
    def _gather(self, u: int, buf: int, stream) -> None:
        P = self.parts[u]
        zero_allgather_params(self.shards, self.shard_off[u], P, self.layer[buf][:self.layout.bucket_padded[u]],
                              stream)
        self.gathers += 1

    def _update(self, u: int, hp) -> None:
        L, P = self.layout, self.parts[u]
        pad = L.bucket_padded[u]
        g = [x[:pad] for x in self.grads]
        flag = self.unit_flags[u:u + 1]
        if self.update_mode == "staged":
            red = self.reduced[:pad]
            zero_reduce_scatter_grads(g, pad, -1, self.scale, red, flag)
            for r in range(self.world):
                sl = slice(r * P, (r + 1) * P)
                zero_adam_step_reduced(red[sl], P, self.master[u][sl], self.m[u][sl], self.v[u][sl],
                                       self.master[u][sl], self.m[u][sl], self.v[u][sl],
                                       self.shards[r][self.shard_off[u]:self.shard_off[u] + P],
                                       hp, self.step_flag, gate=flag)
            return
        zero_grad_stats(g, pad, -1, self.scale, flag)
        for r in range(self.world):
            sl = slice(r * P, (r + 1) * P)
            zero_reduce_scatter_adam_step_gated(
                g, pad, r, self.master[u][sl], self.m[u][sl], self.v[u][sl],
                self.master[u][sl], self.m[u][sl], self.v[u][sl],
                self.shards[r][self.shard_off[u]:self.shard_off[u] + P],
                hp, self.scale, self.step_flag, gate=flag)

    def step(self, grad_fill=None) -> bool:
        """One layer-wise step; grad_fill(u, grad_bufs) writes unit u's N
        replica gradients (on the current stream).  Returns True when no
        unit overflowed."""
        main = torch.cuda.current_stream(self.device)
        self.unit_flags.zero_()
        self.step_flag.zero_()
        hp = hparams(self.lr, self.betas[0], self.betas[1], self.eps, self.weight_decay, self.t + 1)
        U = self.U
        order = list(range(U)) + list(range(U - 1, -1, -1))     # forward, then backward
        if not self.prefetch:
            for i, u in enumerate(order):
                self._gather(u, i % 2, main)
                if i >= U:
                    if grad_fill is not None:
                        grad_fill(u, self.grads)
                    self._update(u, hp)
        else:
            done = [torch.cuda.Event() for _ in order]
            free = [torch.cuda.Event() for _ in range(2)]
            for e in free:
                e.record(main)
            # the side stream runs the gathers one ahead of the main stream
            self.side.wait_stream(main)
            with torch.cuda.stream(self.side):
                self.side.wait_event(free[0])
                self._gather(order[0], 0, self.side)
                done[0].record(self.side)
            for i, u in enumerate(order):
                if i + 1 < len(order):
                    with torch.cuda.stream(self.side):
                        self.side.wait_event(free[(i + 1) % 2])
                        self._gather(order[i + 1], (i + 1) % 2, self.side)
                        done[i + 1].record(self.side)
                main.wait_event(done[i])           # unit u's full parameters are in layer[i % 2]
                if i >= U:
                    if grad_fill is not None:
                        grad_fill(u, self.grads)
                    self._update(u, hp)
                free[i % 2].record(main)           # layer[i % 2] may be overwritten
            main.wait_stream(self.side)
        flags = self.unit_flags.cpu()
        ovf = bool(flags.any()) or bool(self.step_flag.item() & 2)
        if int(self.step_flag.item()) & 2:
            raise RuntimeError("fused step kernel timed out waiting on its copy pipeline")
        if not ovf:
            self.t += 1
        self.scale, self.good_steps = zero_loss_scale_update(self.scale, self.good_steps, ovf,
                                                             self.growth_interval, self.min_scale)
        return not ovf
