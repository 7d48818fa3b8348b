"""DistributedZeroStage3: the layer-wise ZeRO-3 step with one process per rank.

ZeRO explainer, "Stage 3 - Parameter Partitioning (P_os+g+p)": each rank
keeps only its 1/N slice of every parameter, of the gradients and of the
optimizer states; a unit's full parameters are rebuilt by all-gather before
its forward and again before its backward, then dropped.

Each process (rank r of N on one node) holds:
  - its shard: the concatenation over units of its slice of each unit's
    low-precision parameters (the only parameter memory it keeps),
  - fp32 master / m / v of its slices (one bank) and a reduced-gradient
    buffer of one slice,
  - one unit's worth of its own replica's gradients (reused by every unit)
    and one layer buffer for the gathered unit.

Peers' shards and gradient buffers are mapped once through CUDA IPC.  A step:
  forward:  for every unit, gather it from every rank's shard (peer reads);
  backward: for every unit in reverse, gather it again, let the caller write
    this rank's gradients of the unit, host barrier, then the staged
    reduce-scatter with partition = r reads slice r of every rank's gradient
    buffer in rank order (the fixed fp32 order of the oracle) into the
    reduced buffer and the unit's flag; the flags are OR-ed over the group,
    and when no rank saw inf / NaN the update runs in place on this rank's
    slice and writes its shard; host barrier before the gradient buffers
    are reused.
Skip scope: a unit whose reduced gradients overflowed on any rank is left
unchanged on every rank; t advances when no unit overflowed (the units'
gradients never coexist, so the step cannot wait for all of them).
No kernel waits on another rank: all ordering is host barriers.  This class
sequences library calls; all arithmetic runs in libzero's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (DevicePtr, hparams, zero_adam_step_reduced, zero_allgather_params, zero_ipc_close, zero_ipc_export,
               zero_ipc_import, zero_loss_scale_update, zero_partition_layout, zero_reduce_scatter_grads)


class DistributedZeroStage3:
    def __init__(self, unit_numels, *, align_elems: int = 8, group=None, lr: float = 1e-3, betas=(0.9, 0.999),
                 eps: float = 1e-8, weight_decay: float = 0.0, grad_dtype=torch.float16,
                 param_dtype=torch.float16, loss_scale: float = 65536.0, growth_interval: int = 1000,
                 min_scale: float = 1.0, device="cuda"):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.device = dev = torch.device(device)
        self.layout = L = zero_partition_layout(list(unit_numels), self.world, 1, align_elems)   # one unit per bucket
        self.U = L.n_buckets
        self.parts = [L.part(u) for u in range(self.U)]
        self.shard_off = [0]
        for p in self.parts:
            self.shard_off.append(self.shard_off[-1] + p)
        self.lr, self.betas, self.eps, self.weight_decay = lr, betas, eps, weight_decay
        self.scale, self.good_steps, self.t = float(loss_scale), 0, 0
        self.growth_interval, self.min_scale = growth_interval, min_scale
        self.grad_dtype, self.param_dtype = grad_dtype, param_dtype
        f32 = dict(dtype=torch.float32, device=dev)
        self.shard = torch.zeros(self.shard_off[-1], dtype=param_dtype, device=dev)
        self.master = [torch.zeros(p, **f32) for p in self.parts]
        self.m = [torch.zeros(p, **f32) for p in self.parts]
        self.v = [torch.zeros(p, **f32) for p in self.parts]
        mx = max(L.bucket_padded)
        self.grads = torch.zeros(mx, dtype=grad_dtype, device=dev)
        self.reduced = torch.zeros(max(self.parts), **f32)
        self.layer = torch.zeros(mx, dtype=param_dtype, device=dev)
        self.flags = torch.zeros(2, dtype=torch.int32, device=dev)   # [unit flag, update status]
        self.gathers = 0
        self._map_peers()

    # ------------------------------------------------------------------ IPC
    def _map_peers(self) -> None:
        mine = (zero_ipc_export(self.shard), zero_ipc_export(self.grads))
        everyone = [None] * self.world
        dist.all_gather_object(everyone, mine, group=self.group)
        self._bases = []
        self.peer_shards, self.peer_grads = [], []
        for q in range(self.world):
            if q == self.rank:
                self.peer_shards.append(self.shard)
                self.peer_grads.append(None)
                continue
            (sh, so), (gh, go) = everyone[q]
            sptr, sbase = zero_ipc_import(sh, so)
            gptr, gbase = zero_ipc_import(gh, go)
            self._bases += [sbase, gbase]
            self.peer_shards.append(DevicePtr(sptr, self.param_dtype))
            self.peer_grads.append(DevicePtr(gptr, self.grad_dtype))

    def close(self) -> None:
        """Unmap the peers' buffers (call on every rank before exit)."""
        torch.cuda.synchronize()
        dist.barrier(group=self.group)
        for base in self._bases:
            zero_ipc_close(base)
        self._bases = []

    # ---------------------------------------------------------------- state
    def load(self, unit_master) -> None:
        """unit_master[u]: fp32 master of unit u (padded, flat, the same on
        every rank).  This rank keeps its slice; the shard gets its
        low-precision copy; m = v = 0."""
        r = self.rank
        for u in range(self.U):
            P = self.parts[u]
            self.master[u].copy_(unit_master[u][r * P:(r + 1) * P])
            self.m[u].zero_()
            self.v[u].zero_()
            self.shard[self.shard_off[u]:self.shard_off[u] + P].copy_(self.master[u])
        torch.cuda.synchronize()
        dist.barrier(group=self.group)
        self.t = 0

    def gather(self, u: int, out=None):
        """Unit u's full parameters from every rank's shard (rank order)."""
        pad = self.layout.bucket_padded[u]
        out = self.layer[:pad] if out is None else out
        zero_allgather_params(self.peer_shards, self.shard_off[u], self.parts[u], out)
        self.gathers += 1
        return out

    # ----------------------------------------------------------------- step
    def _or_over_ranks(self, flag: int) -> int:
        backend = dist.get_backend(self.group)
        t = torch.tensor([flag], dtype=torch.int32, device=self.device if backend == "nccl" else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=self.group)
        return int(t.item())

    def step(self, grad_fill) -> bool:
        """One layer-wise step.  grad_fill(u, buf) writes this rank's replica
        gradients of unit u into buf (padded length).  Returns True when no
        unit overflowed on any rank."""
        L, r = self.layout, self.rank
        hp = hparams(self.lr, self.betas[0], self.betas[1], self.eps, self.weight_decay, self.t + 1)
        for u in range(self.U):                         # forward reconstruct
            self.gather(u)
        all_ok = True
        for u in range(self.U - 1, -1, -1):             # backward
            pad, P = L.bucket_padded[u], self.parts[u]
            self.gather(u)
            grad_fill(u, self.grads[:pad])
            torch.cuda.synchronize()
            dist.barrier(group=self.group)              # every rank's gradients of unit u are written
            self.flags.zero_()
            bufs = [self.grads[:pad] if q == r else self.peer_grads[q] for q in range(self.world)]
            zero_reduce_scatter_grads(bufs, pad, r, self.scale, self.reduced[:P], self.flags[0:1])
            ovf = self._or_over_ranks(int(self.flags[0].item()))     # synchronizes this rank's stream
            if ovf & 2:
                raise RuntimeError("reduce-scatter kernel timed out waiting on its copy pipeline")
            if ovf == 0:
                st = (self.master[u], self.m[u], self.v[u])
                zero_adam_step_reduced(self.reduced[:P], P, *st, *st,
                                       self.shard[self.shard_off[u]:self.shard_off[u] + P], hp, self.flags[1:2])
            else:
                all_ok = False
            torch.cuda.synchronize()
            if int(self.flags[1].item()) & 2:
                raise RuntimeError("staged update timed out waiting on its copy pipeline; states incomplete")
            dist.barrier(group=self.group)              # nobody still reads a gradient buffer
        if all_ok:
            self.t += 1
        self.scale, self.good_steps = zero_loss_scale_update(self.scale, self.good_steps, not all_ok,
                                                             self.growth_interval, self.min_scale)
        return all_ok
