"""DistributedZeroAdam: the ZeRO-2 step with one process per data-parallel rank.

Each process (rank r of N on one node) holds:
  - its own replica's gradient buckets (full padded buckets, as a backward
    pass produces them),
  - only its partition of the fp32 master / momentum / variance states
    (P = padded / N elements per bucket, two banks for the exact skip),
  - the full low-precision parameter buckets (the all-gather target).

A step (ZeRO explainer, "Stage 2 - Gradient Partitioning (P_os+g)"):
  1. host barrier: every rank's gradients are written;
  2. the fused kernel with partition = r reads rank r's slice of every peer's
     gradient buffer through CUDA IPC mappings, in rank order (the reduce-
     scatter happens inside the kernel: P2P loads over NVLink between GPUs),
     unscales, tests for overflow, updates the partition and writes the new
     parameters into slot r of this rank's own parameter buffer;
  3. the overflow flags are OR-ed over the process group (all ranks skip or
     commit together), banks flip, the loss scale updates;
  4. host barrier, then every rank copies the peers' updated slots from
     their parameter buffers (the all-gather, again through the mappings);
  5. host barrier: nobody overwrites a buffer a peer is still reading.

mode="staged" keeps one bank of partition states (the pages' 12 Psi / N
bytes) plus the partition's reduced fp32 gradients (4 Psi / N): step 2 is
the staged reduce-scatter (the same peer reads, storing the reduced
gradients and the flag), the flags are OR-ed over the group, and only when
no rank overflowed does every rank run the update from its reduced
gradients in place.  That update stores the new parameters of its slot
straight into every rank's parameter buffer (peer stores through the same
mappings), so the all-gather needs no step of its own: one barrier after
the update and every rank holds every slot.

No kernel waits on another rank: all cross-rank ordering is host barriers,
so the ranks may also share one GPU (each with its own context).  This class
sequences library calls; all arithmetic runs in libzero's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (DevicePtr, hparams, zero_adam_step_reduced_bcast, zero_allgather_params, zero_ipc_close,
               zero_ipc_export, zero_ipc_import, zero_loss_scale_update, zero_partition_layout,
               zero_reduce_scatter_adam_step, zero_reduce_scatter_grads)


class DistributedZeroAdam:
    def __init__(self, numels, bucket_elems: int = 0, align_elems: int = 8, *, group=None, lr: float = 1e-3,
                 betas=(0.9, 0.999),
                 eps: float = 1e-8, weight_decay: float = 0.0, grad_dtype=torch.float16,
                 param_dtype=torch.float16, loss_scale: float = 65536.0, growth_interval: int = 1000,
                 min_scale: float = 1.0, mode: str = "banks", device="cuda"):
        if mode not in ("banks", "staged"):
            raise ValueError("mode must be 'banks' or 'staged'")
        self.mode = mode
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.device = torch.device(device)
        # align_elems = 8 pads every bucket to a multiple of 8N elements, so each
        # rank's partition starts on a 16-byte boundary of the peers' buffers
        # (the vector and pipeline paths); 1 pads to a multiple of N only
        self.layout = zero_partition_layout(list(numels), self.world, bucket_elems, align_elems)
        self.lr, self.betas, self.eps, self.weight_decay = lr, betas, eps, weight_decay
        self.scale, self.good_steps, self.t, self.cur = float(loss_scale), 0, 0, 0
        self.growth_interval, self.min_scale = growth_interval, min_scale
        self.grad_dtype, self.param_dtype = grad_dtype, param_dtype
        L, dev = self.layout, self.device
        f32 = dict(dtype=torch.float32, device=dev)
        self.grads = [torch.zeros(L.bucket_padded[b], dtype=grad_dtype, device=dev) for b in range(L.n_buckets)]
        self.params = [torch.zeros(L.bucket_padded[b], dtype=param_dtype, device=dev) for b in range(L.n_buckets)]
        nbank = 2 if mode == "banks" else 1
        self.master = [[torch.zeros(L.part(b), **f32) for _ in range(nbank)] for b in range(L.n_buckets)]
        self.m = [[torch.zeros(L.part(b), **f32) for _ in range(nbank)] for b in range(L.n_buckets)]
        self.v = [[torch.zeros(L.part(b), **f32) for _ in range(nbank)] for b in range(L.n_buckets)]
        if mode == "banks":
            # spare parameter slot: the update of a step that may still be skipped
            self.param_spare = [torch.zeros(L.part(b), dtype=param_dtype, device=dev) for b in range(L.n_buckets)]
        else:
            self.reduced = [torch.zeros(L.part(b), **f32) for b in range(L.n_buckets)]
        self.flags = torch.zeros(2, dtype=torch.int32, device=dev)    # [step flag, update status]
        self.flag = self.flags[0:1]
        self._map_peers()

    # ------------------------------------------------------------------ IPC
    def _map_peers(self) -> None:
        mine = [[zero_ipc_export(t) for t in self.grads], [zero_ipc_export(t) for t in self.params]]
        everyone = [None] * self.world
        dist.all_gather_object(everyone, mine, group=self.group)
        self._bases = []
        self.peer_grads, self.peer_params = [], []       # [bucket][rank]
        for b in range(self.layout.n_buckets):
            g_row, p_row = [], []
            for r in range(self.world):
                if r == self.rank:
                    g_row.append(self.grads[b])
                    p_row.append(self.params[b])
                    continue
                (gh, go), (ph, po) = everyone[r][0][b], everyone[r][1][b]
                gptr, gbase = zero_ipc_import(gh, go)
                pptr, pbase = zero_ipc_import(ph, po)
                self._bases += [gbase, pbase]
                g_row.append(DevicePtr(gptr, self.grad_dtype))
                p_row.append(DevicePtr(pptr, self.param_dtype))
            self.peer_grads.append(g_row)
            self.peer_params.append(p_row)

    def close(self) -> None:
        """Unmap the peers' buffers (call on every rank before exit)."""
        torch.cuda.synchronize()
        dist.barrier(group=self.group)
        for base in self._bases:
            zero_ipc_close(base)
        self._bases = []

    # ---------------------------------------------------------------- state
    def load(self, master_flat, params_flat) -> None:
        """master_flat[b]: this bucket's fp32 master (padded, flat order);
        params_flat[b]: its low-precision parameters.  m = v = 0."""
        for b in range(self.layout.n_buckets):
            P = self.layout.part(b)
            own = slice(self.rank * P, (self.rank + 1) * P)
            for bank in range(len(self.master[b])):
                self.master[b][bank].copy_(master_flat[b][own])
                self.m[b][bank].zero_()
                self.v[b][bank].zero_()
            self.params[b].copy_(params_flat[b])
        torch.cuda.synchronize()
        self.cur, self.t = 0, 0

    def partition_state(self, b: int):
        """Committed (master, m, v) of this rank's partition of bucket b."""
        c = self.cur
        return self.master[b][c], self.m[b][c], self.v[b][c]

    # ----------------------------------------------------------------- step
    def _or_over_ranks(self, flag: int) -> int:
        backend = dist.get_backend(self.group)
        t = torch.tensor([flag], dtype=torch.int32, device=self.device if backend == "nccl" else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=self.group)
        return int(t.item())

    def step(self) -> bool:
        L, r = self.layout, self.rank
        torch.cuda.synchronize()
        dist.barrier(group=self.group)                  # every rank's gradients are written
        self.flags.zero_()
        hp = hparams(self.lr, self.betas[0], self.betas[1], self.eps, self.weight_decay, self.t + 1)
        if self.mode == "staged":
            for b in range(L.n_buckets):
                zero_reduce_scatter_grads(self.peer_grads[b], L.bucket_padded[b], r, self.scale, self.reduced[b],
                                          self.flag)
        else:
            c, n = self.cur, self.cur ^ 1
            for b in range(L.n_buckets):
                zero_reduce_scatter_adam_step(
                    self.peer_grads[b], L.bucket_padded[b], r,
                    self.master[b][c], self.m[b][c], self.v[b][c],
                    self.master[b][n], self.m[b][n], self.v[b][n], self.param_spare[b],
                    hp, self.scale, self.flag)
        ovf = self._or_over_ranks(int(self.flag.item()))     # synchronizes this rank's stream
        if ovf & 2:
            raise RuntimeError("fused step kernel timed out waiting on its copy pipeline; step not committed")
        applied = ovf == 0
        if applied and self.mode == "staged":
            # every rank knows the verdict of the whole group: update in place
            # and store slot r of every rank's parameter buffer
            for b in range(L.n_buckets):
                P = L.part(b)
                st = (self.master[b][0], self.m[b][0], self.v[b][0])
                esz = self.params[b].element_size()
                dsts = [self.params[b][r * P:(r + 1) * P] if q == r else
                        DevicePtr(self.peer_params[b][q].data_ptr() + r * P * esz, self.param_dtype)
                        for q in range(self.world)]
                zero_adam_step_reduced_bcast(self.reduced[b], P, *st, *st, dsts, hp, self.flags[1:2])
            if int(self.flags[1].item()) & 2:
                raise RuntimeError("staged update timed out waiting on its copy pipeline; states incomplete")
            self.t += 1
        elif applied:
            for b in range(L.n_buckets):
                P = L.part(b)
                zero_allgather_params([self.param_spare[b]], 0, P, self.params[b][r * P:(r + 1) * P])
            self.cur ^= 1
            self.t += 1
        self.scale, self.good_steps = zero_loss_scale_update(self.scale, self.good_steps, not applied,
                                                             self.growth_interval, self.min_scale)
        if applied and self.mode == "staged":
            torch.cuda.synchronize()
            dist.barrier(group=self.group)              # every rank's slot is in every buffer
        elif applied:
            torch.cuda.synchronize()
            dist.barrier(group=self.group)              # every rank's own slot is updated
            for b in range(L.n_buckets):
                P = L.part(b)
                for q in range(self.world):
                    if q == r:
                        continue
                    src = DevicePtr(self.peer_params[b][q].data_ptr() + q * P * self.params[b].element_size(),
                                    self.param_dtype)
                    zero_allgather_params([src], 0, P, self.params[b][q * P:(q + 1) * P])
            torch.cuda.synchronize()
            dist.barrier(group=self.group)              # nobody still reads a peer's buffer
        return applied
