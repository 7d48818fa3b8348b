"""ZeroAdam: a ZeRO-2 partitioned mixed-precision Adam step on one GPU.

N data-parallel replicas are simulated by N resident gradient buffers per
bucket.  Two ways to run a step, both with an exact skip on overflow:

  mode="banks" (default): the fused reduce-scatter + Adam kernel runs once
    over every bucket, reading bank `cur` of the fp32 master / momentum /
    variance states and low-precision parameters and writing bank `cur ^ 1`;
    the bank flips only when no reduced gradient of the whole step was inf or
    NaN.  One pass over HBM (2N + 26 bytes per element); the second bank
    doubles the 12 Psi/N bytes of optimizer state that ZeRO keeps per rank
    (ZeRO explainer, "Stage 1 - Optimizer State Partitioning").
  mode="inplace": a statistics pass over every bucket (rank-order sums,
    overflow flag, squared norm) and then the update in place, gated on the
    device by that flag: one bank, the pages' 12 Psi/N, for 4N + 26 bytes per
    element.
  mode="staged": the reduce-scatter stores every bucket's reduced fp32
    gradients (with the flag and norm), then the in-place update reads them,
    gated by that flag: one bank plus 4 bytes per element of reduced
    gradients, for 2N + 34 bytes per element (ZeRO explainer, "Stage 2 -
    Gradient Partitioning": each rank keeps the reduced gradients of its own
    partition).

max_grad_norm (any mode) clips the unscaled gradients to that global
norm, with the coefficient computed on the device from the statistics pass
(banks mode then also takes the two-pass route).

The loss scale follows zero_loss_scale_update (halve on overflow, double
after `growth_interval` good steps) and the Adam step count t advances only
on applied updates.  This class only allocates buffers and sequences library
calls; all arithmetic is in libzero's kernels.
"""
from __future__ import annotations

import torch

from . import (ZERO_ALL_PARTITIONS, Runner, hparams, zero_adam_step_reduced, zero_flatten_bucket, zero_grad_stats,
               zero_loss_scale_update, zero_partition_layout, zero_reduce_scatter_adam_step,
               zero_reduce_scatter_adam_step_gated, zero_reduce_scatter_grads, zero_step_workspace_bytes)


class ZeroAdam:
    def __init__(self, numels, world: int, bucket_elems: int = 0, align_elems: int = 1, *,
                 lr: float = 1e-3, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
                 grad_dtype=torch.float16, param_dtype=torch.float16, loss_scale: float = 65536.0,
                 growth_interval: int = 1000, min_scale: float = 1.0, grad_divisor: float = 0.0,
                 track_grad_norm: bool = False, mode: str = "banks", max_grad_norm: float | None = None,
                 device="cuda"):
        if mode not in ("banks", "inplace", "staged"):
            raise ValueError("mode must be 'banks', 'inplace' or 'staged'")
        if max_grad_norm is not None and not max_grad_norm > 0:
            raise ValueError("max_grad_norm must be positive")
        self.mode, self.max_grad_norm = mode, max_grad_norm
        self.two_pass = mode != "banks" or max_grad_norm is not None
        self.layout = zero_partition_layout(list(numels), world, bucket_elems, align_elems)
        self.world = world
        self.device = torch.device(device)
        self.lr, self.betas, self.eps, self.weight_decay = lr, betas, eps, weight_decay
        self.grad_divisor = grad_divisor
        self.scale, self.good_steps = float(loss_scale), 0
        self.growth_interval, self.min_scale = growth_interval, min_scale
        self.t = 0
        self.cur = 0
        L, dev = self.layout, self.device
        f32 = dict(dtype=torch.float32, device=dev)
        nbank = 2 if mode == "banks" else 1
        self.master = [[torch.zeros(L.bucket_padded[b], **f32) for _ in range(nbank)] for b in range(L.n_buckets)]
        self.m = [[torch.zeros(L.bucket_padded[b], **f32) for _ in range(nbank)] for b in range(L.n_buckets)]
        self.v = [[torch.zeros(L.bucket_padded[b], **f32) for _ in range(nbank)] for b in range(L.n_buckets)]
        self.params_bank = [[torch.zeros(L.bucket_padded[b], dtype=param_dtype, device=dev) for _ in range(nbank)]
                            for b in range(L.n_buckets)]
        self.grads = [[torch.zeros(L.bucket_padded[b], dtype=grad_dtype, device=dev) for _ in range(world)]
                      for b in range(L.n_buckets)]
        # staged mode: every rank's reduced fp32 gradient partition, per bucket
        self.reduced = ([torch.zeros(L.bucket_padded[b], **f32) for b in range(L.n_buckets)]
                        if mode == "staged" else None)
        # flags[0]: the step's overflow flag (read by the host, the gate of
        # the two-pass update); flags[1]: the gated update's own flag
        self.flags = torch.zeros(2, dtype=torch.int32, device=dev)
        self.flag = self.flags[0:1]
        self.flag_host = torch.zeros(2, dtype=torch.int32, pin_memory=True)
        self.track_grad_norm = track_grad_norm
        need_norm = track_grad_norm or max_grad_norm is not None
        self.sqnorm = torch.zeros(1, dtype=torch.float64, device=dev) if need_norm else None
        self.workspace = (torch.zeros(zero_step_workspace_bytes(), dtype=torch.uint8, device=dev)
                          if need_norm else None)
        self.last_overflow = 0
        # the single-pass banks mode runs through the native step runner:
        # one C call enqueues the whole step, one commits it
        self._runner = None
        hp1 = hparams(lr, betas[0], betas[1], eps, weight_decay, 1, grad_divisor)
        buckets = [(self.grads[b], self.master[b], self.m[b], self.v[b], self.params_bank[b])
                   for b in range(L.n_buckets)]
        if not self.two_pass and L.n_buckets > 0:
            self._flag_pinned = torch.zeros(1, dtype=torch.int32, pin_memory=True)
            self._runner = Runner(buckets, hp1, self.scale, self.flag, self._flag_pinned, self.sqnorm, self.workspace,
                                  growth_interval, min_scale)
        elif mode == "staged" and L.n_buckets > 0:
            # the staged route is native too: both passes over every bucket in one C call
            self._flag_pinned = torch.zeros(2, dtype=torch.int32, pin_memory=True)
            self._runner = Runner(buckets, hp1, self.scale, self.flags, self._flag_pinned, self.sqnorm,
                                  self.workspace, growth_interval, min_scale, reduced=self.reduced,
                                  max_norm=max_grad_norm or 0.0)

    def _sync_runner(self) -> None:
        """Hand the Python-side step state to the runner."""
        if self._runner is not None:
            self._runner.set_state(self.t, self.scale, self.good_steps, self.cur)

    # ------------------------------------------------------------ state access
    def load(self, params, master=None, stream=None) -> None:
        """Fill both banks from per-tensor parameters (and fp32 masters).

        `params`: list of low-precision tensors (one per tensor of the layout);
        `master`: list of fp32 tensors, default the parameters widened to fp32.
        m and v start at zero; t restarts at 0.
        """
        if master is None:
            master = [p.float() for p in params]
        for b in range(self.layout.n_buckets):
            zero_flatten_bucket(self.layout, b, master, self.master[b][0], stream)
            zero_flatten_bucket(self.layout, b, params, self.params_bank[b][0], stream)
            for bank in (self.master, self.params_bank):
                for extra in bank[b][1:]:
                    extra.copy_(bank[b][0])
            for bank in (self.m, self.v):
                for t in bank[b]:
                    t.zero_()
        self.cur = 0
        self.t = 0
        self._sync_runner()

    def state(self, b: int):
        """Committed (master, m, v, params) of bucket b."""
        c = self.cur
        return self.master[b][c], self.m[b][c], self.v[b][c], self.params_bank[b][c]

    def bucket_kernels(self):
        """The fused-step kernel each bucket's next step runs (STEP_KERNEL_REGISTER,
        _PIPE or _QUAD, per zero_runner_bucket_kernel); None in the two-pass
        modes, which run the statistics and update kernels instead."""
        if self._runner is None or self.two_pass:
            return None
        return [self._runner.bucket_kernel(b) for b in range(self.layout.n_buckets)]

    def grad_buffers(self, b: int):
        """The N replicas' gradient buffers of bucket b (write gradients here)."""
        return self.grads[b]

    # -------------------------------------------------------------------- step
    def launch(self, stream=None, on_launch=None, before_bucket=None) -> None:
        """Enqueue the fused kernel over every bucket (no host synchronization).

        `on_launch(bucket, phase)` is called with phase "before" / "after"
        around each kernel launch (used to record timing events);
        `before_bucket(bucket)` runs before bucket b's first kernel is
        enqueued (used to make the stream wait for that bucket's inputs).
        """
        if stream is not None:
            with torch.cuda.stream(stream):
                return self.launch(None, on_launch, before_bucket)
        self.flags.zero_()
        if self.sqnorm is not None:
            self.sqnorm.zero_()
        hp = hparams(self.lr, self.betas[0], self.betas[1], self.eps, self.weight_decay,
                     self.t + 1, self.grad_divisor)
        if self.two_pass:
            return self._launch_two_pass(hp, on_launch, before_bucket)
        c, n = self.cur, self.cur ^ 1
        for b in range(self.layout.n_buckets):
            if before_bucket is not None:
                before_bucket(b)
            if on_launch is not None:
                on_launch(b, "before")
            zero_reduce_scatter_adam_step(
                self.grads[b], self.layout.bucket_padded[b], ZERO_ALL_PARTITIONS,
                self.master[b][c], self.m[b][c], self.v[b][c],
                self.master[b][n], self.m[b][n], self.v[b][n], self.params_bank[b][n],
                hp, self.scale, self.flag, self.sqnorm, self.workspace)
            if on_launch is not None:
                on_launch(b, "after")

    def _launch_two_pass(self, hp, on_launch, before_bucket=None) -> None:
        """Statistics (or the staged reduce-scatter) over every bucket, then
        the gated (and clipped) update."""
        L = self.layout
        for b in range(L.n_buckets):
            if before_bucket is not None:
                before_bucket(b)
            if self.mode == "staged":
                zero_reduce_scatter_grads(self.grads[b], L.bucket_padded[b], ZERO_ALL_PARTITIONS, self.scale,
                                          self.reduced[b], self.flag, self.sqnorm, self.workspace,
                                          self.grad_divisor)
            else:
                zero_grad_stats(self.grads[b], L.bucket_padded[b], ZERO_ALL_PARTITIONS, self.scale, self.flag,
                                self.sqnorm, self.workspace, self.grad_divisor)
        c = self.cur
        n = c ^ 1 if self.mode == "banks" else c
        clip = self.sqnorm if self.max_grad_norm is not None else None
        for b in range(L.n_buckets):
            if on_launch is not None:
                on_launch(b, "before")
            if self.mode == "staged":
                zero_adam_step_reduced(
                    self.reduced[b], L.bucket_padded[b], self.master[b][c], self.m[b][c], self.v[b][c],
                    self.master[b][n], self.m[b][n], self.v[b][n], self.params_bank[b][n],
                    hp, self.flags[1:2], gate=self.flag, clip_sqnorm=clip, max_norm=self.max_grad_norm or 0.0)
                if on_launch is not None:
                    on_launch(b, "after")
                continue
            zero_reduce_scatter_adam_step_gated(
                self.grads[b], L.bucket_padded[b], ZERO_ALL_PARTITIONS,
                self.master[b][c], self.m[b][c], self.v[b][c],
                self.master[b][n], self.m[b][n], self.v[b][n], self.params_bank[b][n],
                hp, self.scale, self.flags[1:2], None, None, gate=self.flag, clip_sqnorm=clip,
                max_norm=self.max_grad_norm or 0.0)
            if on_launch is not None:
                on_launch(b, "after")

    def commit(self, stream=None) -> bool:
        """Read the overflow flag (device -> host), flip banks or skip, update the scale."""
        s = torch.cuda.current_stream() if stream is None else stream
        self.flag_host.copy_(self.flags, non_blocking=True)
        s.synchronize()
        flag, step_flag = int(self.flag_host[0]), int(self.flag_host[1])
        ovf = int(flag != 0)
        if (flag | step_flag) & 2:
            # the kernel abandoned its copy pipeline: the banks were not
            # committed, but the device needs attention
            raise RuntimeError("fused step kernel timed out waiting on its copy pipeline; step not committed")
        if not ovf:
            if self.mode == "banks":
                self.cur ^= 1
            self.t += 1
        self.scale, self.good_steps = zero_loss_scale_update(self.scale, self.good_steps, bool(ovf),
                                                             self.growth_interval, self.min_scale)
        self.last_overflow = ovf
        self._sync_runner()
        return not ovf

    def step(self, stream=None, on_launch=None) -> bool:
        """One whole step over all buckets; returns True if the update was applied.

        In the single-pass banks mode and in the staged mode the native
        runner enqueues and commits the step; `on_launch(-1, phase)` then
        brackets the whole step's device work (flag clear, every bucket's
        kernels, the flag read-back).  Otherwise `on_launch(b, phase)`
        brackets each bucket's update kernel."""
        if self._runner is None:
            self.launch(stream, on_launch)
            return self.commit(stream)
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
            if on_launch is not None:
                on_launch(-1, "before")
            self._runner.launch()
            if on_launch is not None:
                on_launch(-1, "after")
            try:
                applied = self._runner.commit()
            finally:
                self.t, self.scale, self.good_steps, self.cur = self._runner.state()
        self.last_overflow = int(not applied)
        return applied

    def step_from_host(self, host_grads, stream=None) -> bool:
        """Copy host gradients (host_grads[b][k], pinned) in, then step.

        The copies run bucket by bucket on a separate copy stream; bucket b's
        kernel waits only for bucket b's copies, so it overlaps the copies of
        the buckets after it."""
        main = stream if stream is not None else torch.cuda.current_stream()
        if not hasattr(self, "_copy_stream"):
            self._copy_stream = torch.cuda.Stream(device=self.device)
        cs = self._copy_stream
        cs.wait_stream(main)           # the previous step's kernels are done reading the buffers
        ready = []
        with torch.cuda.stream(cs):
            for b in range(self.layout.n_buckets):
                for k in range(self.world):
                    self.grads[b][k].copy_(host_grads[b][k], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(cs)
                ready.append(ev)
        with torch.cuda.stream(main):
            self.launch(before_bucket=lambda b: main.wait_event(ready[b]))
            return self.commit()

    # -------------------------------------------------------------- checkpoint
    def state_dict(self) -> dict:
        """Host copy of everything a resumed run needs: the committed master,
        m, v and parameters of every bucket, t, the loss scale and the
        good-step count, plus the layout they belong to."""
        L = self.layout
        return {
            "world": self.world, "bucket_padded": list(L.bucket_padded), "mode": self.mode,
            "t": self.t, "scale": self.scale, "good_steps": self.good_steps,
            "buckets": [{name: x.detach().cpu().clone() for name, x in zip(("master", "m", "v", "params"),
                                                                            self.state(b))}
                        for b in range(L.n_buckets)],
        }

    def load_state_dict(self, sd: dict) -> None:
        """Restore a state_dict taken from an optimizer with the same layout."""
        L = self.layout
        if sd["world"] != self.world or list(sd["bucket_padded"]) != list(L.bucket_padded):
            raise ValueError("checkpoint layout does not match this optimizer")
        for b, bucket in enumerate(sd["buckets"]):
            for bank_list, name in ((self.master, "master"), (self.m, "m"), (self.v, "v"),
                                    (self.params_bank, "params")):
                for t in bank_list[b]:
                    t.copy_(bucket[name].view(t.dtype) if bucket[name].dtype != t.dtype else bucket[name])
        self.cur = 0
        self.t, self.scale, self.good_steps = int(sd["t"]), float(sd["scale"]), int(sd["good_steps"])
        self._sync_runner()

    def grad_sqnorm(self) -> float:
        """Sum of squared unscaled gradients of the last step (if tracked)."""
        return float(self.sqnorm.item()) if self.sqnorm is not None else float("nan")
