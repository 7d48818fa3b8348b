"""zero_reduce_scatter_adam_step_noalloc: the fused step for callers that
cannot allocate device memory.

Such callers (code under an allocator that owns all device memory and forbids
direct cudaMalloc, a host thread that must not take cudaMalloc's implicit
synchronization, a C caller without a device allocator) cannot hand the
library the workspace that the gradient norm needs.  This entry point keeps
that scratch in a fixed array inside libzero instead.  The GPU test calls it
through the C ABI twice in a row (the second call reuses the scratch the first
one left behind) and checks every output against the regular entry point.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import zero_sharded_optimizer_reduce_b200 as Z
from _gpu import assert_f32_close, assert_u16_close, host_f32, host_u16


def test_noalloc_entry_validates_like_the_regular_one():
    # fake pointers: validation fails before any CUDA call
    g = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    hp = Z.hparams()
    args = [g, 2, 64, -1, 0, 0x7100_0000, 0x7200_0000, 0x7300_0000, 0x7400_0000, 0x7500_0000, 0x7600_0000,
            0x7700_0000, 0, ctypes.byref(hp), 1024.0, 0x7900_0000, None, None]
    bad = list(args)
    bad[0] = None
    assert Z.lib.zero_reduce_scatter_adam_step_noalloc(*bad) == -1
    bad = list(args)
    bad[3] = 5
    assert Z.lib.zero_reduce_scatter_adam_step_noalloc(*bad) == -4
    bad = list(args)
    bad[4] = 9
    assert Z.lib.zero_reduce_scatter_adam_step_noalloc(*bad) == -3
    bad = list(args)
    bad[5] = 0x7100_0002
    assert Z.lib.zero_reduce_scatter_adam_step_noalloc(*bad) == -2
    ok = list(args)
    ok[2] = 0
    assert Z.lib.zero_reduce_scatter_adam_step_noalloc(*ok) == 0    # nothing to do
    assert Z.lib.zero_step_static_scratch_bytes() == 256 + 8 * 4096


def _inputs(world, n, seed):
    dev = lambda a: torch.from_numpy(a).cuda()
    grads = [dev(workloads.grads(n, seed + k, 1e-3, 65536.0).view(np.int16)).view(torch.float16)
             for k in range(world)]
    master = dev(workloads.master(n, seed + 100))
    m = torch.zeros_like(master)
    v = torch.zeros_like(master)
    return grads, [master, m, v]


def _run(entry, grads, state_in, t, world, n, use_ws):
    out = [torch.empty_like(x) for x in state_in]
    params = torch.empty(n, dtype=torch.float16, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    norm = torch.zeros(1, dtype=torch.float64, device="cuda")
    hp = Z.hparams(1e-3, 0.9, 0.999, 1e-8, 0.01, t)
    if use_ws:
        ws = torch.zeros(Z.zero_step_workspace_bytes(), dtype=torch.uint8, device="cuda")
        entry(grads, n, Z.ZERO_ALL_PARTITIONS, *state_in, *out, params, hp, 65536.0, flag, norm, ws)
    else:
        entry(grads, n, Z.ZERO_ALL_PARTITIONS, *state_in, *out, params, hp, 65536.0, flag, norm)
    torch.cuda.synchronize()
    return out, params, int(flag.item()), float(norm.item())


@pytest.mark.gpu
def test_noalloc_matches_regular_entry_on_two_calls_in_a_row():
    world, n = 8, 8 * 100_003 + 8          # several blocks and a ragged per-rank size
    grads, state = _inputs(world, n, 4242)
    ref_state, got_state = state, state
    for t in (1, 2):
        ref = _run(Z.zero_reduce_scatter_adam_step, grads, ref_state, t, world, n, use_ws=True)
        got = _run(Z.zero_reduce_scatter_adam_step_noalloc, grads, got_state, t, world, n, use_ws=False)
        for a, b, name in zip(got[0], ref[0], ("master", "m", "v")):
            assert_f32_close(host_f32(a), host_f32(b), f"{name} (call {t})")
        assert_u16_close(host_u16(got[1]), host_u16(ref[1]), f"params (call {t})")
        assert got[2] == ref[2] == 0
        assert abs(got[3] - ref[3]) <= 1e-5 * ref[3] and ref[3] > 0
        ref_state, got_state = ref[0], got[0]
