"""zero_reduce_scatter_adam_step_noalloc: the fused step for callers that
cannot allocate device memory.

Some callers have no way to hand the library the device workspace that the
gradient norm needs: code running under an allocator that owns all device
memory and forbids direct cudaMalloc, a host thread that must not take
cudaMalloc's implicit device synchronization, or a plain C program with no
device allocator.  This entry point keeps that scratch in a fixed array inside
libzero instead.  The GPU test calls it through the C ABI twice in a row (the
second call reuses the scratch the first one left behind) and checks every
output against the regular entry point (same tolerance as the other parity
tests, and in fact bit for bit, the norm included) and against the oracle.
The cases reach all four step kernels, each forced with
zero_test_force_step_kernel on both entry points: the register, quad and oct
kernels (the oct kernel is the automatic choice at this size) on a ragged
size, the shared-memory pipeline kernel on at least two tiles per SM; plus a
call on a single partition with the automatic choice.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
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


ADAM = workloads.AdamConfig(weight_decay=0.01)
SCALE = 65536.0


def _run(entry, grads, state_in, t, padded, partition, count, use_ws):
    out = [torch.empty_like(x) for x in state_in]
    params = torch.empty(count, dtype=torch.float16, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    norm = torch.zeros(1, dtype=torch.float64, device="cuda")
    hp = Z.hparams(ADAM.lr, ADAM.beta1, ADAM.beta2, ADAM.eps, ADAM.weight_decay, t)
    if use_ws:
        ws = torch.zeros(Z.zero_step_workspace_bytes(), dtype=torch.uint8, device="cuda")
        entry(grads, padded, partition, *state_in, *out, params, hp, SCALE, flag, norm, ws)
    else:
        entry(grads, padded, partition, *state_in, *out, params, hp, SCALE, flag, norm)
    torch.cuda.synchronize()
    return out, params, int(flag.item()), float(norm.item())


@pytest.fixture
def kernel_kind(request):
    Z.zero_test_force_step_kernel(request.param)
    try:
        yield request.param
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)


@pytest.mark.gpu
@pytest.mark.parametrize("world,padded,partition,kernel_kind", [
    (8, 8 * 100_003 + 8, Z.ZERO_ALL_PARTITIONS, Z.STEP_KERNEL_REGISTER),   # ragged vector tail
    (8, 8 * 100_003 + 8, Z.ZERO_ALL_PARTITIONS, Z.STEP_KERNEL_QUAD),
    (8, 8 * 100_003 + 8, Z.ZERO_ALL_PARTITIONS, Z.STEP_KERNEL_OCT),     # the automatic choice at this size
    (8, 8 * (2 * 148 * 3072 + 1000), Z.ZERO_ALL_PARTITIONS, Z.STEP_KERNEL_PIPE),  # >= 2 tiles of 3072 per SM
    (8, 8 * 100_003 + 8, 3, Z.STEP_KERNEL_AUTO),                             # one rank's partition
], indirect=["kernel_kind"])
def test_noalloc_matches_regular_entry_and_oracle_on_two_calls_in_a_row(world, padded, partition, kernel_kind):
    P = padded // world
    begin = 0 if partition < 0 else partition * P
    count = padded if partition < 0 else P
    G = [workloads.grads(padded, 4242 + k, 1e-3, SCALE) for k in range(world)]
    master0 = workloads.master(count, 4342)
    dev = lambda a: torch.from_numpy(a).cuda()
    grads = [dev(g.view(np.int16)).view(torch.float16) for g in G]
    ref = oracle.initial_state(master0)
    start = [dev(master0.copy()), torch.zeros(count, device="cuda"), torch.zeros(count, device="cuda")]
    reg_state, got_state = start, start
    for t in (1, 2):
        reg = _run(Z.zero_reduce_scatter_adam_step, grads, reg_state, t, padded, partition, count, use_ws=True)
        got = _run(Z.zero_reduce_scatter_adam_step_noalloc, grads, got_state, t, padded, partition, count,
                   use_ws=False)
        ovf, sq = oracle.flat_step(G, ref, ADAM, t, SCALE, float(world), begin=begin, count=count)
        assert got[2] == reg[2] == ovf == 0
        for a, b, exp, name in zip(got[0], reg[0], (ref.master, ref.m, ref.v), ("master", "m", "v")):
            ga = host_f32(a)
            # against the regular entry point: the parity tolerance, and bit for bit
            assert assert_f32_close(ga, host_f32(b), f"{name} vs regular entry (call {t})") == 0
            assert assert_f32_close(ga, exp, f"{name} vs oracle (call {t})") == 0
        assert assert_u16_close(host_u16(got[1]), host_u16(reg[1]), f"params vs regular entry (call {t})") == 0
        assert assert_u16_close(host_u16(got[1]), ref.params, f"params vs oracle (call {t})") == 0
        # the same kernel on the same grid folds the same partial sums in the
        # same order: the norms agree bit for bit; against the oracle's
        # sequential fp64 sum of the same exact squares, within the bound of
        # two fp64 summation orders
        assert got[3] == reg[3] and sq > 0
        assert abs(got[3] - sq) <= 2.0 * count * 2.0 ** -53 * sq
        reg_state, got_state = reg[0], got[0]
