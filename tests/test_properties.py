"""Property-based tests (hypothesis, derandomized): random layouts through
the C ABI against the oracle on the CPU, and random small configurations of
the fused step and of the staged step (reduce-scatter to fp32, then the
update from it) on the GPU against the oracle, bit for bit."""
import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
import workloads
import zero_sharded_optimizer_reduce_b200 as Z


@settings(max_examples=300, deadline=None, derandomize=True)
@given(numels=st.lists(st.integers(0, 10_000), max_size=40), world=st.integers(1, 128),
       cap=st.integers(0, 50_000), align=st.integers(1, 16))
def test_layout_matches_oracle(numels, world, cap, align):
    a = Z.zero_partition_layout(numels, world, cap, align)
    b = oracle.partition_layout(numels, world, cap, align)
    assert list(a.bucket_numel) == b.bucket_numel and list(a.bucket_padded) == b.bucket_padded
    assert list(a.bucket_offset) == b.bucket_offset
    assert list(a.tensor_bucket) == b.tensor_bucket and list(a.tensor_offset) == b.tensor_offset


KINDS = [-1, 0, 1, 2, 3]   # automatic, register, pipeline, quad, oct (zero_test_force_step_kernel)


@pytest.mark.gpu
@settings(max_examples=80, deadline=None, derandomize=True)
@given(world=st.integers(1, 17), per_rank=st.integers(1, 5000),
       dtypes=st.sampled_from([(oracle.F16, oracle.F16), (oracle.BF16, oracle.BF16), (oracle.F16, oracle.BF16),
                               (oracle.BF16, oracle.F16)]),
       offs=st.tuples(st.integers(0, 7), st.integers(0, 7), st.integers(0, 7)),
       part=st.integers(-1, 16), inplace=st.booleans(), wd=st.sampled_from([0.0, 0.01, 0.1]),
       t=st.integers(1, 50), seed=st.integers(0, 10_000), kind=st.sampled_from(KINDS))
def test_step_matches_oracle(world, per_rank, dtypes, offs, part, inplace, wd, t, seed, kind):
    """Random sizes, offsets (state offsets of 0-7 fp32 elements put the
    outputs on and off a 32-byte boundary), partitions, dtypes and a forced
    kernel (it runs where it can, else the automatic choice)."""
    import zero_sharded_optimizer_reduce_b200 as Z
    from test_gpu_step import Case
    gd, pd = dtypes
    partition = part if part < world else -1
    c = Case(world * per_rank, world, gdtype=gd, pdtype=pd, seed=seed, partition=partition, goff=offs[0],
             soff=offs[1], poff=offs[2], inplace=inplace)
    adam = workloads.AdamConfig(weight_decay=wd)
    ref, ovf, _ = c.expect(adam, t=t)
    Z.zero_test_force_step_kernel(kind)
    try:
        c.run(adam, t=t)
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)
    assert int(c.flag.item()) == ovf == 0
    assert c.compare(ref) == [0, 0, 0, 0]


@pytest.mark.gpu
@settings(max_examples=30, deadline=None, derandomize=True)
@given(world=st.integers(1, 17), per_rank=st.integers(1, 5000),
       dtypes=st.sampled_from([(oracle.F16, oracle.F16), (oracle.BF16, oracle.BF16), (oracle.F16, oracle.BF16)]),
       offs=st.tuples(st.integers(0, 7), st.integers(0, 7), st.integers(0, 7), st.integers(0, 7)),
       part=st.integers(-1, 16), inplace=st.booleans(), wd=st.sampled_from([0.0, 0.01]),
       t=st.integers(1, 50), seed=st.integers(0, 10_000), kind=st.sampled_from(KINDS))
def test_staged_step_matches_oracle(world, per_rank, dtypes, offs, part, inplace, wd, t, seed, kind):
    import zero_sharded_optimizer_reduce_b200 as Z
    from test_gpu_staged import Staged
    gd, pd = dtypes
    partition = part if part < world else -1
    c = Staged(world * per_rank, world, gdtype=gd, pdtype=pd, seed=seed, partition=partition, goff=offs[0],
               soff=offs[1], poff=offs[2], roff=offs[3], inplace=inplace, scale=1024.0)
    adam = workloads.AdamConfig(weight_decay=wd)
    ref, ovf, _ = c.expect(adam, t=t)
    Z.zero_test_force_step_kernel(kind)
    try:
        c.reduce_scatter()
        s, inv, g = c.oracle_reduced()
        assert np.array_equal(host_reduced(c), g.view(np.uint32))
        c.update(adam, t=t, gate=c.flag)
    finally:
        Z.zero_test_force_step_kernel(Z.STEP_KERNEL_AUTO)
    assert int(c.flag.item()) == ovf == 0
    assert c.compare(ref) == [0, 0, 0, 0]


def host_reduced(c):
    from _gpu import host_f32
    return host_f32(c.red.t).view(np.uint32)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(numels=st.lists(st.integers(1, 3000), min_size=1, max_size=6), world=st.integers(1, 6),
       cap=st.sampled_from([0, 1000, 4000]), dtype=st.sampled_from([oracle.F16, oracle.BF16]),
       inject=st.booleans(), seed=st.integers(0, 1000))
def test_oracle_stages_equal_plain_dp_on_random_layouts(numels, world, cap, dtype, inject, seed):
    """The pages' drop-in claim on random layouts: plain DP, Stage 1, 2 and 3
    of the oracle give bit-identical states after every step, with an
    inf injected into one replica at step 2 (when `inject`), skipped by all."""
    from test_oracle_stages import _assert_equal_states, _grads, _runs
    adam = workloads.AdamConfig(weight_decay=0.01)
    L, runs = _runs(numels, world, cap, adam, 1024.0, dtype, dtype, seed)
    for step in (1, 2, 3):
        G = _grads(L, step, seed, runs[0].scaler.scale, dtype, numels)
        if inject and step == 2:
            inf = workloads.F16_POS_INF if dtype == oracle.F16 else workloads.BF16_POS_INF
            G[0][world - 1][0] = inf
        flags = {s: r.step(G) for s, r in runs.items()}
        assert set(flags.values()) == {int(inject and step == 2)}
        for s in (1, 2, 3):
            for b in range(L.n_buckets):
                _assert_equal_states(runs[0].flat_state(b), runs[s].flat_state(b))
        assert all(r.replicas_identical() for r in runs.values())
