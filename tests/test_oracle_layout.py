"""Pins of the oracle's partition layout and fused constant-size buffers.

Invariants checked by brute force on small cases: every real element lies in
exactly one partition, all partitions of a bucket have the same length, the
padding is below N*align per bucket and zero, concatenating the partitions in
rank order gives the bucket back, and the greedy packing never exceeds the
capacity unless a single tensor does.
"""
import itertools

import numpy as np
import pytest

import oracle
import workloads


def _check_layout(numels, world, cap, align):
    L = oracle.partition_layout(numels, world, cap, align)
    # every tensor in exactly one bucket, in list order, contiguous offsets
    seen = []
    for b, idx in enumerate(L.bucket_tensors):
        off = 0
        for i in idx:
            assert L.tensor_bucket[i] == b and L.tensor_offset[i] == off
            off += numels[i]
            seen.append(i)
        assert L.bucket_numel[b] == off
        # capacity respected unless a single tensor is larger than it
        if cap > 0 and len(idx) > 1:
            assert off <= cap
        # greedy: the next bucket's first tensor did not fit here
        if cap > 0 and b + 1 < L.n_buckets:
            first_next = L.bucket_tensors[b + 1][0]
            assert off + numels[first_next] > cap
        pad = L.bucket_padded[b]
        assert pad % (world * align) == 0 and 0 <= pad - off < world * align
    assert seen == list(range(len(numels)))
    # flat offsets are prefix sums of padded sizes
    assert L.bucket_offset == list(np.cumsum([0] + L.bucket_padded[:-1]).tolist()) or L.n_buckets == 0
    # element ownership: every real element belongs to exactly one (rank, j)
    for b in range(L.n_buckets):
        P = L.part(b)
        owner = np.full(L.bucket_padded[b], -1)
        for r in range(world):
            assert (owner[r * P:(r + 1) * P] == -1).all()
            owner[r * P:(r + 1) * P] = r
        assert (owner >= 0).all()
    return L


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7, 8])
@pytest.mark.parametrize("cap", [0, 5, 16, 40])
@pytest.mark.parametrize("align", [1, 8])
def test_layout_invariants_small(world, cap, align):
    rng = np.random.Generator(np.random.PCG64(world * 100 + cap + align))
    for _ in range(5):
        numels = rng.integers(0, 30, rng.integers(0, 12)).tolist()
        _check_layout(numels, world, cap, align)


def test_flatten_partition_roundtrip_bit_exact():
    rng = np.random.Generator(np.random.PCG64(5))
    numels = [7, 1, 13, 0, 29, 3]
    tensors = [rng.integers(0, 65536, n).astype(np.uint16) for n in numels]
    for world, cap in itertools.product([1, 3, 4], [0, 20]):
        L = oracle.partition_layout(numels, world, cap)
        for b in range(L.n_buckets):
            buf = oracle.flatten_bucket(L, b, tensors)
            parts = oracle.partitions(buf, world)
            again = oracle.allgather(parts, 0, L.part(b))
            assert np.array_equal(again, buf)
            assert (buf[L.bucket_numel[b]:] == 0).all()
            for i in L.bucket_tensors[b]:
                o = L.tensor_offset[i]
                assert np.array_equal(buf[o:o + numels[i]], tensors[i])


def test_odd_flat_model_padding():
    L = oracle.partition_layout([1_000_003], 4)
    assert L.bucket_padded == [1_000_004] and L.part(0) == 250_001


def test_gpt2_tensor_list_and_buckets():
    numels = workloads.gpt2_1p5b_tensor_numels()
    assert len(numels) == 580 and sum(numels) == 1_557_611_200
    L = oracle.partition_layout(numels, 8, 500_000_000)
    assert L.bucket_numel == [491_932_800, 491_852_800, 491_852_800, 81_972_800]
    assert L.bucket_padded == L.bucket_numel          # all multiples of 8 already
    _check_layout(numels, 8, 500_000_000, 1)


def test_gpt_6p7b_units():
    units = workloads.gpt_6p7b_unit_numels()
    assert len(units) == 33 and units[0] == 201_379_840 and units[-1] == 205_860_864
    assert sum(units) == 6_650_015_744
    L = oracle.partition_layout(units, 8, 1)      # capacity 1: one unit per bucket
    assert L.n_buckets == 33 and L.part(0) == 25_172_480 and L.part(32) == 25_732_608


def test_layout_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.partition_layout([3], 0)
    with pytest.raises(ValueError):
        oracle.partition_layout([3], 2, -1)
    with pytest.raises(ValueError):
        oracle.partition_layout([-1], 2)


def test_allgather_with_offset_brute_force():
    rng = np.random.Generator(np.random.PCG64(8))
    shards = [rng.integers(0, 65536, 50).astype(np.uint16) for _ in range(3)]
    for off, part in [(0, 50), (7, 11), (49, 1), (13, 0)]:
        got = oracle.allgather(shards, off, part)
        ref = np.concatenate([sh[off:off + part] for sh in shards])
        assert np.array_equal(got, ref)


def test_bucket_filled_exactly_to_capacity():
    """A constant-size buffer of capacity C takes tensors while their total
    stays within C [ZeRO explainer, "Constant-size buffers"]: a bucket may end
    exactly at C, and the next tensor opens a new one."""
    L = oracle.partition_layout([3, 2, 5, 1, 4], 1, 5)
    assert L.bucket_numel == [5, 5, 5]
    assert L.bucket_tensors == [[0, 1], [2], [3, 4]]
    L = oracle.partition_layout([3, 3], 1, 5)
    assert L.bucket_numel == [3, 3]
