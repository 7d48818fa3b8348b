"""All-gather reconstruct (zero_allgather_params) against the oracle's gather.

The copy kernel writes whole 32-byte aligned destination blocks; each is two
aligned 16-byte source blocks when source and destination share their 16-byte
phase, or three realigned ones when they do not, and the edges before the
first and after the last whole block are copied element by element.  These
cases pin every route bit for bit (ZeRO explainer, "Stage 3 - Parameter
Partitioning (P_os+g+p)": the gathered layer is exactly the concatenation of
the ranks' slices):

- every source element phase below 16 bytes against every destination phase
  below 32 bytes, at sizes below, at and above one block, so that each
  realignment shift, head and tail occurs;
- slices large enough that every block of the grid takes several iterations
  and the iterations end at slice boundaries;
- a Stage-1/2 gather of an odd partition size (every rank but the first off
  the destination's phase), scaled past L2;
- guard bytes around the destination and a status word that stays 0.
"""
import numpy as np
import pytest
import torch

import oracle
from _gpu import Guarded

pytestmark = pytest.mark.gpu

NPDT = {2: np.uint16, 4: np.uint32}
TDT_INT = {2: torch.int16, 4: torch.int32}


def _shards(world, shard_len, dtype, seed, elem_offset=0):
    """`world` device slices of shard_len elements, each starting elem_offset
    elements into its own allocation; returns (device views, host copies)."""
    es = torch.empty((), dtype=dtype).element_size()
    rng = np.random.Generator(np.random.PCG64(seed))
    host, dev, keep = [], [], []
    for _ in range(world):
        h = rng.integers(0, 2 ** (8 * es), shard_len, dtype=np.uint64).astype(NPDT[es])
        base = torch.empty(shard_len + elem_offset + 8, dtype=dtype, device="cuda")
        view = base[elem_offset:elem_offset + shard_len]
        view.view(TDT_INT[es]).copy_(torch.from_numpy(h.view(np.int16 if es == 2 else np.int32)))
        host.append(h)
        dev.append(view)
        keep.append(base)
    return dev, host, keep


def _expect(host, offset, part, es):
    if es == 2:
        return oracle.allgather(host, offset, part)
    halves = [h.view(np.uint16) for h in host]       # the oracle gathers 16-bit words
    return oracle.allgather(halves, 2 * offset, 2 * part).view(np.uint32)


def _gather_and_check(dev, host, offset, part, dtype, dst_elem_offset=0):
    import zero_sharded_optimizer_reduce_b200 as Z
    es = torch.empty((), dtype=dtype).element_size()
    world = len(dev)
    dst = Guarded(world * part, dtype, dst_elem_offset)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Z.zero_allgather_params(dev, offset, part, dst.t, status=status)
    torch.cuda.synchronize()
    dst.check()
    assert int(status.item()) == 0
    got = dst.t.view(TDT_INT[es]).cpu().numpy().view(NPDT[es])
    assert np.array_equal(got, _expect(host, offset, part, es))


@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
@pytest.mark.parametrize("part", [1, 7, 8, 9, 130, 3001])
def test_every_phase_pair(dtype, part):
    """Source slice at element offset a (below 16 bytes), destination at
    element offset b (below 32 bytes): all realignment shifts, heads and
    tails."""
    es = torch.empty((), dtype=dtype).element_size()
    for a in range(16 // es):
        dev, host, keep = _shards(3, a + part + 5, dtype, seed=100 * part + a)
        for b in range(32 // es):
            _gather_and_check(dev, host, a, part, dtype, dst_elem_offset=b)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("world,part,src_off,dst_off", [
    (8, 3_000_000, 0, 0),          # aligned: several iterations per thread
    (8, 3_000_000, 0, 8),          # 16-byte phase shared, 32-byte heads of 16 bytes (fp16)
    (8, 3_000_003, 0, 0),          # ranks off the phase: realigned blocks
    (5, 1_234_567, 3, 1),          # everything off the phase, odd world
    (2, 49_152, 0, 0),             # iterations ending at slice ends
    (16, 65_536 + 8, 8, 0),        # aligned with a shard offset
])
def test_large_gathers(dtype, world, part, src_off, dst_off):
    dev, host, keep = _shards(world, src_off + part + 3, dtype, seed=world * 7 + part)
    _gather_and_check(dev, host, src_off, part, dtype, dst_elem_offset=dst_off)


def test_odd_partition_gather_past_l2():
    """The tiny workload's partition shape (odd P, 4 ranks) scaled to 4 x
    25,000,001 fp16 elements (200 MB of destination): ranks 1-3 sit off the
    destination's 16-byte phase."""
    dev, host, keep = _shards(4, 25_000_001, torch.float16, seed=4242)
    _gather_and_check(dev, host, 0, 25_000_001, torch.float16)


def test_repeated_gathers_into_one_buffer():
    """Consecutive gathers of different units into one reused layer buffer
    (the Stage-3 pattern): each result is the current unit's, bit for bit."""
    import zero_sharded_optimizer_reduce_b200 as Z
    world, parts = 8, [100_000, 70_001, 100_000]
    offs = np.concatenate([[0], np.cumsum(parts)])
    dev, host, keep = _shards(world, int(offs[-1]), torch.bfloat16, seed=77)
    layer = torch.empty(world * max(parts), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for u, P in enumerate(parts):
        Z.zero_allgather_params(dev, int(offs[u]), P, layer[:world * P], status=status)
        torch.cuda.synchronize()
        got = layer[:world * P].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, oracle.allgather(host, int(offs[u]), P))
    assert int(status.item()) == 0
