"""Device memory of each way to run the step, against the byte counts it is
designed to have (the pages' accounting: 2 + 2 + 12 bytes of model state per
parameter, optimizer states 12 bytes per element of the partition).

ZeroAdam on one GPU holds all N partitions, so per element of the bucket:
  banks:   N x 2 (replica gradients) + 2 x (12 state + 2 parameters)
  inplace: N x 2 + 12 + 2                       (one bank: the pages' 12 Psi)
  staged:  N x 2 + 12 + 2 + 4 (reduced fp32 gradients)
plus 8 bytes of flags.  Checked on the tensors the optimizer owns, and with
the caching allocator's count of allocated bytes around the constructor
(which rounds each block up by less than 1 MiB).
"""
import pytest
import torch

import zero_sharded_optimizer_reduce_b200 as Z

pytestmark = pytest.mark.gpu


def _device_tensors(opt):
    out = [g for per in opt.grads for g in per] + [opt.flags]
    for banks in (opt.master, opt.m, opt.v, opt.params_bank):
        out += [t for per in banks for t in per]
    if opt.reduced is not None:
        out += list(opt.reduced)
    return out


@pytest.mark.parametrize("mode,per_elem", [("banks", lambda n: 2 * n + 28), ("inplace", lambda n: 2 * n + 14),
                                           ("staged", lambda n: 2 * n + 18)])
@pytest.mark.parametrize("world", [1, 4, 8])
def test_allocated_bytes_match_the_design(mode, per_elem, world):
    psi = 64_000_000                              # a multiple of every N here
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    before = torch.cuda.memory_allocated()
    opt = Z.ZeroAdam([psi], world, mode=mode)
    torch.cuda.synchronize()
    used = torch.cuda.memory_allocated() - before
    expect = psi * per_elem(world)
    tensors = _device_tensors(opt)
    # the tensors themselves hold exactly the designed bytes (+ the 8-byte flag pair)
    assert sum(t.numel() * t.element_size() for t in tensors) == expect + 8
    # the allocator rounds each block up, by less than 1 MiB (a remainder under
    # 1 MiB is not split off a large segment)
    assert expect <= used <= expect + len(tensors) * (1 << 20), (used, expect)
    # one bank of fp32 state in the one-bank modes: 12 bytes per element, the pages' 12 Psi
    assert sum(len(b) for b in opt.master) == (2 if mode == "banks" else 1)
    del opt, tensors
    torch.cuda.empty_cache()
