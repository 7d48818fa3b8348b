"""Build libzero.so (the C ABI of include/zero.h) for sm_100a with nvcc.

    python zero_sharded_optimizer_reduce_b200/build.py [--verbose-ptxas] [--debug-bounds]

--debug-bounds builds libzero_debug.so instead: the same library compiled
with ZERO_DEBUG_BOUNDS, whose kernels check every index they touch and
record a failed check in the call's flag word (value 4) instead of making
the access.  The tests run parity cases through it.

Run it as a script (or load it by path): importing the package loads the
library, so the package cannot build itself on import.

The library is built in-tree, next to this file.  nvcc cross-compiles, so no
GPU is needed to build.
"""
from __future__ import annotations

import os
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libzero.so")
LIB_DEBUG = os.path.join(PKG, "libzero_debug.so")

SOURCES = ["step.cu", "step_static.cu", "stats.cu", "staged.cu", "selftest.cu", "runner.cu", "copy.cu", "host.cpp",
           "ipc.cpp"]
HEADERS = [os.path.join(CSRC, n) for n in ("bulk.cuh", "common.h", "fused_step.cuh", "grad_stats.cuh", "staged.cuh",
                                                        "staged_launch.h", "step_launch.h")] + [os.path.join(INCLUDE, "zero.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile libzero.so (or, debug_bounds, libzero_debug.so) if it is
    missing or older than its sources."""
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and not _stale(lib):
        return lib
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=PKG)
    os.close(fd)
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    if debug_bounds:
        cmd += ["-DZERO_DEBUG_BOUNDS"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", tmp]
    try:
        subprocess.check_call(cmd)
        os.replace(tmp, lib)
    finally:
        if os.path.exists(tmp):
            os.unlink(tmp)
    return lib


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
