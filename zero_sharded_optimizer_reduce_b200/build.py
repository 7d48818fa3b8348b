"""Build libzero.so (the C ABI of include/zero.h) for sm_100a with nvcc.

    python zero_sharded_optimizer_reduce_b200/build.py [--verbose-ptxas]

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

SOURCES = ["step.cu", "step_static.cu", "stats.cu", "staged.cu", "selftest.cu", "runner.cu", "copy.cu", "host.cpp",
           "ipc.cpp"]
HEADERS = [os.path.join(CSRC, n) for n in ("common.h", "fused_step.cuh", "grad_stats.cuh", "staged.cuh",
                                                        "step_launch.h")] + [os.path.join(INCLUDE, "zero.h")]

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


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile libzero.so if it is missing or older than its sources."""
    if not force and not _stale():
        return LIB
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=PKG)
    os.close(fd)
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", tmp]
    try:
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    finally:
        if os.path.exists(tmp):
            os.unlink(tmp)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
