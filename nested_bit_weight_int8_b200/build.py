"""Builds libmq.so (all CUDA sources of this package) for sm_100a, in-tree."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmq.so")
# The same sources with MQ_DEBUG_BOUNDS: device index checks that turn a bad
# index into the MQ_ERR_BOUNDS status (loaded when MQ_LIBRARY=debug).
DEBUG_LIB = os.path.join(HERE, "libmq_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=true",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps.append(os.path.join(HERE, "..", "include", "mq.h"))
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, extra=None, debug_bounds: bool = False) -> str:
    """Compile every .cu under csrc/ into libmq.so, or with the device index
    checks into libmq_debug.so (skipped when up to date)."""
    lib = DEBUG_LIB if debug_bounds else LIB
    if not force and not _stale(lib):
        return lib
    flags = [*NVCC_FLAGS, *(["-DMQ_DEBUG_BOUNDS"] if debug_bounds else []), *(extra or [])]
    cmd = [NVCC, *flags, "-o", lib + ".tmp", *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None,
          debug_bounds="--debug-bounds" in sys.argv)
