"""Build libfp8q.so in-tree with nvcc for sm_100a (no JIT cache, no install)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libfp8q.so")
# The checked build: the same sources with -DFP8Q_CHECKS (device-side bounds
# checks that record FP8Q_ERR_BOUNDS instead of writing out of bounds).
LIB_CHECKS = os.path.join(HERE, "libfp8q_checks.so")
MAIN = os.path.join(CSRC, "fp8q_lib.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    # IEEE division and denormals: the scale s = amax/448 and the cast input
    # x/s are specified as correctly rounded FP32 operations.
    "-prec-div=true", "-prec-sqrt=true", "-ftz=false", "-fmad=true",
    "-Xcompiler", "-fPIC", "-shared",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(ROOT, "include", "fp8q.h")])


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def needs_build(checks: bool = False) -> bool:
    lib = LIB_CHECKS if checks else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    lib = LIB_CHECKS if checks else LIB
    if not force and not needs_build(checks):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *(["-DFP8Q_CHECKS"] if checks else []), "-o", tmp, MAIN]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checks="--checks" in sys.argv))
