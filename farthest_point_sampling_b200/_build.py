"""Builds the in-tree CUDA library ``libfpstok.so`` for sm_100a with nvcc.

Flags: ``-fmad=false`` (no contraction anywhere in device code; the distance
also uses explicit round-to-nearest operations), ``-lineinfo`` for profiling,
no fast-math.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfpstok.so")
MICROBENCH_SRC = os.path.join(HERE, "microbench", "fp32_rate.cu")
MICROBENCH_LIB = os.path.join(HERE, "libfpstok_microbench.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-fmad=false",
    "-Xcompiler", "-fPIC,-O2", "-shared", "-Xptxas", "-warn-spills",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the fpstok CUDA library cannot be built")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in deps())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile every ``csrc/*.cu`` into ``libfpstok.so`` (in-tree) when stale."""
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, *sources(), "-o", tmp]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


def build_microbench(force: bool = False) -> str:
    """Compile the FP32-rate microbenchmark used by bench.py for its roofline."""
    if force or not os.path.exists(MICROBENCH_LIB) or \
            os.path.getmtime(MICROBENCH_LIB) < os.path.getmtime(MICROBENCH_SRC):
        tmp = MICROBENCH_LIB + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc(), *NVCC_FLAGS, MICROBENCH_SRC, "-o", tmp])
        os.replace(tmp, MICROBENCH_LIB)
    return MICROBENCH_LIB


if __name__ == "__main__":
    import sys
    build(force=True, verbose=True, extra=sys.argv[1:])
    build_microbench(force=True)
