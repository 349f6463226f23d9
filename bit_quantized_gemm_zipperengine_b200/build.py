"""Build libmosaic.so (CUDA, sm_100a) in-tree with nvcc."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmosaic.so")
# the same library with MQ_TIMELINE defined: the small decode GEMM records per-CTA event
# times (mq_timeline_read); used by timeline.py, never by the path
LIB_TIMELINE = os.path.join(PKG, "libmosaic_timeline.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    # IEEE fp32 division / rounding are part of the quantization spec: no fast math,
    # no contraction of multiply-add pairs.
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC", "-shared",
    "-I" + INCLUDE, "-I" + CSRC,
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return (sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + sorted(glob.glob(os.path.join(INCLUDE, "*.h")))
            + [__file__])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in deps())


def build(force: bool = False, verbose: bool = False, timeline: bool = False) -> str:
    lib = LIB_TIMELINE if timeline else LIB
    if not (force or stale(lib)):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(["-DMQ_TIMELINE"] if timeline else []), *(["-Xptxas", "-v"] if verbose else []),
           "-o", tmp, *sources()]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
