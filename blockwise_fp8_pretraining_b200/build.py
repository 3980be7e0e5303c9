"""Build the CUDA library in-tree: libfp8blk.so next to this file.

    python -m blockwise_fp8_pretraining_b200.build [--force]

Compiles csrc/fp8blk.cu for sm_100a only.  IEEE division, square root and
denormals are kept (no fast-math, no flush-to-zero): the quantizer's
bit-exact definition depends on them.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8blk.so")
SOURCES = [os.path.join(CSRC, f) for f in ("fp8blk.cu", "gemm.cuh", "quantize.cuh", "ptx.cuh", "swiglu.cuh", "rmsnorm.cuh")]
HEADER = os.path.join(os.path.dirname(HERE), "include", "fp8blk.h")

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in SOURCES + [HEADER] if os.path.exists(s))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-o", tmp, os.path.join(CSRC, "fp8blk.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
