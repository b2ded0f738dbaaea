"""Build libfp4.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m fp4_block_scaled_deterministic_b200.build [--force]

The library is one translation unit (csrc/fp4_api.cu including the kernel headers),
compiled with -gencode arch=compute_100a,code=sm_100a and linked against the static
CUDA runtime; the CUDA driver is reached at run time through the runtime's
driver-entry-point query, so no -lcuda is needed at build time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfp4.so")
SOURCES = [os.path.join(CSRC, f) for f in ("fp4_api.cu",)]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("common.cuh", "quantize.cuh", "gemm.cuh")] + [
    os.path.join(ROOT, "include", "fp4.h")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(extra=()):
    return ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", os.path.join(ROOT, "include"), *extra]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *flags(), "-shared", "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
