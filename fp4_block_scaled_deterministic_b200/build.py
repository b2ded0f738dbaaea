"""Build libfp4.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m fp4_block_scaled_deterministic_b200.build [--force] [--debug]

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
# The same sources with -DFP4_DEBUG_BOUNDS: every kernel range-checks its computed
# shared-memory offsets, TMEM columns, tile coordinates and global indices, records a
# failure in the status word and skips the access (fp4_check_status -> FP4_ERR_BOUNDS).
LIB_DEBUG = os.path.join(PKG, "libfp4_debug.so")
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


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile libfp4.so (debug=True: libfp4_debug.so with the device-side range checks)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc(), *flags(["-DFP4_DEBUG_BOUNDS"] if debug else []), "-shared", "-o", tmp,
           *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False) -> None:
    """Both libraries, compiled in parallel."""
    import concurrent.futures as cf
    with cf.ThreadPoolExecutor(2) as ex:
        for f in [ex.submit(build, force, False, d) for d in (False, True)]:
            f.result()


if __name__ == "__main__":
    if "--debug" in sys.argv:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug=True))
    else:
        build_all(force="--force" in sys.argv)
        print(LIB)
        print(LIB_DEBUG)
