"""Compile the CUDA library (libfgfp8.so) for sm_100a with nvcc, in-tree."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfgfp8.so")
# The same library with the kernels' index checks compiled in
# (-DFGFP8_DEBUG_CHECKS): a debug build for tests, never loaded by the
# package itself.
DEBUG_LIB = os.path.join(HERE, "libfgfp8_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-shared",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          debug: bool = False) -> str:
    """Build libfgfp8.so (or, with debug, libfgfp8_debug.so with the kernels'
    index checks) if missing or older than its sources; return its path."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not is_stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    flags = [*NVCC_FLAGS, *(extra_flags or []), *(["-DFGFP8_DEBUG_CHECKS"] if debug else [])]
    cmd = [nvcc(), *flags, "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "fgfp8.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None, debug="--debug" in sys.argv))
