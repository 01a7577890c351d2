"""Builds the CUDA library libconv_b200.so in the package directory (sm_100a only).

The whole library is one translation unit (csrc/capi.cu includes the kernel headers), built
with nvcc for compute_100a / sm_100a. Floating-point flags keep IEEE behaviour: no fast math,
denormals preserved (-ftz=false), no implicit multiply-add contraction (-fmad=false); the
kernels ask for fused multiply-adds explicitly where the contract wants them.
"""
from __future__ import annotations

import fcntl
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libconv_b200.so")
# the same sources compiled with -DCONV_DEBUG_BOUNDS: every computed global access and 1-D bulk
# copy checked against its tensor's extent (failures set a status bit and skip the access)
LIB_DEBUG = os.path.join(PKG, "libconv_b200_debug.so")
MAIN = os.path.join(PKG, "csrc", "capi.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*")) + [os.path.join(ROOT, "include", "conv_b200.h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile the library (or, with debug_bounds, its bounds-checked variant) if it is missing
    or older than its sources; returns its path."""
    lib = LIB_DEBUG if debug_bounds else LIB
    lock_path = os.path.join(PKG, ".build.lock")
    with open(lock_path, "w") as lk:
        fcntl.flock(lk, fcntl.LOCK_EX)
        try:
            if force or stale(lib):
                tmp = lib + f".tmp{os.getpid()}"
                cmd = [nvcc(), *NVCC_FLAGS, *(["-DCONV_DEBUG_BOUNDS"] if debug_bounds else []),
                       *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, MAIN, "-lcublas"]
                r = subprocess.run(cmd, capture_output=True, text=True)
                if r.returncode != 0:
                    raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
                if verbose:
                    sys.stderr.write(r.stdout + r.stderr)
                os.replace(tmp, lib)
        finally:
            fcntl.flock(lk, fcntl.LOCK_UN)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
