"""Compile the sm_100a CUDA library (libffd_b200.so) in-tree with nvcc.

The library is rebuilt when any source under csrc/ or include/ is newer than
the shared object.  Usage: ``python -m sparse_long_context_ffd_b200.build``.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libffd_b200.so")
# the same sources with FFD_DEBUG: every global index the decode kernel
# computes is bounds-checked and flagged (FFD_DEVICE_FLAG_BOUNDS); for tests
# (ffd.use_debug_library())
DEBUG_LIB = os.path.join(PKG, "libffd_b200_debug.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def is_stale(path: str = None) -> bool:
    path = path or LIB
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(f) > t for f in _inputs())


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the FFD CUDA library cannot be built")
    return path


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    target = DEBUG_LIB if debug else LIB
    if not force and not is_stale(target):
        return target
    tmp = target + f".tmp{os.getpid()}"
    flags = [*extra, "-DFFD_DEBUG"] if debug else list(extra)
    cmd = [nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, *flags, "-I", INCLUDE, "-I", CSRC,
           "-cudart", "static", "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    debug = "--debug" in sys.argv
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else (), debug=debug))
