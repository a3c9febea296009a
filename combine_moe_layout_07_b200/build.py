"""Builds the CUDA library ``libmoe_b200.so`` in-tree with nvcc for sm_100a.

Sources: ``csrc/*.cu`` (kernels and the C ABI of ``include/moe.h``).  The CUDA runtime is
linked statically, so the library needs only the driver at run time.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe_b200.so")
DEBUG_LIB = os.path.join(PKG, "libmoe_b200_debug.so")  # MOE_DEBUG: index checks in the kernels

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-Xptxas", "-warn-spills",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "moe.h")])


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile csrc/*.cu into the in-tree library; debug=True adds the MOE_DEBUG index checks
    (a separate library file, used only when MOE_B200_DEBUG=1)."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not stale(lib):
        return lib
    cus = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DMOE_DEBUG"] if debug else []), "-I", INCLUDE, "-I", CSRC, "-o", tmp, *cus]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
