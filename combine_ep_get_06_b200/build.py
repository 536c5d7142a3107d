"""Builds the CUDA library libep_b200.so in-tree (sm_100a only).

    python -m combine_ep_get_06_b200.build [--force] [--verbose] [--checked]

--checked builds libep_b200_checked.so instead: the same kernels compiled
with EP_CHECKED, whose device-side invariant checks set EP_DEVERR_CHECK in
the error word (and skip the access) instead of trapping.  The binding
loads it when EP_CHECKED=1 is set in the environment.

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically, exports only the ep_* C-ABI symbols (include/ep.h) and is
loaded by the ctypes binding in this package.
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
OUT_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(OUT_DIR, "libep_b200.so")
CHECKED_LIB = os.path.join(OUT_DIR, "libep_b200_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put the CUDA toolkit on PATH)")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def up_to_date(checked: bool = False) -> bool:
    lib = CHECKED_LIB if checked else LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = CHECKED_LIB if checked else LIB
    if not force and up_to_date(checked):
        return lib
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-cudart", "static",
           "-Xcompiler", "-fPIC,-fvisibility=hidden,-O2", "-I", INCLUDE, "-I", CSRC,
           *(["-DEP_CHECKED=1"] if checked else []), "-o", tmp, *sources()]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
