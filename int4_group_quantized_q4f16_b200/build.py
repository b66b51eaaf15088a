"""Build the CUDA library in-tree: nvcc for sm_100a -> libzt_q4.so beside this file,
and the bounds-checked build of the same sources (-DZT_Q4_CHECKED) -> libzt_q4_checked.so.

Run ``python -m int4_group_quantized_q4f16_b200.build``.  The library links the
CUDA runtime statically, so it loads on a machine without a GPU (every entry
point that needs the device then returns an error status instead).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libzt_q4.so")
LIB_CHECKED = os.path.join(PKG, "libzt_q4_checked.so")
SOURCES = ["zt_q4.cu"]
HEADERS = ["q4_common.cuh", "q4_mma.cuh", "q4_pass.cuh", "q4_gemm_tc.cuh"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def sources():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS] +
            [os.path.join(INCLUDE, h) for h in os.listdir(INCLUDE) if h.endswith(".h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build_checked(force: bool = False, verbose: bool = False) -> str:
    return build(force, verbose, LIB_CHECKED, ["-DZT_Q4_CHECKED"])


def build(force: bool = False, verbose: bool = False, out: str = LIB, extra=()) -> str:
    if not force and not stale(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build_checked(force="--force" in sys.argv, verbose=True))
