"""Builds ``libsdnq.so`` in-tree with nvcc for sm_100a (B200). No GPU is needed to build."""
from __future__ import annotations

import glob
import os
import subprocess
import sys
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsdnq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-fmad=false",            # no implicit multiply-add contraction anywhere in the library
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-shared",
]

_lock = threading.Lock()


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "sdnq.h")])


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None) -> str:
    """Compile ``csrc/libsdnq.cu`` (which includes every kernel) into ``libsdnq.so``."""
    with _lock:
        if not force and not is_stale():
            return LIB
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-I", CSRC,
               os.path.join(CSRC, "libsdnq.cu"), "-o", tmp]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(LIB)
