"""Build libternary.so in-tree with nvcc for sm_100a.

    python -m ternary_weight_03_b200.build [--force]

The library holds the host codec (tl_host.cpp) and every CUDA kernel
(tl_device.cu and the headers it includes), compiled for
``-gencode arch=compute_100a,code=sm_100a`` with line info.  nvcc
cross-compiles, so this runs on a machine without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libternary.so"
SOURCES = [CSRC / "tl_device.cu", CSRC / "tl_host.cpp"]
DEPENDS = SOURCES + sorted(CSRC.glob("*.cuh")) + [INCLUDE / "tl.h"]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-pthread"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    return any(p.stat().st_mtime > t for p in DEPENDS)


def build(force: bool = False, verbose: bool = False) -> Path:
    if not force and not stale():
        return LIB
    tmp = LIB.with_name(f"libternary.so.tmp{os.getpid()}")
    cmd = [nvcc(), *NVCC_FLAGS, f"-I{INCLUDE}", f"-I{CSRC}", *map(str, SOURCES), "-o", str(tmp)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
