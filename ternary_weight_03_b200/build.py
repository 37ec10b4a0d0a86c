"""Build libternary.so in-tree with nvcc for sm_100a.

    python -m ternary_weight_03_b200.build [--force]

The library holds the host codec (tl_host.cpp) and every CUDA kernel
(tl_device.cu and the headers it includes), compiled for
``-gencode arch=compute_100a,code=sm_100a`` with line info.  nvcc
cross-compiles, so this runs on a machine without a GPU.

A second library, libternary_debug.so, is the same sources compiled with
TL_DEBUG_HOOKS: it also honours TL_FLAG_DEBUG_DROP_ARRIVE (failure-detection
tests).  The product binding never loads it.
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
DEBUG_LIB = PKG / "libternary_debug.so"
SOURCES = [CSRC / "tl_device.cu", CSRC / "tl_host.cpp"]
EXPORTS = CSRC / "exports.map"
DEPENDS = SOURCES + sorted(CSRC.glob("*.cuh")) + [INCLUDE / "tl.h", INCLUDE / "tl_debug.h", EXPORTS]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-pthread",
              f"-Xlinker=--version-script={EXPORTS}"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale(lib: Path = LIB) -> bool:
    if not lib.exists():
        return True
    t = lib.stat().st_mtime
    return any(p.stat().st_mtime > t for p in DEPENDS)


def _compile(lib: Path, defines: list[str], verbose: bool) -> None:
    tmp = lib.with_name(f"{lib.name}.tmp{os.getpid()}")
    cmd = [nvcc(), *NVCC_FLAGS, *defines, f"-I{INCLUDE}", f"-I{CSRC}", *map(str, SOURCES), "-o",
           str(tmp)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> Path:
    """Build the product library (and, unless debug=False, the debug one)."""
    if force or stale(LIB):
        _compile(LIB, [], verbose)
    if debug and (force or stale(DEBUG_LIB)):
        _compile(DEBUG_LIB, ["-DTL_DEBUG_HOOKS"], verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
