"""Seeded synthetic inputs (random numbers only; no layer arithmetic).

Both sides of every comparison draw their inputs from here: the oracle and
the CUDA path receive the same trits, activations and scales.  The numbers
come from SplitMix64 (``synth.c``); see that file for the exact recipe.

Workload recipe (layer shapes of the benchmarks):
  * trits T[n, k] i.i.d. with P(0) = p0, P(-1) = P(+1) = (1 - p0) / 2
  * activations X[m, k] = binary16 round-to-nearest-even of N(0, 1)
  * scale alpha fixed (0.02) or U(0.01, 0.05) per matrix
Stream tags keep T, X and alpha of one seed independent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "synth.c"
LIB = HERE / "libsynth.so"

STREAM_T = 1
STREAM_X = 2
STREAM_ALPHA = 3


def build(force: bool = False) -> Path:
    if LIB.exists() and not force and LIB.stat().st_mtime >= SRC.stat().st_mtime:
        return LIB
    tmp = LIB.with_suffix(f".so.tmp{os.getpid()}")
    subprocess.run(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread", str(SRC),
                    "-o", str(tmp), "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(str(build()))
        u64, i64, p = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        _lib.sy_next.argtypes = [ctypes.POINTER(u64)]
        _lib.sy_next.restype = u64
        _lib.sy_key.argtypes = [u64, u64]
        _lib.sy_key.restype = u64
        _lib.sy_u64.argtypes = [u64, i64, p]
        _lib.sy_uniform.argtypes = [u64, i64, ctypes.c_double, ctypes.c_double, p]
        _lib.sy_trits.argtypes = [u64, i64, i64, i64, ctypes.c_double, p, ctypes.c_int]
        _lib.sy_normals.argtypes = [u64, i64, i64, i64, p, ctypes.c_int]
    return _lib


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def splitmix64(seed: int, n: int) -> list[int]:
    """The first n outputs of sequential SplitMix64 started at state `seed`."""
    st = ctypes.c_uint64(seed & (2**64 - 1))
    return [int(_L().sy_next(ctypes.byref(st))) for _ in range(n)]


def key(seed: int, stream: int) -> int:
    return int(_L().sy_key(seed & (2**64 - 1), stream))


def u64_stream(k: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _L().sy_u64(k, n, out.ctypes.data)
    return out


def uniform(seed: int, n: int, lo: float = 0.0, hi: float = 1.0,
            stream: int = STREAM_ALPHA) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _L().sy_uniform(key(seed, stream), n, lo, hi, out.ctypes.data)
    return out


def trits(seed: int, N: int, K: int, p0: float = 1.0 / 3.0, out: np.ndarray | None = None,
          stream: int = STREAM_T) -> np.ndarray:
    """int8 [N, K] trits; `out` may be a wider C-contiguous int8 [N, ld] buffer."""
    if out is None:
        out = np.empty((N, K), dtype=np.int8)
    assert out.dtype == np.int8 and out.flags.c_contiguous and out.shape[0] == N
    ld = out.shape[1] if out.ndim == 2 else K
    assert ld >= K
    _L().sy_trits(key(seed, stream), N, K, ld, float(p0), out.ctypes.data, _threads())
    return out


def normals(seed: int, M: int, K: int, stream: int = STREAM_X) -> np.ndarray:
    out = np.empty((M, K), dtype=np.float64)
    _L().sy_normals(key(seed, stream), M, K, K, out.ctypes.data, _threads())
    return out


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """float16 [M, K]: binary16 round-to-nearest-even of standard normals."""
    return normals(seed, M, K).astype(np.float16)


def alpha_for(seed: int, fixed: float | None = None) -> float:
    """The layer scale: `fixed` if given, else U(0.01, 0.05) drawn from the seed."""
    if fixed is not None:
        return float(fixed)
    return float(uniform(seed, 1, 0.01, 0.05)[0])
