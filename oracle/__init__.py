"""Python binding of the CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke
check and the benchmark's CPU-baseline leg, never by the product.  The
oracle shares no code with the CUDA path; see ``oracle.c`` for the passages
each function follows and the readings taken where the pages are silent.

Arrays are numpy: trits ``int8 [N, K]``, packed ``uint8 [N, ldp]``,
activations ``float16 [M, K]`` (passed as their IEEE bit patterns),
outputs ``float64 [M, N]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "oracle.c"

FMT_2BIT = 2
FMT_1P6BIT = 16
OK, INVALID_ARG, BAD_TRIT, BAD_CODE = 0, 1, 2, 3


def lib_path(mutant: int = 0) -> Path:
    return HERE / ("liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so")


def build(mutant: int = 0, force: bool = False) -> Path:
    """Compile oracle.c with gcc (optionally with one planted mistake)."""
    out = lib_path(mutant)
    if out.exists() and not force and out.stat().st_mtime >= SRC.stat().st_mtime:
        return out
    tmp = out.with_suffix(f".so.tmp{os.getpid()}")
    cmd = ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread",
           f"-DORACLE_MUTANT={mutant}", str(SRC), "-o", str(tmp), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


_i64 = ctypes.c_int64
_p = ctypes.c_void_p


class Oracle:
    """ctypes wrapper around one build of the oracle library."""

    def __init__(self, mutant: int = 0):
        self.mutant = mutant
        self.lib = ctypes.CDLL(str(build(mutant)))
        L = self.lib
        L.or_digits_per_byte.argtypes = [ctypes.c_int]
        L.or_digit_base.argtypes = [ctypes.c_int]
        L.or_fits.argtypes = [ctypes.c_int, ctypes.c_int]
        L.or_row_bytes.argtypes = [ctypes.c_int, _i64]
        L.or_row_bytes.restype = _i64
        L.or_pack.argtypes = [ctypes.c_int, _p, _i64, _i64, _i64, _p, _i64]
        L.or_unpack.argtypes = [ctypes.c_int, _p, _i64, _i64, _i64, _p, _i64,
                                ctypes.POINTER(_i64)]
        L.or_half_to_double.argtypes = [ctypes.c_uint16]
        L.or_half_to_double.restype = ctypes.c_double
        L.or_linear.argtypes = [_p, _i64, _p, _i64, ctypes.c_double, _i64, _i64, _i64,
                                _p, _i64, ctypes.c_int]
        L.or_linear_at.argtypes = [_p, _i64, _p, _i64, ctypes.c_double, _i64, _p, _p,
                                   _i64, _p]

    # -- packing ----------------------------------------------------------
    def digits_per_byte(self, fmt: int) -> int:
        return self.lib.or_digits_per_byte(fmt)

    def fits(self, k: int, p: int) -> bool:
        return bool(self.lib.or_fits(k, p))

    def row_bytes(self, fmt: int, K: int) -> int:
        return int(self.lib.or_row_bytes(fmt, K))

    def pack(self, fmt: int, T: np.ndarray, ldp: int | None = None) -> np.ndarray:
        T = np.ascontiguousarray(T, dtype=np.int8)
        N, K = T.shape
        rb = self.row_bytes(fmt, K)
        ldp = rb if ldp is None else ldp
        P = np.full((N, max(ldp, 1)), 0xEE, dtype=np.uint8)
        rc = self.lib.or_pack(fmt, T.ctypes.data, N, K, K, P.ctypes.data, ldp)
        if rc != OK:
            raise ValueError(f"or_pack failed with status {rc}")
        return P[:, :ldp]

    def pack_status(self, fmt: int, T: np.ndarray) -> int:
        T = np.ascontiguousarray(T, dtype=np.int8)
        N, K = T.shape
        rb = self.row_bytes(fmt, K)
        P = np.zeros((N, max(rb, 1)), dtype=np.uint8)
        return self.lib.or_pack(fmt, T.ctypes.data, N, K, K, P.ctypes.data, rb)

    def unpack(self, fmt: int, P: np.ndarray, K: int):
        """Returns (status, trits int8 [N,K], bad_index or -1)."""
        P = np.ascontiguousarray(P, dtype=np.uint8)
        N, ldp = P.shape
        T = np.full((N, max(K, 1)), 99, dtype=np.int8)
        bad = _i64(-1)
        rc = self.lib.or_unpack(fmt, P.ctypes.data, N, K, ldp, T.ctypes.data, max(K, 1),
                                ctypes.byref(bad))
        return rc, T[:, :K], int(bad.value)

    # -- arithmetic ---------------------------------------------------------
    def half_to_double(self, bits: int) -> float:
        return float(self.lib.or_half_to_double(bits))

    def linear(self, T: np.ndarray, X: np.ndarray, alpha: float, nthreads: int = 1) -> np.ndarray:
        """Y[m,n] = alpha * sum_k T[n,k] X[m,k] in double, from int8 trits."""
        T = np.ascontiguousarray(T, dtype=np.int8)
        X = np.ascontiguousarray(X, dtype=np.float16).view(np.uint16)
        N, K = T.shape
        M, K2 = X.shape
        assert K == K2
        Y = np.empty((M, N), dtype=np.float64)
        rc = self.lib.or_linear(T.ctypes.data, K, X.ctypes.data, K, float(alpha), M, N, K,
                                Y.ctypes.data, N, int(nthreads))
        if rc != OK:
            raise ValueError(f"or_linear failed with status {rc}")
        return Y

    def linear_at(self, T: np.ndarray, X: np.ndarray, alpha: float, ms, ns) -> np.ndarray:
        """The same definition at the listed (m, n) pairs only."""
        T = np.ascontiguousarray(T, dtype=np.int8)
        X = np.ascontiguousarray(X, dtype=np.float16).view(np.uint16)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        ns = np.ascontiguousarray(ns, dtype=np.int64)
        N, K = T.shape
        assert ms.shape == ns.shape
        assert (ms >= 0).all() and (ms < X.shape[0]).all()
        assert (ns >= 0).all() and (ns < N).all()
        out = np.empty(ms.shape, dtype=np.float64)
        rc = self.lib.or_linear_at(T.ctypes.data, K, X.ctypes.data, X.shape[1], float(alpha), K,
                                   ms.ctypes.data, ns.ctypes.data, ms.size, out.ctypes.data)
        if rc != OK:
            raise ValueError(f"or_linear_at failed with status {rc}")
        return out


_default: Oracle | None = None


def get() -> Oracle:
    """The unmodified oracle (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(0)
    return _default


def tolerance(y_ref: np.ndarray, X: np.ndarray, alpha: float) -> np.ndarray:
    """Per-element bound |y - y_ref| <= 1e-3 * |alpha| * sum_k |x[m,k]| + ulp16(y_ref).

    ulp16(v) is the spacing of binary16 numbers at |v|: 2^(floor(log2|v|) - 10)
    for |v| >= 2^-14, else 2^-24.  y_ref is [M, N] (or a vector of sampled
    values, in which case X must already be the matching rows).
    """
    X = np.asarray(X, dtype=np.float16).astype(np.float64)
    s = np.abs(X).sum(axis=-1)
    a = np.abs(y_ref)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.where(a >= 2.0 ** -14, np.exp2(e - 10), 2.0 ** -24)
    if y_ref.ndim == 2:
        return 1e-3 * abs(alpha) * s[:, None] + ulp
    return 1e-3 * abs(alpha) * s + ulp
