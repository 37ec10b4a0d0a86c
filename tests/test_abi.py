"""The C ABI library loads and exports every symbol of include/tl.h, and the
host-side argument rules reject bad calls before anything reaches a GPU."""
import re
from pathlib import Path

import pytest

import ternary_weight_03_b200 as tl
from ternary_weight_03_b200 import build as tlbuild

HEADER = Path(__file__).resolve().parent.parent / "include" / "tl.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tl_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    tlbuild.build()
    return tl.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "tl_gemv" in names and "tl_pack2" in names
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(tl.SIGNATURES), "binding and header disagree"


def test_status_strings(L):
    for code, name in tl.STATUS.items():
        assert tl.status_str(code).startswith(name)
    assert tl.status_str(99) == "unknown tl status"


def test_row_bytes(L):
    assert tl.row_bytes(2, 1024) == 256 and tl.row_bytes(2, 1025) == 257
    assert tl.row_bytes(16, 1024) == 205 and tl.row_bytes(16, 5) == 1
    assert tl.row_bytes(3, 10) == -1 and tl.row_bytes(2, -1) == -1
    assert tl.padded_ldp(16, 1024) == 208


A = 0x10000  # fake, 16-byte aligned device addresses (never dereferenced)


def gemv_rc(L, fmt=2, dT=A, ldp=256, dX=A, ldx=1024, dY=A, ldy=1024, M=1, N=1024, K=1024,
            fn="tl_gemv"):
    return getattr(L, fn)(fmt, dT, ldp, 0.5, dX, ldx, dY, ldy, M, N, K, None)


@pytest.mark.parametrize("kw,rc", [
    (dict(fmt=3), 1), (dict(dT=0), 1), (dict(dX=0), 1), (dict(dY=0), 1),
    (dict(M=0), 1), (dict(M=9), 1), (dict(N=0), 1), (dict(K=0), 1), (dict(K=-5), 1),
    (dict(ldp=255), 1), (dict(ldx=1016), 1), (dict(ldy=1000), 1),
    (dict(dT=A + 8), 4), (dict(dX=A + 2), 4), (dict(dY=A + 4), 4),
    (dict(ldp=272, K=1024), 0), (dict(ldp=264), 4), (dict(ldx=1028), 4), (dict(ldy=1028), 4),
    (dict(fmt=16, ldp=204), 1), (dict(fmt=16, ldp=200), 1),
])
def test_gemv_argument_rules(L, kw, rc):
    if rc == 0:
        pytest.skip("valid arguments would launch a kernel (GPU test)")
    assert gemv_rc(L, **kw) == rc


def test_gemm_argument_rules(L):
    assert gemv_rc(L, fn="tl_gemm", M=15) == 1
    assert gemv_rc(L, fn="tl_gemm", M=0) == 1
    assert gemv_rc(L, fn="tl_gemm", M=64, dX=A + 2) == 4
    assert gemv_rc(L, fn="tl_gemm", M=64, ldp=128) == 1


def test_build_flags_target_sm100a():
    flags = " ".join(tlbuild.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags and "-lineinfo" in flags


def test_gemv_ex_flags(L):
    assert gemv_rc(L, fn="tl_gemv", M=0) == 1
    A_ = 0x10000
    # unknown flag bits are rejected before anything reaches a device
    assert L.tl_gemv_ex(2, A_, 256, 1.0, A_, 1024, A_, 1024, 1, 1024, 1024, 2, None) == 1
    assert L.tl_gemv_ex(2, A_, 256, 1.0, A_, 1024, A_, 1024, 9, 1024, 1024, 1, None) == 1
