"""The product's host codec (tl_pack2 / tl_pack16 / tl_unpack) against the
oracle, bit for bit, on exhaustive and random inputs."""
import itertools

import numpy as np
import pytest

import oracle
import synth
import ternary_weight_03_b200 as tl
from ternary_weight_03_b200 import build as tlbuild

FMTS = (2, 16)


@pytest.fixture(scope="module", autouse=True)
def _built():
    tlbuild.build()


@pytest.fixture(scope="module")
def o():
    return oracle.get()


@pytest.mark.parametrize("fmt", FMTS)
def test_exhaustive_tuples(o, fmt):
    g = 4 if fmt == 2 else 5
    T = np.array(list(itertools.product((-1, 0, 1), repeat=g)), dtype=np.int8)
    assert np.array_equal(tl.pack(fmt, T, ldp=1), o.pack(fmt, T))


@pytest.mark.parametrize("fmt", FMTS)
def test_every_K_1_to_300(o, fmt):
    for K in range(1, 301):
        N = 1 + K % 4
        T = synth.trits(K, N, K, p0=[0.2, 1 / 3, 0.6][K % 3])
        rb = tl.row_bytes(fmt, K)
        for ldp in (rb, rb + 3, tl.padded_ldp(fmt, K)):
            got = tl.pack(fmt, T, ldp=ldp)
            ref = o.pack(fmt, T, ldp=ldp)
            assert np.array_equal(got, ref), (fmt, K, ldp)
            assert np.array_equal(tl.unpack(fmt, got, K), T)


@pytest.mark.parametrize("fmt", FMTS)
def test_large_matrix_threaded(o, fmt):
    # large enough to take the multithreaded path of the packer
    T = synth.trits(5, 1024, 4100)
    got = tl.pack(fmt, T)
    ref = o.pack(fmt, T, ldp=got.shape[1])
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_unpack_all_bytes(o, fmt):
    g = 4 if fmt == 2 else 5
    for v in range(256):
        P = np.array([[v]], dtype=np.uint8)
        rc_o, T_o, _ = o.unpack(fmt, P, g)
        if rc_o == 0:
            assert np.array_equal(tl.unpack(fmt, P, g), T_o)
        else:
            with pytest.raises(tl.TLError) as e:
                tl.unpack(fmt, P, g)
            assert e.value.status == 3 and e.value.bad_index == 0


@pytest.mark.parametrize("fmt,bad", [(2, 0xFF), (2, 0x03), (16, 243), (16, 255)])
def test_bad_index_matches_oracle(o, fmt, bad):
    T = synth.trits(1, 9, 77)
    P = tl.pack(fmt, T, ldp=32)
    P[4, 7] = bad
    P[6, 1] = bad
    rc, _, idx = o.unpack(fmt, P, 77)
    with pytest.raises(tl.TLError) as e:
        tl.unpack(fmt, P, 77)
    assert rc == 3 and e.value.bad_index == idx == 4 * 32 + 7


@pytest.mark.parametrize("fmt", FMTS)
def test_bad_trit_rejected(fmt):
    T = np.zeros((4, 9), dtype=np.int8)
    T[2, 3] = 2
    with pytest.raises(tl.TLError) as e:
        tl.pack(fmt, T)
    assert e.value.status == 2


def test_invalid_args():
    L = tl.lib()
    T = np.zeros((2, 8), dtype=np.int8)
    P = np.zeros((2, 16), dtype=np.uint8)
    assert L.tl_pack2(T.ctypes.data, 2, 8, 4, P.ctypes.data, 16) == 1   # ldt < K
    assert L.tl_pack2(T.ctypes.data, 2, 8, 8, P.ctypes.data, 1) == 1    # ldp < row bytes
    assert L.tl_pack16(None, 2, 8, 8, P.ctypes.data, 16) == 1
    assert L.tl_pack2(T.ctypes.data, 0, 8, 8, P.ctypes.data, 16) == 0   # empty is fine
    assert L.tl_unpack(5, P.ctypes.data, 2, 8, 16, T.ctypes.data, 8, None) == 1


def test_memory_ratio():
    """2-bit is 1/8 of fp16 bytes; 1.6-bit is about 1/10."""
    assert tl.row_bytes(2, 4096) * 8 == 2 * 4096
    assert abs(2 * 14335 / tl.row_bytes(16, 14335) - 10) < 0.01
