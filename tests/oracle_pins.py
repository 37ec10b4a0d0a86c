"""Pins of the CPU oracle against facts fixed outside it.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with something the pages or mathematics fix independently:
positional notation as implemented by Python's ``int(s, base)`` and numpy's
``base_repr``, numpy's IEEE binary16 conversion, numpy's float64 matrix
product, closed forms of special matrices, brute force over every ternary
matrix of a tiny shape, and the packing theorem U(P(t)) = t ("Circularity
Check" of the Pith review of Spectra 1.1: the packing maps P and U are proved
correct from their definitions, paper appendix E).

The same pins run against builds of the oracle with one planted mistake each
(tests/test_oracle_mutants.py) to show that every plausible mistake fails
at least one of them.
"""
from __future__ import annotations

import itertools
import math

import numpy as np

FMTS = {2: (4, 4), 16: (5, 3)}  # fmt -> (trits per byte g, digit base b)


def _positional(tup, base):
    """Byte of a trit tuple under readings R1/R2 via Python's int(s, base):
    digit t+1, the first trit least significant."""
    return int("".join(str(t + 1) for t in reversed(tup)), base)


def pin_fits(o):
    """k trits fit p bits iff 3^k tuples <= 2^p codes (count by enumeration);
    the pages fix k=5, p=8 as fitting and 1.6 bits near log2(3)."""
    for k in range(0, 9):
        tuples = sum(1 for _ in itertools.product(range(3), repeat=k))
        for p in range(0, 16):
            assert o.fits(k, p) == (tuples <= 2 ** p), (k, p)
    assert o.fits(5, 8) and not o.fits(6, 8) and o.fits(4, 8)
    assert 8 / 5 >= math.log2(3) and 8 / 5 - math.log2(3) < 0.016
    assert o.digits_per_byte(2) == 4 and o.digits_per_byte(16) == 5


def pin_row_bytes(o):
    """ceil(K/g) bytes per row, and the ~8x (2-bit) / ~10x (1.6-bit) memory
    reduction against 16-bit weights."""
    for fmt, (g, _) in FMTS.items():
        for K in range(0, 60):
            assert o.row_bytes(fmt, K) == -(-K // g)
    assert 2 * 4096 / o.row_bytes(2, 4096) == 8.0
    assert abs(2 * 4100 / o.row_bytes(16, 4100) - 10.0) < 1e-12


def pin_pack_positional(o):
    """Every trit tuple packs to its base-b positional value (library int())."""
    for fmt, (g, b) in FMTS.items():
        tuples = list(itertools.product((-1, 0, 1), repeat=g))
        T = np.array(tuples, dtype=np.int8)
        P = o.pack(fmt, T)
        assert P.shape == (len(tuples), 1)
        for tup, byte in zip(tuples, P[:, 0]):
            assert int(byte) == _positional(tup, b), (fmt, tup, int(byte))
        codes = sorted(int(x) for x in P[:, 0])
        assert len(set(codes)) == len(codes)  # lossless: injective
        if fmt == 16:
            assert codes == list(range(243))  # a bijection onto 0..242


def pin_unpack_all_bytes(o):
    """All 256 byte values: validity and digits from numpy base_repr."""
    for fmt, (g, b) in FMTS.items():
        P = np.arange(256, dtype=np.uint8).reshape(256, 1)
        n_valid = 0
        for v in range(256):
            rep = np.base_repr(v, b)
            valid = len(rep) <= g and "3" not in rep
            rc, T, bad = o.unpack(fmt, P[v:v + 1], g)
            assert (rc == 0) == valid, (fmt, v, rc)
            if valid:
                n_valid += 1
                digits = [int(c) for c in reversed(rep.zfill(g))]
                assert T[0].tolist() == [d - 1 for d in digits], (fmt, v)
            else:
                assert bad == 0
        assert n_valid == 3 ** g  # 81 valid 2-bit bytes, 243 valid 1.6-bit bytes


def pin_bad_index(o):
    """The first invalid byte in a row-major scan is reported."""
    for fmt, bad_byte in ((2, 0xFF), (16, 250)):
        rng = np.random.default_rng(5)
        T = rng.integers(-1, 2, size=(7, 23), dtype=np.int8)
        P = o.pack(fmt, T, ldp=16)
        P[3, 2] = bad_byte
        P[5, 0] = bad_byte
        rc, _, bad = o.unpack(fmt, P, 23)
        assert rc == 3 and bad == 3 * 16 + 2
        P2 = o.pack(fmt, T, ldp=16)
        P2[4, 10] = bad_byte  # past row_bytes: ignored
        assert o.unpack(fmt, P2, 23)[0] == 0


def pin_round_trip(o):
    """U(P(t)) = t for every K from 1 to 300 and odd strides; the tail is padded
    with 0-trits and bytes past row_bytes are zero."""
    rng = np.random.default_rng(11)
    for fmt, (g, b) in FMTS.items():
        for K in list(range(1, 40)) + [63, 64, 65, 79, 80, 81, 127, 128, 255, 256, 299, 300]:
            N = 1 + (K % 5)
            T = rng.integers(-1, 2, size=(N, K), dtype=np.int8)
            rb = -(-K // g)
            ldp = rb + (K % 3) * 7
            P = o.pack(fmt, T, ldp=ldp)
            assert (P[:, rb:] == 0).all()
            rc, T2, _ = o.unpack(fmt, P, K)
            assert rc == 0 and np.array_equal(T, T2), (fmt, K)
            # the pad trits are 0-trits: decoding the full last byte shows them
            rc, T3, _ = o.unpack(fmt, P[:, :rb], rb * g)
            assert rc == 0 and np.array_equal(T3[:, :K], T) and (T3[:, K:] == 0).all()
        # P(U(byte)) = byte for every valid byte (K a multiple of g)
        P = np.array([[v] for v in range(256)
                      if len(np.base_repr(v, b)) <= g and "3" not in np.base_repr(v, b)],
                     dtype=np.uint8)
        rc, T, _ = o.unpack(fmt, P, g)
        assert rc == 0 and np.array_equal(o.pack(fmt, T), P)


def pin_zero_rows(o):
    """A row of 0-trits is digit 1 everywhere: 0x55 per 2-bit byte (1111 in
    base 4) and 121 per 1.6-bit byte (11111 in base 3)."""
    assert int("1111", 4) == 0x55 and int("11111", 3) == 121
    for fmt, val in ((2, 0x55), (16, 121)):
        for K in (1, 2, 3, 4, 5, 6, 9, 10, 11):
            P = o.pack(fmt, np.zeros((2, K), dtype=np.int8))
            assert (P == val).all(), (fmt, K)


def pin_bad_trits(o):
    for fmt in FMTS:
        for v in (2, -2, 5, 127, -128):
            T = np.zeros((3, 7), dtype=np.int8)
            T[1, 4] = v
            assert o.pack_status(fmt, T) == 2


def pin_half(o):
    """The oracle's binary16 decoder equals numpy's for all 65536 patterns."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([o.half_to_double(int(h)) for h in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def _matmul_ref(T, X, alpha):
    return alpha * (X.astype(np.float64) @ T.astype(np.float64).T)


def pin_linear_matmul(o):
    """Against numpy's float64 matrix product on random shapes (ragged, M=1..8)."""
    rng = np.random.default_rng(3)
    for (M, N, K) in [(1, 1, 1), (1, 5, 7), (3, 4, 1), (8, 17, 33), (2, 64, 130),
                      (5, 3, 257), (1, 40, 1000), (16, 9, 31)]:
        T = rng.integers(-1, 2, size=(N, K), dtype=np.int8)
        X = rng.standard_normal((M, K)).astype(np.float16)
        alpha = float(rng.uniform(0.01, 2.0))
        Y = o.linear(T, X, alpha)
        R = _matmul_ref(T, X, alpha)
        assert Y.shape == (M, N)
        assert np.allclose(Y, R, rtol=1e-12, atol=1e-12), (M, N, K)


def pin_linear_bruteforce(o):
    """Every ternary T with N*K = 8 (3^8 = 6561 matrices per shape) against a
    dense einsum, on one fixed X."""
    rng = np.random.default_rng(8)
    all_t = np.array(list(itertools.product((-1, 0, 1), repeat=8)), dtype=np.int8)
    for (N, K) in ((1, 8), (2, 4), (4, 2), (8, 1)):
        X = rng.standard_normal((2, K)).astype(np.float16)
        Ts = all_t.reshape(-1, N, K)
        # stack every T as rows of one tall matrix: one oracle call per shape
        big = Ts.reshape(-1, K)
        Y = o.linear(big, X, 0.75)
        R = 0.75 * np.einsum("mk,rk->mr", X.astype(np.float64), big.astype(np.float64))
        assert np.allclose(Y, R, rtol=1e-12, atol=1e-13), (N, K)


def pin_linear_special(o):
    """Closed forms: T = 0 -> 0, T = I -> alpha x, T = -I -> -alpha x,
    permutation -> permuted alpha x, all-ones -> alpha * sum(x)."""
    rng = np.random.default_rng(21)
    for K in (1, 7, 64, 129):
        X = rng.standard_normal((3, K)).astype(np.float16)
        x64 = X.astype(np.float64)
        a = 0.02
        assert (o.linear(np.zeros((5, K), np.int8), X, a) == 0).all()
        eye = np.eye(K, dtype=np.int8)
        assert np.array_equal(o.linear(eye, X, a), a * x64)
        assert np.array_equal(o.linear(-eye, X, a), -a * x64)
        perm = rng.permutation(K)
        assert np.array_equal(o.linear(eye[perm], X, a), a * x64[:, perm])
        ones = np.ones((2, K), dtype=np.int8)
        Y = o.linear(ones, X, a)
        for m in range(3):
            s = math.fsum(x64[m])
            assert abs(Y[m, 0] - a * s) <= 1e-14 * max(1.0, abs(s)) and Y[m, 0] == Y[m, 1]


def pin_linear_threads_and_at(o):
    """Threaded evaluation and spot evaluation give the same numbers."""
    rng = np.random.default_rng(4)
    T = rng.integers(-1, 2, size=(37, 91), dtype=np.int8)
    X = rng.standard_normal((4, 91)).astype(np.float16)
    Y1 = o.linear(T, X, 0.3, nthreads=1)
    Y4 = o.linear(T, X, 0.3, nthreads=4)
    assert np.array_equal(Y1, Y4)
    ms = rng.integers(0, 4, size=50)
    ns = rng.integers(0, 37, size=50)
    assert np.array_equal(o.linear_at(T, X, 0.3, ms, ns), Y1[ms, ns])


ALL_PINS = [pin_fits, pin_row_bytes, pin_pack_positional, pin_unpack_all_bytes, pin_bad_index,
            pin_round_trip, pin_zero_rows, pin_bad_trits, pin_half, pin_linear_matmul,
            pin_linear_bruteforce, pin_linear_special, pin_linear_threads_and_at]


def failing_pins(o) -> list[str]:
    """Names of the pins that fail for oracle build `o`."""
    bad = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except AssertionError:
            bad.append(pin.__name__)
        except Exception as e:  # a mistake may also surface as an error
            bad.append(f"{pin.__name__}:{type(e).__name__}")
    return bad
