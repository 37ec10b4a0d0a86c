"""Pins of the ternariser oracle (oracle/ternarise.py) against what the
definition and the mathematics fix, independently of the oracle's own steps:
exact rational arithmetic (Python fractions) for the scale and the nearest
trit, closed forms, special cases and invariances.  Every planted mistake in
the oracle must fail at least one pin.

The pages give the form (ternary weights times one shared scale, rounding
to the nearest ternary value: "Pith review of Spectra 1.1", "What carries the
argument" and the domain assumptions it lists) but no formula for the scale;
the scale pin therefore checks the stated reading (mean |W|), not the pages.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import ternarise as tz


def _fp16_matrix(seed, N, K, kind="normal"):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        W = rng.standard_normal((N, K)) * 0.02
    elif kind == "wide":  # magnitudes from fp16 subnormals up to 1e4
        W = rng.standard_normal((N, K)) * np.exp2(rng.uniform(-26, 13, (N, K)))
    elif kind == "sparse":
        W = rng.standard_normal((N, K)) * (rng.random((N, K)) < 0.3)
    else:
        raise ValueError(kind)
    return W.astype(np.float16)


def _ulp32(x):
    x = abs(float(x))
    return float(np.spacing(np.float32(x)))


def _exact_mean(W):
    flat = W.astype(np.float64).reshape(-1)
    return sum((abs(Fraction(float(v))) for v in flat), Fraction(0)) / flat.size


# ---- pins: each returns a list of failure strings ---------------------------
def pin_scale_is_mean(m):
    bad = []
    for seed, (N, K), kind in [(1, (3, 7), "normal"), (2, (5, 33), "wide"), (3, (8, 40), "sparse"),
                               (4, (1, 1), "normal"), (5, (16, 5), "wide")]:
        W = _fp16_matrix(seed, N, K, kind)
        _, a = tz.ternarise(W, m)
        exact = _exact_mean(W)
        if abs(Fraction(float(a)) - exact) > Fraction(_ulp32(exact)):
            bad.append(f"alpha {float(a)!r} vs exact mean {float(exact)!r} ({kind} {N}x{K})")
    return bad


def pin_nearest_trit(m):
    """t is the nearest of {-1, 0, 1} to w / alpha in exact arithmetic, ties to 0."""
    bad = []
    for seed, (N, K), kind in [(6, (4, 50), "normal"), (7, (6, 20), "wide"), (8, (3, 64), "sparse")]:
        W = _fp16_matrix(seed, N, K, kind)
        T, a = tz.ternarise(W, m)
        A = Fraction(float(a))
        for (n, k), w in np.ndenumerate(W.astype(np.float64)):
            r = Fraction(float(w)) / A
            dist = {t: abs(r - t) for t in (-1, 0, 1)}
            best = min(dist.values())
            cands = [t for t in (-1, 0, 1) if dist[t] == best]
            want = 0 if 0 in cands else cands[0]
            if T[n, k] != want:
                bad.append(f"w={w!r} alpha={float(a)!r}: t={T[n, k]} want {want}")
                break
    return bad


def pin_closed_forms(m):
    bad = []
    rng = np.random.default_rng(9)
    # W = c * T0 with T0 in {-1, 1}: alpha = c exactly, T = T0
    for c in (0.25, 0.0137, 3.5, 6.1e-5):
        T0 = rng.choice(np.array([-1, 1], np.int8), size=(4, 9))
        W = (np.float16(c) * T0.astype(np.float16)).astype(np.float16)
        T, a = tz.ternarise(W, m)
        if a != np.float32(np.float16(c)) or not np.array_equal(T, T0):
            bad.append(f"c * T0, c={c}: alpha={float(a)!r}")
    # fewer than a third zeros: q = +-1 / (1 - f) < 1.5, so T = T0
    T0 = rng.choice(np.array([-1, 0, 1], np.int8), size=(6, 30), p=[0.4, 0.2, 0.4])
    W = (np.float16(0.5) * T0.astype(np.float16)).astype(np.float16)
    T, _ = tz.ternarise(W, m)
    if not np.array_equal(T, T0):
        bad.append("c * T0 with 20% zeros not recovered")
    # ties: W = [3, 1] has alpha = 2 and q = [1.5, 0.5] -> [1, 0]
    W = np.array([[3, 1], [-3, -1], [1, 3]], np.float16)
    T, a = tz.ternarise(W, m)
    if a != 2 or not np.array_equal(T, np.array([[1, 0], [-1, 0], [0, 1]], np.int8)):
        bad.append(f"tie case: alpha={float(a)!r} T={T.tolist()}")
    # zero matrix
    T, a = tz.ternarise(np.zeros((3, 5), np.float16), m)
    if a != 0 or T.any():
        bad.append("zero matrix")
    return bad


def pin_invariances(m):
    bad = []
    rng = np.random.default_rng(10)  # magnitudes in [0.01, 2): scaling by 2^j stays exact
    W = (rng.choice([-1.0, 1.0], (7, 23)) * rng.uniform(0.01, 2.0, (7, 23))).astype(np.float16)
    T, a = tz.ternarise(W, m)
    Tn, an = tz.ternarise(-W, m)
    if an != a or not np.array_equal(Tn, -T):
        bad.append("negation")
    for j in (1, 3, -2):  # exact in fp16 for these magnitudes
        Ws = (W.astype(np.float64) * 2.0 ** j).astype(np.float16)
        assert np.array_equal(Ws.astype(np.float64), W.astype(np.float64) * 2.0 ** j)
        Tj, aj = tz.ternarise(Ws, m)
        if aj != np.float32(a * np.float32(2.0 ** j)) or not np.array_equal(Tj, T):
            bad.append(f"scaling by 2^{j}")
    perm = np.random.default_rng(11).permutation(W.size)
    Wp = W.reshape(-1)[perm].reshape(W.shape)
    Tp, ap = tz.ternarise(Wp, m)
    if ap != a or not np.array_equal(Tp, T.reshape(-1)[perm].reshape(W.shape)):
        bad.append("permutation")
    return bad


PINS = [pin_scale_is_mean, pin_nearest_trit, pin_closed_forms, pin_invariances]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_passes(pin):
    assert pin(0) == []


@pytest.mark.parametrize("mutant", sorted(tz.MUTANTS), ids=lambda m: tz.MUTANTS[m])
def test_mutant_is_caught(mutant):
    assert any(pin(mutant) for pin in PINS), f"mutant {mutant} passed every pin"


def test_abs_units_are_exact():
    """Every binary16 magnitude is an integer number of 2^-24 units (all 63488
    finite bit patterns)."""
    bits = np.arange(0, 0x7C00, dtype=np.uint16)
    v = bits.view(np.float16)
    u = tz.abs_units(v.reshape(1, -1))[0]
    assert all(Fraction(int(x), 2 ** 24) == abs(Fraction(float(f))) for x, f in zip(u[::97], v[::97]))
    assert u.max() == 65504 * 2 ** 24
