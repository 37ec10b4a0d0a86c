"""CPU oracle of the ternariser: fp16 weights W [N, K] -> trits T and a scale alpha.

TEST INFRASTRUCTURE ONLY: imported by the test suite and the benchmark's
CPU-baseline leg, never by the product.  It shares no code with the CUDA
path (numpy and Python integers only).

What the pages fix ("Pith review of Spectra 1.1: Scaling Laws and Efficient
Inference for Ternary Language Models", section "What carries the
argument"): the layer's weights are {-1, 0, 1} times one shared
floating-point scale, produced from latent full-precision weights by
rounding on the fly; the section listing the paper's domain assumptions
names that rounding as round-to-nearest ternary quantisation.  The pages do
not give the scale's formula, so these readings are taken:

  R-T1  alpha = the mean of |W| over the whole matrix, computed as
          S     = sum of |w| exactly: every binary16 magnitude is an integer
                  number of 2^-24 units, so S is an integer;
          alpha = fp32_rn( fp64_rn( fp64_rn(S) / (N K) ) * 2^-24 ).
        The sum is exact, so alpha does not depend on the summation order.
        Parity of this formula against the pages is unpinned (they give
        none); the tests pin that alpha is the exact mean within one fp32
        ulp and the invariances it must have.
  R-T2  q = fp32_rn(fp32(w) / alpha) and t is the nearest of {-1, 0, 1}
        to q, ties to the even value 0: t = +1 if q > 0.5, -1 if q < -0.5,
        else 0 (values beyond +-1.5 clip to +-1).  alpha = 0 (an all-zero
        W) gives t = 0 everywhere.  The decision is taken in fp32, the
        precision of the kernel; it equals the exact comparison of |w| / alpha
        with 1/2 (0.5 is an fp32 value and no fp32 alpha puts an fp16 w
        within rounding distance of it without being exactly 2 |w|), which a
        test checks with rational arithmetic.
  R-T3  W must be finite; NaN or Inf entries give unspecified results.

``mutant`` plants one known mistake (for the tests that show the pins catch
it); 0 is the oracle itself.
"""
from __future__ import annotations

import numpy as np

UNIT_EXP = 24  # |w| of a binary16 value is an integer multiple of 2^-24

MUTANTS = {
    1: "ties rounded away from zero",
    2: "scale is max |W| instead of the mean",
    3: "mean taken over one row (divides by K)",
    4: "signed mean (abs dropped)",
    5: "no clip: t = rint(q)",
}


def abs_units(W: np.ndarray) -> np.ndarray:
    """|w| of every entry as an exact int64 count of 2^-24 units."""
    W = np.asarray(W, dtype=np.float16)
    u = np.abs(W.astype(np.float64)) * float(2 ** UNIT_EXP)  # exact: fp16 -> fp64, x 2^24
    assert np.all(u == np.floor(u))
    return u.astype(np.int64)


def abs_sum_units(W: np.ndarray, mutant: int = 0) -> int:
    """S = sum |w| in 2^-24 units, as an exact Python integer (R-T1)."""
    W = np.asarray(W, dtype=np.float16)
    flat = W.reshape(-1)
    total = 0
    chunk = 1 << 20  # 2^20 entries x < 2^40 units stays far inside int64
    for i in range(0, flat.size, chunk):
        part = flat[i:i + chunk]
        if mutant == 4:
            u = (part.astype(np.float64) * float(2 ** UNIT_EXP)).astype(np.int64)
        else:
            u = abs_units(part)
        total += int(u.sum(dtype=np.int64))
    return total


def scale(W: np.ndarray, mutant: int = 0) -> np.float32:
    """alpha of R-T1."""
    W = np.asarray(W, dtype=np.float16)
    N, K = W.shape
    if mutant == 2:
        return np.float32(np.abs(W.astype(np.float64)).max()) if W.size else np.float32(0)
    S = abs_sum_units(W, mutant)
    count = K if mutant == 3 else N * K
    d = float(S) / float(count)  # int -> fp64 and the division both round to nearest
    d = d * 2.0 ** -UNIT_EXP     # exact scaling by a power of two
    return np.float32(d)


def quantise(W: np.ndarray, alpha: np.float32, mutant: int = 0) -> np.ndarray:
    """T of R-T2, int8 [N, K]."""
    W = np.asarray(W, dtype=np.float16)
    alpha = np.float32(alpha)
    if alpha == 0:
        return np.zeros(W.shape, dtype=np.int8)
    q = W.astype(np.float32) / alpha  # IEEE fp32 division, round to nearest
    T = np.zeros(W.shape, dtype=np.int8)
    if mutant == 5:
        return np.rint(q).astype(np.int8)
    if mutant == 1:
        T[q >= 0.5] = 1
        T[q <= -0.5] = -1
    else:
        T[q > 0.5] = 1
        T[q < -0.5] = -1
    return T


def ternarise(W: np.ndarray, mutant: int = 0):
    """(T int8 [N, K], alpha float32): the ternary weights and their shared scale."""
    alpha = scale(W, mutant)
    return quantise(W, alpha, mutant), alpha
