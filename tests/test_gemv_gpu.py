"""tl_gemv on the GPU against the oracle (parity tests proper).

Tolerance (per element): |y - y_ref| <= 1e-3 * alpha * sum_k |x[m,k]| + ulp16(y_ref),
y_ref the oracle's double-precision value of alpha * sum_k T[n,k] x[m,k].
"""
import numpy as np
import pytest

import synth
from layer_cases import check_against_oracle, make_case, run_layer

pytestmark = pytest.mark.gpu

FMTS = (2, 16)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ternary_weight_03_b200 import build
    build.build()


SMALL = [(1, 1, 1), (1, 7, 5), (2, 15, 63), (3, 16, 64), (8, 31, 255), (5, 30, 256),
         (1, 45, 257), (8, 46, 319), (4, 61, 320), (6, 100, 321), (7, 64, 1000),
         (8, 129, 1025), (1, 200, 2047), (2, 33, 5000)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", SMALL)
def test_small_ragged(fmt, M, N, K):
    T, X, a = make_case(fmt, M, N, K, seed=N * 1000 + K, p0=[0.2, 1 / 3, 0.6][K % 3])
    Y, _ = run_layer(fmt, T, X, a, repeat=2)
    check_against_oracle(T, X, a, Y)


# Rows longer than one cluster of the single-layer kernel stages (2-bit
# K > 16384, 1.6-bit K > 20480) go to the register-streaming kernel: ragged N,
# K with a tail inside a byte, both token extremes, junk padding, repeat calls.
LONG_K = [(2, 1, 300, 20000), (2, 8, 77, 20000), (2, 3, 129, 40001),
          (16, 1, 300, 24000), (16, 8, 77, 24000), (16, 5, 33, 65537)]


@pytest.mark.parametrize("fmt,M,N,K", LONG_K)
def test_long_rows(fmt, M, N, K):
    T, X, a = make_case(fmt, M, N, K, seed=K + N, p0=[0.2, 1 / 3, 0.6][N % 3])
    Y, _ = run_layer(fmt, T, X, a, ldx_extra=1, repeat=2)
    check_against_oracle(T, X, a, Y)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("extra", [(1, 0, 0), (0, 2, 0), (0, 0, 3), (2, 1, 1)])
def test_strides(fmt, extra):
    T, X, a = make_case(fmt, 3, 77, 700, seed=9)
    Y, _ = run_layer(fmt, T, X, a, ldp_extra=extra[0], ldx_extra=extra[1], ldy_extra=extra[2])
    check_against_oracle(T, X, a, Y)


@pytest.mark.parametrize("fmt", FMTS)
def test_special_matrices(fmt):
    K = 300
    X = synth.activations(4, 8, K)
    a = 0.02
    x64 = X.astype(np.float64)
    # zero matrix -> exactly zero
    Y, _ = run_layer(fmt, np.zeros((50, K), np.int8), X, a)
    assert (Y == 0).all()
    # identity, negative identity, permutation -> alpha * x within the tolerance
    eye = np.eye(K, dtype=np.int8)
    for T, ref in ((eye, a * x64), (-eye, -a * x64)):
        Y, _ = run_layer(fmt, T, X, a)
        check_against_oracle(T, X, a, Y)
        assert np.abs(Y - ref).max() <= np.abs(ref).max() * 2 ** -10
    perm = np.random.default_rng(1).permutation(K)
    Y, _ = run_layer(fmt, eye[perm], X, a)
    check_against_oracle(eye[perm], X, a, Y)
    # all ones -> alpha * sum x
    ones = np.ones((20, K), np.int8)
    Y, _ = run_layer(fmt, ones, X, a)
    check_against_oracle(ones, X, a, Y)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("p0", [0.2, 0.33, 0.6])
def test_sparsity(fmt, p0):
    T, X, a = make_case(fmt, 8, 300, 3072, seed=17, p0=p0)
    Y, _ = run_layer(fmt, T, X, a)
    check_against_oracle(T, X, a, Y)


def test_config1_full():
    """K = N = 1024, M = 1, 2-bit, uniform trits, alpha = 0.02, seed 0."""
    T, X, a = make_case(2, 1, 1024, 1024, seed=0, alpha=0.02)
    Y, _ = run_layer(2, T, X, a, repeat=3)
    check_against_oracle(T, X, a, Y)


SWEEP = [(3072, 3072), (3072, 8192), (8192, 3072), (4096, 4096), (4096, 14336), (14336, 4096)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 8])
@pytest.mark.parametrize("K,N", SWEEP)
def test_sweep_shapes_full(fmt, M, K, N):
    """Every output of the decode-sweep shapes (full sizes), one seed per shape."""
    T, X, a = make_case(fmt, M, N, K, seed=SWEEP.index((K, N)))
    Y, _ = run_layer(fmt, T, X, a)
    check_against_oracle(T, X, a, Y, nthreads=16)


def test_large_magnitudes():
    """Activations near the fp16 range still accumulate within tolerance."""
    K, N = 2048, 64
    rng = np.random.default_rng(3)
    X = (rng.standard_normal((2, K)) * 3000).astype(np.float16)
    T = synth.trits(3, N, K)
    for fmt in FMTS:
        Y, _ = run_layer(fmt, T, X, 1e-4)
        check_against_oracle(T, X, 1e-4, Y)
