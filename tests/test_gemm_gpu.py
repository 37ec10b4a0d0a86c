"""tl_gemm (tcgen05 tensor-core kernel, M >= 16) on the GPU against the oracle,
for both storage formats (2-bit base 4, 1.6-bit base 3).

Tolerance (per element): |y - y_ref| <= 1e-3 * alpha * sum_k |x[m,k]| + ulp16(y_ref).
Small ragged shapes are compared in full; the batched/prefill shapes at full
size are compared on sampled outputs computed one by one by the oracle.
"""
import numpy as np
import pytest

import oracle
import synth
from layer_cases import check_against_oracle, make_case, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ternary_weight_03_b200 import build
    build.build()


SMALL = [(16, 128, 64), (16, 1, 1), (17, 130, 65), (32, 256, 128), (48, 200, 100),
         (64, 129, 1000), (100, 300, 257), (128, 128, 64), (200, 260, 640), (256, 384, 512),
         (300, 129, 1111), (513, 256, 320)]


FMTS = [2, 16]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", SMALL)
def test_small_ragged(fmt, M, N, K):
    T, X, a = make_case(fmt, M, N, K, seed=M * 7 + N + K, p0=[0.2, 1 / 3, 0.6][K % 3])
    Y, _ = run_layer(fmt, T, X, a, fn="tl_gemm", repeat=2)
    check_against_oracle(T, X, a, Y)


# Few output tiles: the kernel splits K over a cluster of 2 to 8 CTAs (2-bit:
# one K-step of 64 per rank at K = 256 / 200, uneven ranges at K = 520;
# 1.6-bit: whole 320-trit blocks, uneven at K = 2048 / 1000, one per rank at
# K = 2560) and reduces the partials in rank order, so repeated calls must
# agree bit for bit.
SPLIT_K = [(64, 1000, 2048), (256, 512, 256), (16, 640, 1000), (32, 300, 200),
           (128, 2048, 520), (512, 1024, 4096), (96, 129, 777), (16, 256, 2560),
           (32, 512, 3200)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", SPLIT_K)
def test_split_k(fmt, M, N, K):
    T, X, a = make_case(fmt, M, N, K, seed=M + 3 * N + 7 * K)
    Y, _ = run_layer(fmt, T, X, a, fn="tl_gemm", repeat=3)
    check_against_oracle(T, X, a, Y)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("extra", [(1, 0, 0), (0, 2, 0), (0, 0, 3)])
def test_strides(fmt, extra):
    T, X, a = make_case(fmt, 40, 200, 300, seed=5)
    Y, _ = run_layer(fmt, T, X, a, fn="tl_gemm", ldp_extra=extra[0], ldx_extra=extra[1],
                     ldy_extra=extra[2])
    check_against_oracle(T, X, a, Y)


@pytest.mark.parametrize("fmt", FMTS)
def test_special_matrices(fmt):
    K = 336  # 1.6-bit: a whole 320-trit block and a ragged one
    X = synth.activations(6, 32, K)
    a = 0.02
    Y, _ = run_layer(fmt, np.zeros((128, K), np.int8), X, a, fn="tl_gemm")
    assert (Y == 0).all()
    eye = np.eye(K, dtype=np.int8)
    for T in (eye, -eye, np.ones((130, K), np.int8), -np.ones((129, K), np.int8)):
        Y, _ = run_layer(fmt, T, X, a, fn="tl_gemm")
        check_against_oracle(T, X, a, Y)


def _sampled(fmt, M, N, K, seed, samples=3000):
    import torch
    import ternary_weight_03_b200 as tl
    T = synth.trits(seed, N, K)
    X = synth.activations(seed, M, K)
    a = synth.alpha_for(seed)
    dP = torch.from_numpy(tl.pack(fmt, T)).cuda()
    dX = torch.from_numpy(X).cuda()
    Y = tl.gemm(fmt, dP, a, dX, K).float().cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(seed)
    ms = rng.integers(0, M, samples)
    ns = rng.integers(0, N, samples)
    # always include the corners and the last rows / columns
    ms = np.concatenate([ms, [0, M - 1, 0, M - 1]])
    ns = np.concatenate([ns, [0, 0, N - 1, N - 1]])
    ref = oracle.get().linear_at(T, X, a, ms, ns)
    tol = oracle.tolerance(ref, X[ms], a)
    err = np.abs(Y[ms, ns] - ref)
    assert (err <= tol).all(), f"{int((err > tol).sum())} sampled outputs outside tolerance"
    assert np.isfinite(Y).all()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [16, 64, 256, 1024, 4096])
@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096), (4096, 4096)])
def test_prefill_shapes_sampled(fmt, M, K, N):
    _sampled(fmt, M, N, K, seed=M + K + fmt)


def test_formats_agree_without_split():
    """With one CTA per output tile (no split K) both formats run the same MMAs
    in the same order on the same exact -1 / 0 / +1 operands, so the 1.6-bit
    result must equal the 2-bit one bit for bit."""
    for M, N, K in [(256, 20480, 640), (300, 18944, 1111), (16, 38016, 333)]:
        T, X, a = make_case(2, M, N, K, seed=N + K)
        Y2, _ = run_layer(2, T, X, a, fn="tl_gemm")
        Y16, _ = run_layer(16, T, X, a, fn="tl_gemm")
        assert np.array_equal(Y2, Y16), (M, N, K)
