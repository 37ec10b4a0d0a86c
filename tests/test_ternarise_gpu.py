"""tl_ternarise (device ternariser + packer) against the CPU oracle
(oracle/ternarise.py for the scale and the trits, the oracle's packer for the
bytes).  Both the scale alpha and every packed byte must match bit for bit:
the scale is an exact integer sum rounded by fixed steps, and the trit
decision is a comparison both sides take on the same fp32 values.
"""
import numpy as np
import pytest

import oracle
from oracle import ternarise as tz

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ternary_weight_03_b200 import build
    build.build()


def _weights(seed, N, K, kind):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        W = rng.standard_normal((N, K)) * 0.02
    elif kind == "wide":  # binary16 subnormals up to ~1e4
        W = rng.standard_normal((N, K)) * np.exp2(rng.uniform(-26, 13, (N, K)))
    elif kind == "sparse":
        W = rng.standard_normal((N, K)) * (rng.random((N, K)) < 0.3)
    elif kind == "ties":  # many entries exactly at alpha / 2: rows of [3, 1, 3, 1, ...]
        W = np.tile(np.array([3.0, 1.0]), (N, (K + 1) // 2))[:, :K] * rng.choice([-1, 1], (N, 1))
    else:
        raise ValueError(kind)
    return W.astype(np.float16)


def _run(fmt, W, ldw_extra=0, ldp_extra=0):
    import torch
    import ternary_weight_03_b200 as tl
    N, K = W.shape
    ldw = K + (-K) % 8 + 8 * ldw_extra
    Wd = torch.full((N, ldw), float("nan"), dtype=torch.float16)  # junk past K
    Wd[:, :K] = torch.from_numpy(W)
    Wd = Wd.cuda()
    ldp = tl.padded_ldp(fmt, K) + 16 * ldp_extra
    P = torch.full((N, ldp), 0xEE, dtype=torch.uint8, device="cuda")
    alpha = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.full((tl.TERNARISE_WORKSPACE_BYTES,), 0xAB, dtype=torch.uint8, device="cuda")
    tl.ternarise(fmt, Wd[:, :K], out=P, alpha=alpha, workspace=ws)
    torch.cuda.synchronize()
    return P.cpu().numpy(), np.float32(alpha.item())


def _expect(fmt, W, ldp):
    O = oracle.get()
    T, a = tz.ternarise(W)
    P = O.pack(fmt, T, ldp=ldp)
    P[:, O.row_bytes(fmt, W.shape[1]):] = 0
    return P, a


SHAPES = [(1, 1), (2, 7), (3, 16), (3, 20), (4, 33), (5, 100), (7, 333), (64, 1111),
          (300, 4096), (129, 5000), (1, 70000)]


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("kind", ["normal", "wide", "sparse", "ties"])
def test_matches_oracle(fmt, N, K, kind):
    W = _weights(N * 31 + K, N, K, kind)
    P, a = _run(fmt, W)
    Pref, aref = _expect(fmt, W, P.shape[1])
    assert a.view(np.uint32) == aref.view(np.uint32), (float(a), float(aref))
    assert np.array_equal(P, Pref)


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("extra", [(1, 0), (0, 2), (3, 1)])
def test_strides(fmt, extra):
    W = _weights(5, 37, 203, "normal")
    P, a = _run(fmt, W, ldw_extra=extra[0], ldp_extra=extra[1])
    Pref, aref = _expect(fmt, W, P.shape[1])
    assert a == aref and np.array_equal(P, Pref)


@pytest.mark.parametrize("fmt", [2, 16])
def test_zero_matrix(fmt):
    W = np.zeros((9, 50), np.float16)
    W[::2] = -0.0
    P, a = _run(fmt, W)
    assert a == 0
    Pref, _ = _expect(fmt, W, P.shape[1])
    assert np.array_equal(P, Pref)


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("N,K", [(4096, 14336), (14336, 4096)])
def test_full_size(fmt, N, K):
    """The largest layer shapes of the decode sweep, compared in full."""
    W = _weights(N + K, N, K, "normal")
    P, a = _run(fmt, W)
    Pref, aref = _expect(fmt, W, P.shape[1])
    assert a == aref and np.array_equal(P, Pref)


def test_packed_output_feeds_the_layer():
    """tl_ternarise's bytes and alpha drive tl_gemv directly: y matches the
    oracle's layer on the oracle's trits and scale."""
    import torch
    import ternary_weight_03_b200 as tl
    import synth
    N, K = 1000, 3000
    W = _weights(77, N, K, "normal")
    Wd = torch.from_numpy(W).cuda()
    P, alpha = tl.ternarise(2, Wd)
    X = synth.activations(3, 4, K)
    Y = tl.gemv(2, P, float(alpha.item()), torch.from_numpy(X).cuda(), K)
    T, a = tz.ternarise(W)
    ref = oracle.get().linear(T, X, float(a))
    tol = oracle.tolerance(ref, X, float(a))
    assert (np.abs(Y.float().cpu().numpy().astype(np.float64) - ref) <= tol).all()
