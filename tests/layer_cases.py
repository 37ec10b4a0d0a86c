"""Helpers of the GPU parity tests: build one layer case from seeded inputs,
run it through the C ABI, and compare with the oracle."""
from __future__ import annotations

import numpy as np

import oracle
import synth
import ternary_weight_03_b200 as tl


def make_case(fmt, M, N, K, seed=0, p0=1 / 3, alpha=None, T=None, X=None):
    """Trits, activations and scale of one case (numpy, host)."""
    if T is None:
        T = synth.trits(seed, N, K, p0=p0)
    if X is None:
        X = synth.activations(seed, M, K)
    a = synth.alpha_for(seed, alpha)
    return T, X, a


def run_layer(fmt, T, X, alpha, fn="tl_gemv", ldp_extra=0, ldx_extra=0, ldy_extra=0,
              pad_byte=0xFF, repeat=1):
    """Pack with the product codec, upload, call tl_gemv / tl_gemm via ctypes.

    Padding bytes of each packed row, activations past K and outputs past N
    are filled with junk (0xFF bytes, NaN) to show they are never used or
    written.  Returns (Y [M, N] float64, full Y buffer as float16 numpy).
    """
    import torch
    N, K = T.shape
    M = X.shape[0]
    ldp = tl.padded_ldp(fmt, K) + 16 * ldp_extra
    P = tl.pack(fmt, T, ldp=ldp)
    rb = tl.row_bytes(fmt, K)
    P[:, rb:] = pad_byte
    ldx = K + (-K) % 8 + 8 * ldx_extra
    Xh = np.full((M, ldx), np.nan, dtype=np.float16)
    Xh[:, :K] = X
    ldy = N + (-N) % 8 + 8 * ldy_extra
    dP = torch.from_numpy(P).cuda()
    dX = torch.from_numpy(Xh).cuda()
    outs = []
    for _ in range(repeat):
        dY = torch.full((M + 1, ldy), float("nan"), dtype=torch.float16, device="cuda")
        rc = getattr(tl.lib(), fn)(fmt, dP.data_ptr(), ldp, float(alpha), dX.data_ptr(), ldx,
                                   dY.data_ptr(), ldy, M, N, K,
                                   torch.cuda.current_stream().cuda_stream)
        assert rc == 0, f"{fn} -> {tl.status_str(rc)}"
        torch.cuda.synchronize()
        outs.append(dY.cpu().numpy())
    for o in outs[1:]:
        assert np.array_equal(o.view(np.uint16), outs[0].view(np.uint16)), "not deterministic"
    Yfull = outs[0]
    # nothing written outside [0, M) x [0, N)
    assert np.isnan(Yfull[M, :].astype(np.float32)).all(), "wrote past row M"
    if ldy > N:
        assert np.isnan(Yfull[:M, N:].astype(np.float32)).all(), "wrote past column N"
    return Yfull[:M, :N].astype(np.float64), Yfull


def check_against_oracle(T, X, alpha, Y, nthreads=8):
    ref = oracle.get().linear(T, X, alpha, nthreads=nthreads)
    tol = oracle.tolerance(ref, X, alpha)
    err = np.abs(Y - ref)
    bad = ~(err <= tol)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"got {Y[tuple(i)]}, ref {ref[tuple(i)]}, tol {tol[tuple(i)]}")
    return float((err / tol).max()) if err.size else 0.0
