"""tl_gemv_ex with TL_FLAG_PDL: a call may start before the preceding kernel on
the stream finishes, so it must read its activations only after that kernel
completes.  A chain of dependent layers (layer 2 reads layer 1's output as X)
checks exactly that, eagerly and inside a CUDA graph.

Expected values: the oracle applied layer by layer, with the intermediate
rounded to binary16 as the GPU stores it.  The bound for layer 2 adds, to the
usual tolerance, alpha2 * sum_k ulp16(y1[k]): the GPU's y1 may differ from the
oracle's rounded y1 by one ulp per element.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ternary_weight_03_b200 import build
    build.build()


def _chain_reference(T1, T2, X, a1, a2):
    o = oracle.get()
    y1 = o.linear(T1, X, a1, nthreads=8).astype(np.float16)
    y2 = o.linear(T2, y1, a2, nthreads=8)
    tol = oracle.tolerance(y2, y1, a2)
    ulp = np.spacing(np.abs(y1).astype(np.float16)).astype(np.float64)
    tol = tol + abs(a2) * ulp.sum(axis=1)[:, None]
    return y2, tol


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("M,K,N", [(1, 3072, 3072), (8, 4096, 4096), (3, 1000, 1000)])
@pytest.mark.parametrize("graph", [False, True])
def test_dependent_chain(fmt, M, K, N, graph):
    import torch
    import ternary_weight_03_b200 as tl
    assert K == N  # layer 2 consumes layer 1's output
    T1 = synth.trits(11, N, K)
    T2 = synth.trits(12, N, N)
    X = synth.activations(13, M, K)
    a1, a2 = 0.02, 0.03
    dP1 = torch.from_numpy(tl.pack(fmt, T1)).cuda()
    dP2 = torch.from_numpy(tl.pack(fmt, T2)).cuda()
    dX = torch.from_numpy(X).cuda()
    ld = N + (-N) % 8
    Y1 = torch.full((M, ld), float("nan"), dtype=torch.float16, device="cuda")
    Y2 = torch.full((M, ld), float("nan"), dtype=torch.float16, device="cuda")
    s = torch.cuda.Stream()

    def run():
        tl.gemv(fmt, dP1, a1, dX, K, out=Y1, stream=s, flags=tl.FLAG_PDL)
        tl.gemv(fmt, dP2, a2, Y1, N, out=Y2, stream=s, flags=tl.FLAG_PDL)

    if graph:
        with torch.cuda.stream(s):
            run()  # per-device setup outside capture
            torch.cuda.synchronize()
            Y1.fill_(float("nan"))
            Y2.fill_(float("nan"))
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                run()
        for _ in range(3):
            Y1.fill_(float("nan"))
            Y2.fill_(float("nan"))
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
    else:
        for _ in range(3):
            run()
        torch.cuda.synchronize()
    ref, tol = _chain_reference(T1, T2, X, a1, a2)
    got = Y2[:, :N].float().cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= tol).all()
    assert tl.device_status(s) == 0

