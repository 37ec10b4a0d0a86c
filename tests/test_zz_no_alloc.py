"""tl_gemv_batch_plan_static: the batch planned into the library's own fixed
per-device array (no caller workspace, nothing allocated) gives the same bits
as the same batch planned into a caller workspace, on two different batches
planned one after the other (the second static plan replaces the first)."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ternary_weight_03_b200 import build
    build.build()


def _batch(fmt, shapes, seed):
    import torch
    import ternary_weight_03_b200 as tl
    specs = []
    for i, (M, N, K) in enumerate(shapes):
        P = tl.pack(fmt, synth.trits(seed + i, N, K))
        X = np.zeros((M, K + (-K) % 8), np.float16)
        X[:, :K] = synth.activations(seed + 50 + i, M, K)
        specs.append((torch.from_numpy(P).cuda(), synth.alpha_for(seed + i),
                      torch.from_numpy(X).cuda(), K,
                      torch.full((M, N + (-N) % 8), float("nan"), dtype=torch.float16,
                                 device="cuda")))
    return specs


def _outputs(specs):
    return [sp[4].cpu().numpy().view(np.uint16).copy() for sp in specs]


@pytest.mark.parametrize("fmt", [2, 16])
def test_static_workspace_matches_caller_workspace(fmt):
    import torch
    import ternary_weight_03_b200 as tl
    batches = [_batch(fmt, [(1, 1000, 4096), (8, 250, 14336), (3, 77, 700)], 400),
               _batch(fmt, [(2, 3072, 3072), (1, 129, 8200)], 500)]
    for specs in batches:
        layers = tl.make_layers(fmt, specs)
        assert tl.gemv_batch_bytes(fmt, layers) <= tl.STATIC_WORKSPACE_BYTES
        ws = torch.zeros(tl.gemv_batch_bytes(fmt, layers), dtype=torch.uint8, device="cuda")
        tl.gemv_batch_run(tl.gemv_batch_plan(fmt, layers, ws))
        assert tl.device_status() == 0
        want = _outputs(specs)
        plan = tl.gemv_batch_plan_static(fmt, layers)
        for _ in range(2):  # run again without clearing
            for sp in specs:
                sp[4].fill_(float("nan"))
            tl.gemv_batch_run(plan)
            assert tl.device_status() == 0
            for a, b in zip(want, _outputs(specs)):
                assert np.array_equal(a, b)


def test_replaced_static_plan_is_rejected():
    """A static plan made before a later tl_gemv_batch_plan_static describes a
    table that has since been overwritten: running it returns
    TL_ERR_INVALID_ARG without launching, and the newer plan still runs."""
    import ternary_weight_03_b200 as tl
    a = tl.make_layers(2, _batch(2, [(1, 500, 3000)], 600))
    b_specs = _batch(2, [(8, 130, 4100), (2, 77, 700)], 700)
    b = tl.make_layers(2, b_specs)
    plan_a = tl.gemv_batch_plan_static(2, a)
    plan_b = tl.gemv_batch_plan_static(2, b)
    assert plan_a.generation != 0 and plan_b.generation != plan_a.generation
    with pytest.raises(tl.TLError) as err:
        tl.gemv_batch_run(plan_a)
    assert err.value.status == 1
    tl.gemv_batch_run(plan_b)
    assert tl.device_status() == 0
    for sp in b_specs:
        assert not np.isnan(sp[4].float().cpu().numpy()[:, :sp[0].shape[0]]).any()


def test_static_workspace_rejects_oversized_batch():
    import ctypes
    import ternary_weight_03_b200 as tl
    A = 0x10000  # fake aligned device addresses: rejected before any device access
    # long rows split into many parts at M = 8: partial sums beyond the array
    n, k = 1 << 20, 1 << 16
    arr = (tl.Layer * 1)()
    arr[0] = tl.Layer(A, k // 4, 0.5, A, k, A, n, 8, n, k, 0)
    assert tl.gemv_batch_bytes(2, arr) > tl.STATIC_WORKSPACE_BYTES
    plan = tl.Plan()
    assert tl.lib().tl_gemv_batch_plan_static(2, 1, arr, ctypes.byref(plan)) == 1
