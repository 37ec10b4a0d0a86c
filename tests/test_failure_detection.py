"""Failure detection without a GPU fault.

Every wait inside the kernels is bounded (1 s of wall time); a wait that runs
out sets the device error word, the kernel gives up its work and exits
cleanly, and tl_device_status reports TL_ERR_TIMEOUT.  The debug library
(libternary_debug.so, the product sources compiled with TL_DEBUG_HOOKS) can
leave out one software barrier arrival in the 2-bit batch kernel
(TL_FLAG_DEBUG_DROP_ARRIVE), which makes exactly such a wait run out.  No
hardware completion (TMA byte count) is ever skipped, so nothing is in flight
when the kernel exits.  The product library rejects the flag.
"""
import ctypes
import time

import numpy as np
import pytest

import oracle
import synth
import ternary_weight_03_b200 as tl
from ternary_weight_03_b200 import build as tlbuild

TL_ERR_INVALID_ARG = 1
TL_ERR_CUDA = 5
TL_ERR_TIMEOUT = 6


@pytest.fixture(scope="module")
def libs():
    tlbuild.build()
    return tl.lib(), tl.debug_lib()


def test_status_codes_match_header():
    assert tl.STATUS[TL_ERR_INVALID_ARG] == "TL_ERR_INVALID_ARG"
    assert tl.STATUS[TL_ERR_CUDA] == "TL_ERR_CUDA"
    assert tl.STATUS[TL_ERR_TIMEOUT] == "TL_ERR_TIMEOUT"


def test_debug_library_exports_the_same_entry_points(libs):
    for L in libs:
        for name in tl.SIGNATURES:
            assert hasattr(L, name), name


def test_product_library_rejects_the_hook(libs):
    """The hook bit is an invalid flag for the product library, and is
    accepted by the debug one (which then goes on to the device checks: with
    no CUDA device here that is TL_ERR_CUDA).  The plan is a fake, so this
    runs only without a device."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only argument check (the plan here is not a real plan)")
    prod, dbg = libs
    plan = tl.Plan()
    plan.fmt, plan.count, plan.max_m = 2, 1, 1
    plan.total_items, plan.total_tiles, plan.total_units = 1, 1, 0
    plan.chained, plan.dWorkspace, plan.workspace_bytes, plan.generation = 0, 256, 4096, 0
    flag = tl.FLAG_DEBUG_DROP_ARRIVE
    assert prod.tl_gemv_batch_run(ctypes.byref(plan), flag, None) == TL_ERR_INVALID_ARG
    assert dbg.tl_gemv_batch_run(ctypes.byref(plan), flag, None) == TL_ERR_CUDA
    assert dbg.tl_gemv_batch_run(ctypes.byref(plan), flag | 2, None) == TL_ERR_INVALID_ARG


def _debug_plan(D, layers, ws):
    plan = tl.Plan()
    rc = D.tl_gemv_batch_plan(2, len(layers), layers, ws.data_ptr(), ws.numel(),
                              ctypes.byref(plan))
    assert rc == 0, tl.status_str(rc)
    return plan


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [(1, 200, 1000), (2, 256, 2000)])
def test_dropped_arrival_times_out_then_recovers(libs, M, N, K):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    prod, D = libs
    T = synth.trits(900 + M, N, K)
    X = synth.activations(910 + M, M, K)
    a = synth.alpha_for(920 + M)
    dP = torch.from_numpy(tl.pack(2, T)).cuda()
    dX = torch.from_numpy(X).cuda()
    dY = torch.full((M, N + (-N) % 8), float("nan"), dtype=torch.float16, device="cuda")
    layers = tl.make_layers(2, [(dP, a, dX, K, dY)])
    n = ctypes.c_size_t(0)
    assert D.tl_gemv_batch_bytes(2, 1, layers, ctypes.byref(n)) == 0
    ws = torch.full((n.value,), 0xAB, dtype=torch.uint8, device="cuda")
    plan = _debug_plan(D, layers, ws)
    # one item (one row tile, one K-part): CTA 0 converts its stages on chip
    assert plan.total_items == 1 and plan.total_tiles == 1
    stream = torch.cuda.current_stream().cuda_stream
    assert D.tl_device_status(stream) == 0

    t0 = time.monotonic()
    assert D.tl_gemv_batch_run(ctypes.byref(plan), tl.FLAG_DEBUG_DROP_ARRIVE, stream) == 0
    assert D.tl_device_status(stream) == TL_ERR_TIMEOUT
    elapsed = time.monotonic() - t0
    assert elapsed < 20.0, f"the bounded waits took {elapsed:.1f} s"
    # the status read clears the word; the context is still usable
    assert D.tl_device_status(stream) == 0
    assert torch.cuda.is_available() and torch.zeros(4, device="cuda").sum().item() == 0.0
    # the product library's error word is its own and untouched
    assert tl.device_status() == 0

    # after a timeout the batch is planned again; the next normal run is correct
    plan = _debug_plan(D, layers, ws)
    dY.fill_(float("nan"))
    assert D.tl_gemv_batch_run(ctypes.byref(plan), 0, stream) == 0
    assert D.tl_device_status(stream) == 0
    got = dY[:, :N].float().cpu().numpy().astype(np.float64)
    ref = oracle.get().linear(T, X, a)
    tol = oracle.tolerance(ref, X, a)
    assert (np.abs(got - ref) <= tol).all()
    # and the product library still runs the same layer the same way
    ws_p = torch.zeros_like(ws)
    plan_p = tl.gemv_batch_plan(2, layers, ws_p)
    dY2 = dY.clone()
    dY.fill_(float("nan"))
    tl.gemv_batch_run(plan_p)
    assert tl.device_status() == 0
    assert torch.equal(dY.view(torch.int16), dY2.view(torch.int16))
