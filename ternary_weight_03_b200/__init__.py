"""Python binding of libternary (ctypes; argument marshalling only).

Every step of the layer runs inside ``libternary.so``: the host codec
(tl_pack2 / tl_pack16 / tl_unpack) and the sm_100a kernels (tl_gemv,
tl_gemm, tl_gemv_batch).  PyTorch is used only for device buffers and streams.  There is no
fallback: if the library is missing or a call fails, an exception is raised.

Functions take numpy arrays (host codec) or torch CUDA tensors (layer calls).
Activations and outputs are fp16; packed weights are uint8 [N, ldp].
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import numpy as np

PKG = Path(__file__).resolve().parent
LIB_PATH = PKG / "libternary.so"
DEBUG_LIB_PATH = PKG / "libternary_debug.so"

FMT_2BIT = 2
FMT_1P6BIT = 16
GEMV_MAX_M = 8
GEMM_MIN_M = 16

STATUS = {0: "TL_OK", 1: "TL_ERR_INVALID_ARG", 2: "TL_ERR_BAD_TRIT", 3: "TL_ERR_BAD_CODE",
          4: "TL_ERR_ALIGN", 5: "TL_ERR_CUDA", 6: "TL_ERR_TIMEOUT", 7: "TL_ERR_UNSUPPORTED"}

GEMV_BATCH_MAX = 4096
LAYER_READS_EARLIER = 1
LAYER_SWIGLU_INPUT = 2


class Layer(ctypes.Structure):
    """tl_gemv_layer: one layer of a tl_gemv_batch call (device pointers)."""
    _fields_ = [("dT", ctypes.c_void_p), ("ldp", ctypes.c_int64), ("alpha", ctypes.c_float),
                ("dX", ctypes.c_void_p), ("ldx", ctypes.c_int64), ("dY", ctypes.c_void_p),
                ("ldy", ctypes.c_int64), ("M", ctypes.c_int), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("flags", ctypes.c_uint)]


class Plan(ctypes.Structure):
    """tl_gemv_plan: a planned batch (filled by tl_gemv_batch_plan)."""
    _fields_ = [("fmt", ctypes.c_int), ("count", ctypes.c_int), ("max_m", ctypes.c_int),
                ("total_items", ctypes.c_int), ("total_tiles", ctypes.c_int),
                ("total_units", ctypes.c_int), ("chained", ctypes.c_int),
                ("dWorkspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("generation", ctypes.c_uint64)]


# (name, restype, argtypes) of every symbol the C header declares
_i64, _i32, _p, _f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_float
SIGNATURES = {
    "tl_status_str": (ctypes.c_char_p, [_i32]),
    "tl_last_cuda_error": (_i32, []),
    "tl_packed_row_bytes": (_i64, [_i32, _i64]),
    "tl_pack2": (_i32, [_p, _i64, _i64, _i64, _p, _i64]),
    "tl_pack16": (_i32, [_p, _i64, _i64, _i64, _p, _i64]),
    "tl_unpack": (_i32, [_i32, _p, _i64, _i64, _i64, _p, _i64, ctypes.POINTER(_i64)]),
    "tl_gemv": (_i32, [_i32, _p, _i64, _f32, _p, _i64, _p, _i64, _i32, _i64, _i64, _p]),
    "tl_gemv_ex": (_i32, [_i32, _p, _i64, _f32, _p, _i64, _p, _i64, _i32, _i64, _i64,
                          ctypes.c_uint, _p]),
    "tl_gemm": (_i32, [_i32, _p, _i64, _f32, _p, _i64, _p, _i64, _i32, _i64, _i64, _p]),
    "tl_gemv_batch_bytes": (_i32, [_i32, _i32, ctypes.POINTER(Layer),
                                   ctypes.POINTER(ctypes.c_size_t)]),
    "tl_gemv_batch_plan": (_i32, [_i32, _i32, ctypes.POINTER(Layer), _p, ctypes.c_size_t,
                                  ctypes.POINTER(Plan)]),
    "tl_gemv_batch_run": (_i32, [ctypes.POINTER(Plan), ctypes.c_uint, _p]),
    "tl_gemv_batch_plan_static": (_i32, [_i32, _i32, ctypes.POINTER(Layer), ctypes.POINTER(Plan)]),
    "tl_device_status": (_i32, [_p]),
    "tl_ternarise": (_i32, [_i32, _p, _i64, _i64, _i64, _p, _i64, _p, _p, _p]),
}


class TLError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda: int = 0):
        self.status = status
        msg = f"{fn} returned {STATUS.get(status, status)}"
        if cuda:
            msg += f" (cudaError {cuda})"
        super().__init__(msg)


_lib = None
_debug_lib = None


def _load(path: Path) -> ctypes.CDLL:
    if not path.exists():
        raise RuntimeError(f"{path.name} not found at {path}: run "
                           "`python -m ternary_weight_03_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(str(path))
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


def lib() -> ctypes.CDLL:
    """The loaded libternary.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


def debug_lib() -> ctypes.CDLL:
    """libternary_debug.so: the same entry points, plus the failure-detection
    hook TL_FLAG_DEBUG_DROP_ARRIVE of tl_gemv_batch_run.  Its device error word
    is its own (read it with its tl_device_status)."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _load(DEBUG_LIB_PATH)
    return _debug_lib


def _check(fn: str, rc: int):
    if rc != 0:
        raise TLError(fn, rc, lib().tl_last_cuda_error() if rc == 5 else 0)


def status_str(rc: int) -> str:
    return lib().tl_status_str(rc).decode()


def row_bytes(fmt: int, K: int) -> int:
    return int(lib().tl_packed_row_bytes(fmt, K))


def padded_ldp(fmt: int, K: int, align: int = 16) -> int:
    """The smallest legal device row stride: row bytes rounded up to 16."""
    rb = row_bytes(fmt, K)
    return max(align, (rb + align - 1) // align * align)


# -- host codec -----------------------------------------------------------------
def pack(fmt: int, T: np.ndarray, ldp: int | None = None, out: np.ndarray | None = None) -> np.ndarray:
    """Pack int8 trits [N, K] into uint8 [N, ldp] (ldp defaults to padded_ldp)."""
    T = np.ascontiguousarray(T, dtype=np.int8)
    N, K = T.shape
    ldp = padded_ldp(fmt, K) if ldp is None else ldp
    if out is None:
        out = np.empty((N, ldp), dtype=np.uint8)
    assert out.dtype == np.uint8 and out.flags.c_contiguous and out.shape == (N, ldp)
    fn = lib().tl_pack2 if fmt == FMT_2BIT else lib().tl_pack16
    if fmt not in (FMT_2BIT, FMT_1P6BIT):
        raise TLError("pack", 1)
    _check("tl_pack", fn(T.ctypes.data, N, K, K, out.ctypes.data, ldp))
    return out


def unpack(fmt: int, P: np.ndarray, K: int) -> np.ndarray:
    """Unpack uint8 [N, ldp] into int8 trits [N, K]; raises TLError on a bad code."""
    P = np.ascontiguousarray(P, dtype=np.uint8)
    N, ldp = P.shape
    T = np.empty((N, max(K, 1)), dtype=np.int8)
    bad = _i64(-1)
    rc = lib().tl_unpack(fmt, P.ctypes.data, N, K, ldp, T.ctypes.data, max(K, 1), ctypes.byref(bad))
    if rc != 0:
        err = TLError("tl_unpack", rc)
        err.bad_index = int(bad.value)
        raise err
    return T[:, :K]


# -- device layer ---------------------------------------------------------------
def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


FLAG_PDL = 1
FLAG_DEBUG_DROP_ARRIVE = 0x80000000  # debug library only


def _layer(fn_name: str, fmt: int, dT, alpha: float, X, K: int, out=None, stream=None, M=None,
           flags=None):
    import torch
    assert dT.is_cuda and dT.dtype == torch.uint8 and dT.dim() == 2
    assert X.is_cuda and X.dtype == torch.float16 and X.dim() == 2
    N, ldp = dT.shape
    M = X.shape[0] if M is None else M
    if out is None:
        out = torch.empty((M, N + (-N) % 8), dtype=torch.float16, device=X.device)
    assert out.is_cuda and out.dtype == torch.float16
    args = [fmt, dT.data_ptr(), dT.stride(0), float(alpha), X.data_ptr(), X.stride(0),
            out.data_ptr(), out.stride(0), M, N, K]
    if flags is not None:
        args.append(int(flags))
    rc = getattr(lib(), fn_name)(*args, _stream_ptr(stream))
    _check(fn_name, rc)
    return out[:, :N]


def gemv(fmt: int, dT, alpha: float, X, K: int, out=None, stream=None, flags: int = 0):
    """Y[M, N] = alpha * X T^T for 1 <= M <= 8 (decode-shaped).  flags=FLAG_PDL:
    programmatic dependent launch (dT must not be written by in-flight work)."""
    if flags:
        return _layer("tl_gemv_ex", fmt, dT, alpha, X, K, out, stream, flags=flags)
    return _layer("tl_gemv", fmt, dT, alpha, X, K, out, stream)


def gemm(fmt: int, dT, alpha: float, X, K: int, out=None, stream=None):
    """Y[M, N] = alpha * X T^T for M >= 16 (tensor-core GEMM)."""
    return _layer("tl_gemm", fmt, dT, alpha, X, K, out, stream)


def linear(fmt: int, dT, alpha: float, X, K: int, out=None, stream=None):
    """Dispatch on M: tl_gemv for M <= 8, two tl_gemv calls (8 + rest) for
    9 <= M <= 15, tl_gemm for M >= 16."""
    import torch
    M = X.shape[0]
    if M <= GEMV_MAX_M:
        return gemv(fmt, dT, alpha, X, K, out, stream)
    if M < GEMM_MIN_M:
        N = dT.shape[0]
        if out is None:
            out = torch.empty((M, N + (-N) % 8), dtype=torch.float16, device=X.device)
        gemv(fmt, dT, alpha, X[:GEMV_MAX_M], K, out[:GEMV_MAX_M], stream)
        gemv(fmt, dT, alpha, X[GEMV_MAX_M:], K, out[GEMV_MAX_M:], stream)
        return out[:, :N]
    return gemm(fmt, dT, alpha, X, K, out, stream)


def make_layers(fmt: int, specs) -> ctypes.Array:
    """ctypes array of tl_gemv_layer from (dT, alpha, X, K, Y[, flags]) tuples of
    torch CUDA tensors (dT uint8 [N, ldp]; X, Y fp16 with M rows)."""
    import torch
    arr = (Layer * len(specs))()
    for i, sp in enumerate(specs):
        dT, alpha, X, K, Y = sp[:5]
        flags = sp[5] if len(sp) > 5 else 0
        assert dT.is_cuda and dT.dtype == torch.uint8 and dT.dim() == 2
        assert X.is_cuda and X.dtype == torch.float16 and Y.dtype == torch.float16
        arr[i] = Layer(dT.data_ptr(), dT.stride(0), float(alpha), X.data_ptr(), X.stride(0),
                       Y.data_ptr(), Y.stride(0), X.shape[0], dT.shape[0], int(K), int(flags))
    return arr


def gemv_batch_bytes(fmt: int, layers) -> int:
    """Workspace bytes of a batch (a ctypes layer array from make_layers)."""
    n = ctypes.c_size_t(0)
    _check("tl_gemv_batch_bytes", lib().tl_gemv_batch_bytes(fmt, len(layers), layers,
                                                              ctypes.byref(n)))
    return int(n.value)


def gemv_batch_plan(fmt: int, layers, workspace) -> Plan:
    """Plan a batch into `workspace` (a CUDA uint8 tensor, 256-byte aligned, of
    at least gemv_batch_bytes bytes, kept alive by the caller).  Blocking."""
    plan = Plan()
    _check("tl_gemv_batch_plan",
           lib().tl_gemv_batch_plan(fmt, len(layers), layers, workspace.data_ptr(),
                                    workspace.numel() * workspace.element_size(),
                                    ctypes.byref(plan)))
    return plan


STATIC_WORKSPACE_BYTES = 16 << 20


def gemv_batch_plan_static(fmt: int, layers) -> Plan:
    """Plan a batch into the library's own per-device workspace (no caller
    memory, nothing allocated; one such plan per device at a time)."""
    plan = Plan()
    _check("tl_gemv_batch_plan_static",
           lib().tl_gemv_batch_plan_static(fmt, len(layers), layers, ctypes.byref(plan)))
    return plan


def gemv_batch_run(plan: Plan, stream=None, flags: int = 0):
    """Run a planned batch in one launch (asynchronous, graph-capturable)."""
    _check("tl_gemv_batch_run", lib().tl_gemv_batch_run(ctypes.byref(plan), int(flags),
                                                          _stream_ptr(stream)))


TERNARISE_WORKSPACE_BYTES = 16384


def ternarise(fmt: int, W, out=None, alpha=None, workspace=None, stream=None):
    """Ternarise and pack fp16 weights W [N, K] (CUDA, row stride a multiple of
    8) on the device: returns (P uint8 [N, ldp], alpha float32 [1]) with
    alpha = mean |W| and P the packed nearest trits of W / alpha."""
    import torch
    assert W.dtype == torch.float16 and W.dim() == 2 and W.stride(1) == 1
    N, K = W.shape
    if out is None:
        out = torch.empty((N, padded_ldp(fmt, K)), dtype=torch.uint8, device=W.device)
    if alpha is None:
        alpha = torch.empty(1, dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = torch.empty(TERNARISE_WORKSPACE_BYTES, dtype=torch.uint8, device=W.device)
    _check("tl_ternarise", lib().tl_ternarise(fmt, W.data_ptr(), W.stride(0), N, K,
                                              out.data_ptr(), out.stride(0), alpha.data_ptr(),
                                              workspace.data_ptr(), _stream_ptr(stream)))
    return out, alpha


def device_status(stream=None) -> int:
    return int(lib().tl_device_status(_stream_ptr(stream)))
