"""The C ABI library loads and exports every symbol of include/tl.h, and the
host-side argument rules reject bad calls before anything reaches a GPU."""
import re
from pathlib import Path

import pytest

import ternary_weight_03_b200 as tl
from ternary_weight_03_b200 import build as tlbuild

HEADER = Path(__file__).resolve().parent.parent / "include" / "tl.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tl_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    tlbuild.build()
    return tl.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "tl_gemv" in names and "tl_pack2" in names
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(tl.SIGNATURES), "binding and header disagree"


def test_only_the_c_abi_is_exported(L):
    """Both libraries export nothing but tl_* symbols: no C++ function-local
    static (process-unique symbol) is shared between two of them loaded into
    one process."""
    import shutil
    import subprocess
    if shutil.which("readelf") is None:
        pytest.skip("readelf not available")
    for lib in (tlbuild.LIB, tlbuild.DEBUG_LIB):
        out = subprocess.run(["readelf", "--dyn-syms", "-W", str(lib)], check=True,
                             capture_output=True, text=True).stdout
        defined = []
        for line in out.splitlines():
            f = line.split()
            if len(f) >= 8 and f[0][:-1].isdigit() and f[6] != "UND":
                defined.append((f[4], f[7]))
        assert defined, lib
        bad = [d for d in defined if not d[1].startswith("tl_") or d[0] == "UNIQUE"]
        assert not bad, f"{lib.name} exports {bad[:5]}"


def test_status_strings(L):
    for code, name in tl.STATUS.items():
        assert tl.status_str(code).startswith(name)
    assert tl.status_str(99) == "unknown tl status"


def test_row_bytes(L):
    assert tl.row_bytes(2, 1024) == 256 and tl.row_bytes(2, 1025) == 257
    assert tl.row_bytes(16, 1024) == 205 and tl.row_bytes(16, 5) == 1
    assert tl.row_bytes(3, 10) == -1 and tl.row_bytes(2, -1) == -1
    assert tl.padded_ldp(16, 1024) == 208


A = 0x10000  # fake, 16-byte aligned device addresses (never dereferenced)


def gemv_rc(L, fmt=2, dT=A, ldp=256, dX=A, ldx=1024, dY=A, ldy=1024, M=1, N=1024, K=1024,
            fn="tl_gemv"):
    return getattr(L, fn)(fmt, dT, ldp, 0.5, dX, ldx, dY, ldy, M, N, K, None)


@pytest.mark.parametrize("kw,rc", [
    (dict(fmt=3), 1), (dict(dT=0), 1), (dict(dX=0), 1), (dict(dY=0), 1),
    (dict(M=0), 1), (dict(M=9), 1), (dict(N=0), 1), (dict(K=0), 1), (dict(K=-5), 1),
    (dict(ldp=255), 1), (dict(ldx=1016), 1), (dict(ldy=1000), 1),
    (dict(dT=A + 8), 4), (dict(dX=A + 2), 4), (dict(dY=A + 4), 4),
    (dict(ldp=272, K=1024), 0), (dict(ldp=264), 4), (dict(ldx=1028), 4), (dict(ldy=1028), 4),
    (dict(fmt=16, ldp=204), 1), (dict(fmt=16, ldp=200), 1),
])
def test_gemv_argument_rules(L, kw, rc):
    if rc == 0:
        pytest.skip("valid arguments would launch a kernel (GPU test)")
    assert gemv_rc(L, **kw) == rc


def test_gemm_argument_rules(L):
    assert gemv_rc(L, fn="tl_gemm", M=15) == 1
    assert gemv_rc(L, fn="tl_gemm", M=0) == 1
    assert gemv_rc(L, fn="tl_gemm", M=64, dX=A + 2) == 4
    assert gemv_rc(L, fn="tl_gemm", M=64, ldp=128) == 1


def test_build_flags_target_sm100a():
    flags = " ".join(tlbuild.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags and "-lineinfo" in flags


def test_gemv_ex_flags(L):
    assert gemv_rc(L, fn="tl_gemv", M=0) == 1
    A_ = 0x10000
    # unknown flag bits are rejected before anything reaches a device
    assert L.tl_gemv_ex(2, A_, 256, 1.0, A_, 1024, A_, 1024, 1, 1024, 1024, 2, None) == 1
    assert L.tl_gemv_ex(2, A_, 256, 1.0, A_, 1024, A_, 1024, 9, 1024, 1024, 1, None) == 1


def _layers(specs):
    """ctypes layers with fake, aligned device addresses (never dereferenced)."""
    arr = (tl.Layer * len(specs))()
    for i, sp in enumerate(specs):
        d = dict(dT=A, ldp=256, alpha=0.5, dX=A, ldx=1024, dY=A, ldy=1024, M=1, N=1024, K=1024,
                 flags=0)
        d.update(sp)
        arr[i] = tl.Layer(**d)
    return arr


def _ws(L, fmt, arr):
    import ctypes
    n = ctypes.c_size_t(0)
    rc = L.tl_gemv_batch_bytes(fmt, len(arr), arr, ctypes.byref(n))
    return rc, n.value


def _up(v):
    return (v + 255) // 256 * 256


def _ws_expected(layers, fmt=2):
    """Batch workspace, region by region (each rounded up to 256 bytes):
    counters, one 128-byte tensor map per layer, a 112-byte record per work item
    (256-row tile x K-part of 2..16 stages of 128 packed bytes per row: 512
    trits at 2 bits, 640 at 1.6 bits), a 48-byte record per conversion unit
    (stage x token of a layer that reads no earlier output), a u32 per tile,
    four u32 per layer (ready units, final tiles, tiles, claimed units),
    8-byte partials of split tiles, and the converted activations of layers
    that read no earlier output and of dependent layers with M > 2, which
    convert once during the launch (per stage 64 bytes plus one
    byte per trit and column of 8 per token (M = 1, 2) or two bytes per trit
    and token rounded up to even (M >= 3)).  A layer with a dependency has its
    items sized to spread it over about 148 CTAs (at most 8 parts per tile, 2
    for M > 2).  Independent layers with the same X (pointer, ldx, K, M) share
    the first one's conversion (no units or converted activations of their
    own)."""
    items = units = tiles = slots = staged = 0
    g = 4 if fmt == 2 else 5  # trits per byte
    stg = lambda d: -(-(-(-d["K"] // g)) // 128)
    # relative cost of a stage: fp16 engine x2 (2-bit) or x3 (base 3)
    cm = lambda d: 1 if d["M"] <= 2 else (2 if fmt == 2 else 3)
    total = sum(stg(d) * -(-d["N"] // 256) * cm(d) for d in layers)
    cost = min(16, max(4, total // ((3 if fmt == 2 else 4) * 148)))  # cost per item
    seen = set()
    for d in layers:
        stages = stg(d)
        if d.get("flags", 0):
            target = -(-stages * -(-d["N"] // 256) // 148)
            min_t = -(-stages // (2 if d["M"] > 2 else 8))
            target = max(target, min_t, 1)
        else:
            target = max(1, cost // cm(d))
            if d["M"] > 2:
                target = max(target, 8)
        parts = max(1, min(stages, (stages + target // 2) // target))
        t = -(-d["N"] // 256)
        items += t * parts
        tiles += t
        key = (d.get("dX", A), d.get("ldx", d["K"] + (-d["K"]) % 8), d["K"], d["M"])
        b = 8 * 128 * g * d["M"] if d["M"] <= 2 else 2 * 128 * g * (d["M"] + d["M"] % 2)
        if not d.get("flags", 0) and key not in seen:
            seen.add(key)
            units += stages * d["M"]
            staged += stages * (64 + b)
        elif d.get("flags", 0) and d["M"] > 2:
            staged += stages * (64 + b)
        if parts > 1:
            slots += t * parts * 256 * d["M"]
    off = 256
    for size in (128 * len(layers), 112 * items, 48 * units, 16 * len(layers), 4 * tiles, 8 * slots,
                 staged):
        off = _up(off + size)
    return off


def test_batch_workspace_size(L):
    base = dict(M=1, flags=0)
    cases = [[dict(base, N=1000, K=2048)], [dict(base, N=4096, K=14336)],
             [dict(base, N=4096, K=14336, M=8)], [dict(base, N=4096, K=14336, M=2)],
             [dict(base, N=130, K=700, M=3), dict(base, N=77, K=5000, M=1, flags=1)],
             [dict(base, N=14336, K=4096)] * 12, [dict(base, N=3072, K=8192, M=8)] * 80,
             [dict(base, N=3072, K=3072), dict(base, N=8192, K=3072, flags=1),
              dict(base, N=3072, K=8192, flags=1), dict(base, N=3072, K=8192, M=8, flags=1)],
             # Q, K, V on one X (one conversion), O on its own X, gate and up on a
             # third X, the down projection reading silu(gate) * up
             [dict(base, N=3072, K=3072, M=2)] * 3 + [dict(base, N=3072, K=3072, M=2, dX=A + 65536)]
             + [dict(base, N=8192, K=3072, M=2, dX=A + 131072)] * 2
             + [dict(base, N=3072, K=8192, M=2, flags=3, ldx=16384)]]
    for fmt, g in ((2, 4), (16, 5)):
        for ls in cases:
            arr = _layers([dict(d, ldp=(d["K"] + g - 1) // g + (-((d["K"] + g - 1) // g)) % 16,
                                ldx=d.get("ldx", d["K"] + (-d["K"]) % 8),
                                ldy=d["N"] + (-d["N"]) % 8) for d in ls])
            rc, n = _ws(L, fmt, arr)
            assert rc == 0 and n == _ws_expected(ls, fmt), (fmt, ls, n)


@pytest.mark.parametrize("spec,count,rc", [
    (dict(M=0), 1, 1), (dict(M=9), 1, 1), (dict(flags=2), 1, 1), (dict(flags=1), 1, 1),
    (dict(dT=0), 1, 1), (dict(ldp=255), 1, 1), (dict(dX=A + 2), 1, 4), (dict(ldy=1028), 1, 4),
    (dict(), 0, 1), (dict(), 4097, 1),
])
def test_batch_argument_rules(L, spec, count, rc):
    arr = _layers([spec] * max(count, 1))
    import ctypes
    n = ctypes.c_size_t(0)
    plan = tl.Plan()
    assert L.tl_gemv_batch_bytes(2, count, arr, ctypes.byref(n)) == rc
    assert L.tl_gemv_batch_plan(2, count, arr, A, 1 << 20, ctypes.byref(plan)) == rc


@pytest.mark.parametrize("fmt,second,rc", [
    (2, dict(flags=3, ldx=2048), 0),                 # [gate | up] rows of 2K elements
    (2, dict(flags=2, ldx=2048), 1),                 # SwiGLU input needs READS_EARLIER
    (2, dict(flags=3, ldx=1024), 1),                 # rows shorter than 2K
    (2, dict(flags=3, K=1020, ldx=2048, ldp=256), 4),  # up half not 16-byte aligned
    (2, dict(flags=4), 1),                           # unknown flag
    (16, dict(flags=3, ldx=2048), 0),                # 1.6-bit batch too
    (16, dict(flags=3, ldx=1024), 1),
])
def test_swiglu_input_rules(L, fmt, second, rc):
    import ctypes
    first = dict(ldp=256 if fmt == 2 else 208)
    arr = _layers([first, dict(first, **second)])
    n = ctypes.c_size_t(0)
    assert L.tl_gemv_batch_bytes(fmt, 2, arr, ctypes.byref(n)) == rc


def test_batch_plan_and_run_rules(L):
    import ctypes
    arr = _layers([dict(), dict(flags=1)])  # layer 1 may read layer 0's output
    rc, n = _ws(L, 2, arr)
    assert rc == 0
    plan = tl.Plan()
    pp = ctypes.byref(plan)
    assert L.tl_gemv_batch_plan(2, 2, arr, 0, n, pp) == 1          # no workspace
    assert L.tl_gemv_batch_plan(2, 2, arr, A + 16, n, pp) == 4     # not 256-byte aligned
    assert L.tl_gemv_batch_plan(2, 2, arr, A, n - 1, pp) == 1      # too small
    assert L.tl_gemv_batch_plan(3, 2, arr, A, n, pp) == 1          # unknown format
    assert L.tl_gemv_batch_plan(2, 2, arr, A, n, None) == 1        # no plan
    # run refuses a plan that tl_gemv_batch_plan did not fill
    assert L.tl_gemv_batch_run(None, 0, None) == 1
    assert L.tl_gemv_batch_run(pp, 0, None) == 1
    bad = tl.Plan(fmt=2, count=2, max_m=9, total_items=3, total_tiles=2, dWorkspace=A,
                  workspace_bytes=n)
    assert L.tl_gemv_batch_run(ctypes.byref(bad), 0, None) == 1
    good = tl.Plan(fmt=2, count=2, max_m=1, total_items=3, total_tiles=2, dWorkspace=A,
                   workspace_bytes=n)
    assert L.tl_gemv_batch_run(ctypes.byref(good), 8, None) == 1   # unknown flag
    bad_units = tl.Plan(fmt=2, count=2, max_m=1, total_items=3, total_tiles=2, total_units=-1,
                        dWorkspace=A, workspace_bytes=n)
    assert L.tl_gemv_batch_run(ctypes.byref(bad_units), 0, None) == 1


def ternarise_rc(L, fmt=2, dW=A, ldw=1024, N=64, K=1024, dP=A, ldp=256, dAlpha=A, ws=A):
    return L.tl_ternarise(fmt, dW, ldw, N, K, dP, ldp, dAlpha, ws, None)


@pytest.mark.parametrize("kw,rc", [
    (dict(fmt=4), 1), (dict(dW=0), 1), (dict(dP=0), 1), (dict(dAlpha=0), 1), (dict(ws=0), 1),
    (dict(N=0), 1), (dict(K=0), 1), (dict(N=-1), 1), (dict(N=2 ** 31), 1),
    (dict(ldw=1016), 1), (dict(ldp=240), 1), (dict(fmt=16, ldp=192), 1), (dict(ldp=2 ** 32), 1),
    (dict(dW=A + 8), 4), (dict(dP=A + 4), 4), (dict(ws=A + 8), 4), (dict(dAlpha=A + 2), 4),
    (dict(ldw=1028), 4), (dict(ldp=264), 4),
])
def test_ternarise_argument_rules(L, kw, rc):
    assert ternarise_rc(L, **kw) == rc


def test_ternarise_workspace_constant():
    text = HEADER.read_text()
    m = re.search(r"#define TL_TERNARISE_WORKSPACE_BYTES (\d+)u", text)
    assert m and int(m.group(1)) == tl.TERNARISE_WORKSPACE_BYTES
