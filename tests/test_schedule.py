"""Host logic of the batch plan, on CPU: the work-item table that
tl_gemv_batch_plan writes, read through the debug library's
tl_debug_batch_items (include/tl_debug.h; no device is touched).

Pins: every tile's K-parts cover its stages exactly once; batches without
dependencies hand the costliest items out first; a dependent layer waits
for exactly the earlier layers whose Y overlaps its X (computed here
independently from the address ranges); layers on the same X share one
conversion; dependent fp16-engine layers convert once per launch; and no
dependent item is handed out before an item of a layer it reads.
"""
import ctypes

import numpy as np
import pytest

import ternary_weight_03_b200 as tl
from ternary_weight_03_b200 import build as tlbuild

ITEM = np.dtype([("X", "<u8"), ("Y", "<u8"), ("B", "<u8"), ("part_off", "<i8"),
                 ("alpha", "<f4"), ("layer", "<i4"), ("tile", "<i4"), ("part", "<i4"),
                 ("s0", "<i4"), ("s1", "<i4"), ("M", "<i4"), ("K", "<i4"), ("N", "<i4"),
                 ("ldx", "<i4"), ("ldy", "<i4"), ("parts", "<i4"), ("tile_begin", "<i4"),
                 ("deps", "<i4"), ("need", "<i4"), ("bstride", "<i4"), ("flags", "<i4"),
                 ("pad", "<i4", 3)])
assert ITEM.itemsize == 112

BASE = 1 << 32  # fake, 256-byte aligned device addresses: compared, never read
RE, SW = 1, 2   # TL_LAYER_READS_EARLIER, TL_LAYER_SWIGLU_INPUT


@pytest.fixture(scope="module")
def D():
    tlbuild.build()
    lib = tl.debug_lib()
    lib.tl_debug_batch_items.restype = ctypes.c_int
    lib.tl_debug_batch_items.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.POINTER(ctypes.c_int)]
    return lib


def layer(fmt, M, N, K, X, Y, ldx=None, ldy=None, flags=0):
    g = 4 if fmt == 2 else 5
    rb = -(-K // g)
    return dict(dT=BASE + (1 << 30), ldp=rb + (-rb) % 16, alpha=0.5, dX=X,
                ldx=ldx if ldx is not None else K + (-K) % 8, dY=Y,
                ldy=ldy if ldy is not None else N + (-N) % 8, M=M, N=N, K=K, flags=flags)


def items(D, fmt, specs):
    arr = (tl.Layer * len(specs))()
    for i, d in enumerate(specs):
        arr[i] = tl.Layer(**d)
    n = ctypes.c_int(0)
    assert D.tl_debug_batch_items(fmt, len(specs), arr, None, 0, ctypes.byref(n)) == 0
    out = np.zeros(n.value, dtype=ITEM)
    assert D.tl_debug_batch_items(fmt, len(specs), arr, out.ctypes.data, out.nbytes,
                                  ctypes.byref(n)) == 0
    assert n.value == len(out)
    return out


def stages(fmt, K):
    return -(-(-(-K // (4 if fmt == 2 else 5))) // 128)


def overlap_range(specs, l):
    """Earlier layers whose Y bytes overlap layer l's X bytes: (lo, hi) or None."""
    d = specs[l]
    x0 = d["dX"]
    x1 = x0 + 2 * ((d["M"] - 1) * d["ldx"] + (2 * d["K"] if d["flags"] & SW else d["K"]))
    hits = [j for j in range(l)
            if specs[j]["dY"] < x1 and x0 < specs[j]["dY"] + 2 * ((specs[j]["M"] - 1) *
                                                                  specs[j]["ldy"] + specs[j]["N"])]
    return (hits[0], hits[-1]) if hits else None


def check_cover(fmt, specs, it):
    """Every (layer, tile) is split into K-parts that cover its stages once."""
    for l, d in enumerate(specs):
        mine = it[(it["layer"] & 0xFFFF) == l]
        tiles = -(-d["N"] // 256)
        assert sorted(set(mine["tile"])) == list(range(tiles)), l
        for t in range(tiles):
            parts = np.sort(mine[mine["tile"] == t], order="part")
            assert list(parts["part"]) == list(range(len(parts)))
            assert (parts["parts"] == len(parts)).all()
            assert parts["s0"][0] == 0 and parts["s1"][-1] == stages(fmt, d["K"])
            assert (parts["s0"][1:] == parts["s1"][:-1]).all()
            assert (parts["s1"] > parts["s0"]).all()


def fused_block(fmt, M, base, F=8192, H=3072):
    """One decoder block as the bench's fused step lays it out."""
    X0, X1, XF, GU = base, base + 0x100000, base + 0x200000, base + 0x300000
    Ys = [base + 0x400000 + 0x100000 * i for i in range(5)]
    return [layer(fmt, M, H, H, X0, Ys[0]), layer(fmt, M, H, H, X0, Ys[1]),
            layer(fmt, M, H, H, X0, Ys[2]), layer(fmt, M, H, H, X1, Ys[3]),
            layer(fmt, M, F, H, XF, GU, ldy=2 * F), layer(fmt, M, F, H, XF, GU + 2 * F, ldy=2 * F),
            layer(fmt, M, H, F, GU, Ys[4], ldx=2 * F, flags=RE | SW)]


@pytest.mark.parametrize("fmt", [2, 16])
def test_independent_batch_covers_and_orders(D, fmt):
    specs = [layer(fmt, M, N, K, BASE + 0x1000000 * i, BASE + 0x1000000 * i + 0x800000)
             for i, (M, N, K) in enumerate([(1, 3072, 3072), (8, 8192, 3072), (1, 3072, 8192),
                                            (3, 4096, 4096), (2, 14336, 4096), (8, 4096, 14336),
                                            (1, 130, 700), (5, 1, 1)])]
    it = items(D, fmt, specs)
    check_cover(fmt, specs, it)
    assert (it["deps"] == 0).all() and (it["flags"] == 0).all()
    sc = lambda M: 1 if M <= 2 else (2 if fmt == 2 else 3)
    cost = [(r["s1"] - r["s0"]) * sc(r["M"]) + (r["M"] * ((r["parts"] + 3) // 4) if r["parts"] > 1 else 0)
            for r in it]
    assert all(a >= b for a, b in zip(cost, cost[1:])), "costliest first"
    # fp16-engine items keep at least 8 stages where the layer has them
    for r in it[it["M"] > 2]:
        if stages(fmt, int(r["K"])) >= 8:
            assert r["s1"] - r["s0"] >= 4


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("M", [1, 8])
def test_fused_step_dependencies(D, fmt, M):
    specs = []
    for b in range(3):
        specs += fused_block(fmt, M, BASE + 0x10000000 * b)
    it = items(D, fmt, specs)
    check_cover(fmt, specs, it)
    order = {}
    for pos, r in enumerate(it):
        order.setdefault(int(r["layer"]) & 0xFFFF, []).append(pos)
    for l, d in enumerate(specs):
        mine = it[(it["layer"] & 0xFFFF) == l]
        rng = overlap_range(specs, l)
        if d["flags"] & RE:
            # the down projection reads exactly its own block's gate and up
            assert rng == (l - 2, l - 1)
            assert (mine["deps"] == ((rng[0] << 16) | (rng[1] + 1))).all()
            assert (mine["flags"] & 1).all(), "SwiGLU input"
            coop = M > 2
            assert ((mine["flags"] & 2) != 0).all() == coop
            assert ((mine["B"] != 0).all()) == coop
            if coop:
                st = stages(fmt, d["K"])
                assert (mine["need"] == st * M).all()
            # handed out after every item of the layers it reads
            assert min(order[l]) > max(order[rng[0]] + order[rng[1]])
        else:
            assert rng is None and (mine["deps"] == 0).all()
    # Q, K and V share the first one's conversion of X
    for b in range(3):
        q = 7 * b
        for l in (q, q + 1, q + 2):
            mine = it[(it["layer"] & 0xFFFF) == l]
            assert ((mine["layer"] >> 16) == q).all()
            assert len(set(mine["B"])) == 1
        assert it[(it["layer"] & 0xFFFF) == q]["B"][0] == it[(it["layer"] & 0xFFFF) == q + 1]["B"][0]
        assert ((it[(it["layer"] & 0xFFFF) == q + 3]["layer"] >> 16) == q + 3).all()


@pytest.mark.parametrize("fmt", [2, 16])
def test_interleaved_chains_and_layers_without_producer(D, fmt):
    M = 2
    A0, A1 = BASE, BASE + 0x100000
    bufA, bufB = BASE + 0x200000, BASE + 0x300000
    gu = BASE + 0x400000
    specs = [layer(fmt, M, 1000, 3000, A0, bufA),                              # a0
             layer(fmt, M, 2000, 3000, A1, bufB, ldy=2504),                    # b0
             layer(fmt, M, 700, 1000, bufA, BASE + 0x500000, flags=RE),        # a1 <- a0
             layer(fmt, M, 900, 2500, bufB, BASE + 0x600000, ldx=2504, flags=RE),  # b1 <- b0
             layer(fmt, 5, 600, 800, gu, BASE + 0x700000, ldx=1600, flags=RE | SW),  # no producer
             layer(fmt, M, 300, 500, BASE + 0x500000, BASE + 0x800000, flags=RE)]  # <- a1 only
    it = items(D, fmt, specs)
    check_cover(fmt, specs, it)
    want = {2: (0, 0), 3: (1, 1), 4: None, 5: (2, 2)}
    for l, rng in want.items():
        assert overlap_range(specs, l) == rng
        mine = it[(it["layer"] & 0xFFFF) == l]
        assert (mine["deps"] == (0 if rng is None else (rng[0] << 16) | (rng[1] + 1))).all(), l
    no_prod = it[(it["layer"] & 0xFFFF) == 4]
    assert (no_prod["flags"] == 3).all(), "SwiGLU, converted once (M = 5)"
    assert (it[(it["layer"] & 0xFFFF) == 2]["flags"] == 0).all(), "M = 2: converted on chip"
    assert (it[(it["layer"] & 0xFFFF) == 2]["B"] == 0).all()


def test_hook_rejects_like_plan(D):
    bad = (tl.Layer * 1)()
    bad[0] = tl.Layer(**layer(2, 9, 100, 100, BASE, BASE + 0x100000))  # M > 8
    n = ctypes.c_int(0)
    assert D.tl_debug_batch_items(2, 1, bad, None, 0, ctypes.byref(n)) == 1
    first_dep = (tl.Layer * 1)()
    first_dep[0] = tl.Layer(**layer(2, 1, 100, 100, BASE, BASE + 0x100000, flags=RE))
    assert D.tl_debug_batch_items(2, 1, first_dep, None, 0, ctypes.byref(n)) == 1
    assert not hasattr(tl.lib(), "tl_debug_batch_items"), "product library exports no hook"


def test_debug_header_symbols_are_exported(D):
    import re
    from pathlib import Path
    text = Path(tlbuild.INCLUDE / "tl_debug.h").read_text()
    names = re.findall(r"^\s*int\s+(tl_\w+)\(", text, flags=re.M)
    assert names == ["tl_debug_batch_items"]
    for name in names:
        assert hasattr(D, name), name
