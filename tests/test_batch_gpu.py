"""tl_gemv_batch_plan / tl_gemv_batch_run (one persistent launch over many
decode-shaped layers) on the GPU against the oracle, layer by layer.

Tolerance per element, as for tl_gemv: |y - y_ref| <= 1e-3 * alpha *
sum_k |x[m,k]| + ulp16(y_ref).  Chained layers (TL_LAYER_READS_EARLIER) are
checked against the oracle applied layer by layer on the intermediate as the
GPU stores it (binary16), the bound adding alpha * sum_k ulp16(x_k) for the
one-ulp freedom of each stored intermediate.
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


def _device_layer(fmt, T, X, ldp_extra=0, ldx_extra=0, ldy_extra=0):
    """Upload one layer with junk in every padding byte / element (0xFF codes,
    NaN activations, NaN outputs) and one guard row below Y."""
    import torch
    import ternary_weight_03_b200 as tl
    N, K = T.shape
    M = X.shape[0]
    ldp = tl.padded_ldp(fmt, K) + 16 * ldp_extra
    P = tl.pack(fmt, T, ldp=ldp)
    P[:, tl.row_bytes(fmt, K):] = 0xFF
    ldx = K + (-K) % 8 + 8 * ldx_extra
    Xh = np.full((M, ldx), np.nan, dtype=np.float16)
    Xh[:, :K] = X
    ldy = N + (-N) % 8 + 8 * ldy_extra
    dY = torch.full((M + 1, ldy), float("nan"), dtype=torch.float16, device="cuda")
    return torch.from_numpy(P).cuda(), torch.from_numpy(Xh).cuda(), dY


def _check_layer(T, X, a, dY, N, M):
    Y = dY.cpu().numpy()
    assert np.isnan(Y[M, :].astype(np.float32)).all(), "wrote past row M"
    if Y.shape[1] > N:
        assert np.isnan(Y[:M, N:].astype(np.float32)).all(), "wrote past column N"
    got = Y[:M, :N].astype(np.float64)
    ref = oracle.get().linear(T, X, a, nthreads=8)
    tol = oracle.tolerance(ref, X, a)
    err = np.abs(got - ref)
    assert (err <= tol).all(), f"{int((err > tol).sum())} of {err.size} outside tolerance"


def _plan(fmt, layers):
    """Workspace + plan of a batch (the workspace must outlive the plan)."""
    import torch
    import ternary_weight_03_b200 as tl
    nbytes = tl.gemv_batch_bytes(fmt, layers)
    ws = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")  # junk: plan clears
    return tl.gemv_batch_plan(fmt, layers, ws), ws


def _counters_zero(ws):
    return not ws[:256].cpu().numpy().any()


# (M, N, K, p0): ragged N and K (tails inside a byte, a group and a K-part),
# single rows and columns, long rows split into many K-parts
MIXED = [(1, 1, 1, 1 / 3), (3, 7, 5, 0.2), (8, 121, 255, 0.6), (2, 250, 257, 1 / 3),
         (1, 240, 1000, 1 / 3), (5, 130, 2049, 0.2), (1, 300, 4100, 1 / 3), (8, 64, 14336, 1 / 3),
         (1, 1000, 3072, 0.6), (4, 129, 8200, 1 / 3)]
# short batches whose M = 8 layer has a partial last stage and wraps the ring
SHORT = [[(1, 500, 3000), (8, 130, 4100), (3, 77, 700)], [(8, 130, 4100)],
         [(8, 250, 4100), (8, 130, 1025)]]


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("shapes", SHORT)
def test_short_batches(fmt, shapes):
    import ternary_weight_03_b200 as tl
    cases, specs = [], []
    for i, (M, N, K) in enumerate(shapes):
        T = synth.trits(700 + i, N, K)
        X = synth.activations(710 + i, M, K)
        a = synth.alpha_for(720 + i)
        dP, dX, dY = _device_layer(fmt, T, X)
        cases.append((T, X, a, dY, N, M))
        specs.append((dP, a, dX, K, dY))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    tl.gemv_batch_run(plan)
    assert tl.device_status() == 0
    for T, X, a, dY, N, M in cases:
        _check_layer(T, X, a, dY, N, M)


@pytest.mark.parametrize("fmt", [2, 16])
def test_mixed_independent_layers(fmt):
    import ternary_weight_03_b200 as tl
    cases, specs = [], []
    for i, (M, N, K, p0) in enumerate(MIXED):
        T = synth.trits(100 + i, N, K, p0=p0)
        X = synth.activations(200 + i, M, K)
        a = synth.alpha_for(300 + i)
        dP, dX, dY = _device_layer(fmt, T, X, ldp_extra=i % 2, ldx_extra=i % 3, ldy_extra=i % 2)
        cases.append((T, X, a, dP, dX, dY))
        specs.append((dP, a, dX, K, dY))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    outs = []
    for rep in range(3):  # the plan is run again without clearing anything
        for c in cases:
            c[5].fill_(float("nan"))
        tl.gemv_batch_run(plan)
        assert tl.device_status() == 0
        outs.append([c[5].cpu().numpy().view(np.uint16).copy() for c in cases])
        assert _counters_zero(ws), "workspace counters not reset"
    for r in outs[1:]:
        for a_, b_ in zip(outs[0], r):
            assert np.array_equal(a_, b_), "not deterministic"
    for (T, X, a, dP, dX, dY), (M, N, K, _) in zip(cases, MIXED):
        _check_layer(T, X, a, dY, N, M)


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("graph", [False, True])
def test_chain_reads_earlier(fmt, graph):
    """Layer i + 1 reads layer i's output (TL_LAYER_READS_EARLIER), under PDL."""
    import torch
    import ternary_weight_03_b200 as tl
    M = 3
    dims = [3072, 1000, 4096, 257, 2048]  # K of layer 0, then each layer's N
    Ts = [synth.trits(40 + i, dims[i + 1], dims[i]) for i in range(len(dims) - 1)]
    X0 = synth.activations(50, M, dims[0])
    alphas = [0.02, 0.03, 0.015, 0.05]
    import ternary_weight_03_b200 as tl
    dX0 = torch.from_numpy(X0).cuda()
    ys = [torch.full((M, d + (-d) % 8), float("nan"), dtype=torch.float16, device="cuda")
          for d in dims[1:]]
    specs = []
    for i, T in enumerate(Ts):
        dP = torch.from_numpy(tl.pack(fmt, T)).cuda()
        X = dX0 if i == 0 else ys[i - 1]
        specs.append((dP, alphas[i], X, dims[i], ys[i], 0 if i == 0 else tl.LAYER_READS_EARLIER))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        tl.gemv_batch_run(plan, stream=s, flags=tl.FLAG_PDL)
        torch.cuda.synchronize()
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                tl.gemv_batch_run(plan, stream=s, flags=tl.FLAG_PDL)
                tl.gemv_batch_run(plan, stream=s, flags=tl.FLAG_PDL)
            for y in ys:
                y.fill_(float("nan"))
            torch.cuda.synchronize()
            g.replay()
        else:
            for y in ys:
                y.fill_(float("nan"))
            torch.cuda.synchronize()
            for _ in range(2):
                tl.gemv_batch_run(plan, stream=s, flags=tl.FLAG_PDL)
    torch.cuda.synchronize()
    assert tl.device_status(s) == 0
    o = oracle.get()
    x = X0
    for i, T in enumerate(Ts):
        N = dims[i + 1]
        got = ys[i][:, :N].float().cpu().numpy().astype(np.float64)
        ref = o.linear(T, x, alphas[i], nthreads=8)
        tol = oracle.tolerance(ref, x, alphas[i])
        if i > 0:
            ulp = np.spacing(np.abs(x).astype(np.float16)).astype(np.float64)
            tol = tol + abs(alphas[i]) * ulp.sum(axis=1)[:, None]
        assert (np.abs(got - ref) <= tol).all(), f"layer {i}"
        x = ys[i][:, :N].cpu().numpy()  # the stored intermediate feeds the next reference


@pytest.mark.parametrize("fmt", [2, 16])
def test_sweep_batch_sampled(fmt):
    """The decode sweep's six matrices at M = 1 and 8 as one 12-layer batch;
    sampled outputs per layer against the oracle computed one by one."""
    import torch
    import ternary_weight_03_b200 as tl
    sweep = [(3072, 3072), (3072, 8192), (8192, 3072), (4096, 4096), (4096, 14336),
             (14336, 4096)]
    specs, cases = [], []
    for M in (1, 8):
        for i, (K, N) in enumerate(sweep):
            T = synth.trits(i, N, K)
            X = synth.activations(10 * M + i, M, K)
            a = synth.alpha_for(i)
            dP = torch.from_numpy(tl.pack(fmt, T)).cuda()
            dX = torch.from_numpy(X).cuda()
            dY = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
            specs.append((dP, a, dX, K, dY))
            cases.append((T, X, a, dY))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
    assert tl.device_status() == 0
    rng = np.random.default_rng(fmt)
    o = oracle.get()
    for T, X, a, dY in cases:
        Y = dY.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(Y).all()
        M, N = Y.shape
        ms = np.concatenate([rng.integers(0, M, 400), [0, M - 1]])
        ns = np.concatenate([rng.integers(0, N, 400), [0, N - 1]])
        ref = o.linear_at(T, X, a, ms, ns)
        tol = oracle.tolerance(ref, X[ms], a)
        assert (np.abs(Y[ms, ns] - ref) <= tol).all()


def test_batch_matches_single_calls():
    """Every layer of a batch equals tl_gemv's result within the tolerance of
    both, and the batch is bit-identical across calls."""
    import torch
    import ternary_weight_03_b200 as tl
    specs, singles, cases = [], [], []
    for i, (M, N, K) in enumerate([(1, 512, 4096), (8, 360, 1536), (2, 1000, 700)]):
        T = synth.trits(60 + i, N, K)
        X = synth.activations(70 + i, M, K)
        dP = torch.from_numpy(tl.pack(2, T)).cuda()
        Xp = np.zeros((M, K + (-K) % 8), np.float16)  # row stride a multiple of 8
        Xp[:, :K] = X
        dX = torch.from_numpy(Xp).cuda()
        dY = torch.empty((M, N + (-N) % 8), dtype=torch.float16, device="cuda")
        specs.append((dP, 0.02, dX, K, dY))
        singles.append(tl.gemv(2, dP, 0.02, dX, K).clone())
        cases.append((T, X))
    layers = tl.make_layers(2, specs)
    plan, ws = _plan(2, layers)
    tl.gemv_batch_run(plan)
    torch.cuda.synchronize()
    for (dP, a, dX, K, dY), ys, (T, X) in zip(specs, singles, cases):
        N = dP.shape[0]
        got = dY[:, :N].float().cpu().numpy().astype(np.float64)
        ref = oracle.get().linear(T, X, a, nthreads=8)
        tol = oracle.tolerance(ref, X, a)
        assert (np.abs(got - ref) <= tol).all()
        assert (np.abs(got - ys.float().cpu().numpy()) <= 2 * tol).all()


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("M", [2, 6])
def test_long_chain_multiple_items_per_cta(fmt, M):
    """Eight chained 4096 x 4096 layers: 280 items, more than one per CTA, so a
    CTA holds stages of layer l while its next item waits for layer l (at
    M = 6 the dependent layers convert their X once per launch)."""
    import torch
    import ternary_weight_03_b200 as tl
    D, depth = 4096, 8
    Ts = [synth.trits(80 + i, D, D) for i in range(depth)]
    X0 = synth.activations(90, M, D)
    alphas = [0.02] * depth
    dX0 = torch.from_numpy(X0).cuda()
    ys = [torch.full((M, D), float("nan"), dtype=torch.float16, device="cuda")
          for _ in range(depth)]
    specs = []
    for i, T in enumerate(Ts):
        dP = torch.from_numpy(tl.pack(fmt, T)).cuda()
        specs.append((dP, alphas[i], dX0 if i == 0 else ys[i - 1], D, ys[i],
                      0 if i == 0 else tl.LAYER_READS_EARLIER))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
    assert tl.device_status() == 0
    o = oracle.get()
    x = X0
    for i, T in enumerate(Ts):
        got = ys[i].float().cpu().numpy().astype(np.float64)
        ref = o.linear(T, x, alphas[i], nthreads=8)
        tol = oracle.tolerance(ref, x, alphas[i])
        if i > 0:
            ulp = np.spacing(np.abs(x).astype(np.float16)).astype(np.float64)
            tol = tol + abs(alphas[i]) * ulp.sum(axis=1)[:, None]
        assert (np.abs(got - ref) <= tol).all(), f"layer {i}"
        x = ys[i].cpu().numpy()


DECODE_LAYER = [(3072, 3072)] * 4 + [(3072, 8192)] * 2 + [(8192, 3072)]  # q k v o gate up down


@pytest.mark.parametrize("fmt,M", [(2, 1), (2, 8), (16, 1), (16, 2), (16, 8)])
def test_decode_step_210_layers_sampled(fmt, M):
    """The 30-layer decode step (210 matrices, 849 MB packed at 2 bits) as ONE
    batch launch, the configuration the bench times; per layer, sampled
    outputs against the oracle computed one by one (trits regenerated from
    their seeds for the check, so host memory stays at one layer)."""
    import torch
    import ternary_weight_03_b200 as tl
    mats = [(K, N, 1000 + 7 * layer + j) for layer in range(30)
            for j, (K, N) in enumerate(DECODE_LAYER)]
    specs, xs = [], []
    for (K, N, seed) in mats:
        P = tl.pack(fmt, synth.trits(seed, N, K))
        X = synth.activations(seed, M, K)
        xs.append(X)
        specs.append((torch.from_numpy(P).cuda(), synth.alpha_for(seed), torch.from_numpy(X).cuda(),
                      K, torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
    assert tl.device_status() == 0
    o = oracle.get()
    rng = np.random.default_rng(fmt * 10 + M)
    for (K, N, seed), X, sp in zip(mats, xs, specs):
        Y = sp[4].float().cpu().numpy().astype(np.float64)
        assert np.isfinite(Y).all()
        T = synth.trits(seed, N, K)
        ms = np.concatenate([rng.integers(0, M, 24), [M - 1]])
        ns = np.concatenate([rng.integers(0, N, 24), [N - 1]])
        ref = o.linear_at(T, X, sp[1], ms, ns)
        tol = oracle.tolerance(ref, X[ms], sp[1])
        assert (np.abs(Y[ms, ns] - ref) <= tol).all(), f"layer seed {seed}"


@pytest.mark.parametrize("fmt,M", [(2, 1), (2, 8), (16, 1), (16, 8)])
def test_fused_decode_step_sampled(fmt, M):
    """The decode step as the bench's fused variant runs it, in one batch
    launch: per decoder block Q, K and V on one X (one conversion), O on its
    own X, gate and up writing the two halves of one buffer, and the down
    projection reading silu(gate) * up from it (TL_LAYER_SWIGLU_INPUT, so it
    waits for that block's gate and up only).  Sampled outputs of every
    layer against the oracle: the down projections on fp16(silu(g) u)
    formed here in double from the stored gate and up outputs."""
    import torch
    import ternary_weight_03_b200 as tl
    specs, checks = [], []
    for blk in range(30):
        base = 1000 + 7 * blk
        xa, xo, xf = (synth.activations(base + j, M, 3072) for j in (0, 3, 4))
        dxa, dxo, dxf = (torch.from_numpy(v).cuda() for v in (xa, xo, xf))
        gu = torch.full((M, 2 * 8192), float("nan"), dtype=torch.float16, device="cuda")
        for j, (K, N) in enumerate(DECODE_LAYER):
            seed = base + j
            dP = torch.from_numpy(tl.pack(fmt, synth.trits(seed, N, K))).cuda()
            a = synth.alpha_for(seed)
            if j < 3:
                Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
                specs.append((dP, a, dxa, K, Y))
                checks.append((seed, K, N, a, xa, Y, None))
            elif j == 3:
                Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
                specs.append((dP, a, dxo, K, Y))
                checks.append((seed, K, N, a, xo, Y, None))
            elif j < 6:
                Y = gu[:, :8192] if j == 4 else gu[:, 8192:]
                specs.append((dP, a, dxf, K, Y))
                checks.append((seed, K, N, a, xf, Y, None))
            else:
                Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
                specs.append((dP, a, gu, K, Y, tl.LAYER_READS_EARLIER | tl.LAYER_SWIGLU_INPUT))
                checks.append((seed, K, N, a, None, Y, gu))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
    assert tl.device_status() == 0
    o = oracle.get()
    rng = np.random.default_rng(fmt * 100 + M)
    for seed, K, N, a, X, Yt, GU in checks:
        Y = Yt.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(Y).all(), f"layer seed {seed}"
        T = synth.trits(seed, N, K)
        ms = np.concatenate([rng.integers(0, M, 16), [M - 1]])
        ns = np.concatenate([rng.integers(0, N, 16), [N - 1]])
        if GU is None:
            ref = o.linear_at(T, X, a, ms, ns)
            tol = oracle.tolerance(ref, X[ms], a)
        else:
            x = _silu_glu(GU.cpu().numpy(), K).astype(np.float16)
            ref = o.linear_at(T, x, a, ms, ns)
            ulp = np.spacing(np.abs(x[ms])).astype(np.float64).sum(axis=1)
            tol = oracle.tolerance(ref, x[ms], a) + abs(a) * ulp
        assert (np.abs(Y[ms, ns] - ref) <= tol).all(), f"layer seed {seed}"


def _silu_glu(gu, F):
    """silu(g) * u in double from a [gate | up] row block of fp16 values."""
    g = gu[:, :F].astype(np.float64)
    u = gu[:, F:2 * F].astype(np.float64)
    return g / (1.0 + np.exp(-g)) * u


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("M", [1, 2, 3, 8])
def test_swiglu_down_projection(fmt, M):
    """Gate and up projections write the two halves of one buffer; the down
    projection reads it with TL_LAYER_SWIGLU_INPUT, its input formed on chip
    as fp16(silu(g) * u).  Checked layer by layer against the oracle: gate
    and up as plain layers, the down projection against the oracle applied to
    silu(g) * u computed here in double from the stored gate and up outputs
    and rounded to binary16, the bound adding alpha * sum_k ulp16(x_k) for the
    one-ulp freedom of that rounding.  An independent layer sits between."""
    import torch
    import ternary_weight_03_b200 as tl
    H, F, H2 = 3000, 1000, 700
    X0 = synth.activations(80 + M, M, H)
    Tg, Tu = synth.trits(81, F, H), synth.trits(82, F, H)
    Tx = synth.trits(84, 500, H)
    Td = synth.trits(83, H2, F)
    ag, au, ax, ad = 0.021, 0.033, 0.04, 0.017
    dX0 = torch.from_numpy(X0).cuda()
    GU = torch.full((M, 2 * F), float("nan"), dtype=torch.float16, device="cuda")
    Yx = torch.full((M, 504), float("nan"), dtype=torch.float16, device="cuda")
    Yd = torch.full((M, H2 + (-H2) % 8), float("nan"), dtype=torch.float16, device="cuda")
    pk = lambda T: torch.from_numpy(tl.pack(fmt, T)).cuda()
    specs = [(pk(Tg), ag, dX0, H, GU[:, :F]), (pk(Tu), au, dX0, H, GU[:, F:]),
             (pk(Tx), ax, dX0, H, Yx),
             (pk(Td), ad, GU, F, Yd, tl.LAYER_READS_EARLIER | tl.LAYER_SWIGLU_INPUT)]
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    outs = []
    for _ in range(2):
        Yd.fill_(float("nan"))
        tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
        assert tl.device_status() == 0
        outs.append(Yd.cpu().numpy().view(np.uint16).copy())
    assert np.array_equal(outs[0], outs[1]), "not deterministic"
    o = oracle.get()
    gu = GU.cpu().numpy()
    for T, a, Y in ((Tg, ag, gu[:, :F]), (Tu, au, gu[:, F:]), (Tx, ax, Yx[:, :500].cpu().numpy())):
        ref = o.linear(T, X0, a, nthreads=8)
        assert (np.abs(Y.astype(np.float64) - ref) <= oracle.tolerance(ref, X0, a)).all()
    x = _silu_glu(gu, F).astype(np.float16)  # the down projection's input, rounded once
    ref = o.linear(Td, x, ad, nthreads=8)
    ulp = np.spacing(np.abs(x)).astype(np.float64)
    tol = oracle.tolerance(ref, x, ad) + abs(ad) * ulp.sum(axis=1)[:, None]
    got = Yd[:, :H2].float().cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= tol).all(), f"{int((np.abs(got - ref) > tol).sum())} outside"
    assert np.isnan(Yd[:, H2:].float().cpu().numpy()).all(), "wrote past column N"


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("M", [1, 8])
def test_layers_sharing_x(fmt, M):
    """Q, K and V on one X (one conversion of X, three alphas), O on another
    X, and two layers on a third: each layer against the oracle, and the
    batch needs less workspace than the same layers on distinct X copies."""
    import torch
    import ternary_weight_03_b200 as tl
    K = 2000
    Xa, Xb, Xc = (synth.activations(90 + i + M, M, K) for i in range(3))
    dXa, dXb, dXc = (torch.from_numpy(v).cuda() for v in (Xa, Xb, Xc))
    shapes = [(700, 0.02, 0), (300, 0.03, 0), (300, 0.045, 0), (700, 0.011, 1), (1200, 0.05, 2),
              (1200, 0.013, 2)]
    xs = [(Xa, dXa), (Xb, dXb), (Xc, dXc)]
    cases, specs, specs_copy = [], [], []
    for i, (N, a, xi) in enumerate(shapes):
        T = synth.trits(95 + i, N, K)
        dP = torch.from_numpy(tl.pack(fmt, T)).cuda()
        dY = torch.full((M + 1, N + (-N) % 8), float("nan"), dtype=torch.float16, device="cuda")
        specs.append((dP, a, xs[xi][1], K, dY[:M]))
        specs_copy.append((dP, a, xs[xi][1].clone(), K, dY[:M]))
        cases.append((T, xs[xi][0], a, dY, N))  # row M is a guard row
    layers = tl.make_layers(fmt, specs)
    shared_bytes = tl.gemv_batch_bytes(fmt, layers)
    assert shared_bytes < tl.gemv_batch_bytes(fmt, tl.make_layers(fmt, specs_copy))
    plan, ws = _plan(fmt, layers)
    tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
    assert tl.device_status() == 0
    for T, X, a, dY, N in cases:
        _check_layer(T, X, a, dY, N, M)


@pytest.mark.parametrize("fmt", [2, 16])
def test_dependent_layer_before_independent_ones(fmt):
    """A slow producer (one tile, long K), a layer reading its output, then
    sixteen small independent layers that finish quickly.  The dependent
    layer must see its producer complete however the layers' tiles
    interleave (a count of final tiles alone would let the small layers'
    tiles stand in for the producer's).  Repeated runs agree bit for bit."""
    import torch
    import ternary_weight_03_b200 as tl
    M, K0, N0 = 2, 20000, 256
    T0 = synth.trits(120, N0, K0)
    X0 = synth.activations(121, M, K0)
    T1 = synth.trits(122, 300, N0)
    a0, a1 = 0.004, 0.03
    dX0 = torch.from_numpy(X0).cuda()
    Y0 = torch.full((M, N0), float("nan"), dtype=torch.float16, device="cuda")
    Y1 = torch.full((M, 304), float("nan"), dtype=torch.float16, device="cuda")
    pk = lambda T: torch.from_numpy(tl.pack(fmt, T)).cuda()
    specs = [(pk(T0), a0, dX0, K0, Y0), (pk(T1), a1, Y0, N0, Y1, tl.LAYER_READS_EARLIER)]
    small = []
    for i in range(16):
        T = synth.trits(130 + i, 64, 128)
        X = synth.activations(150 + i, M, 128)
        Y = torch.full((M, 64), float("nan"), dtype=torch.float16, device="cuda")
        specs.append((pk(T), 0.05, torch.from_numpy(X).cuda(), 128, Y))
        small.append((T, X, Y))
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    outs = []
    for _ in range(3):
        Y0.fill_(float("nan"))
        Y1.fill_(float("nan"))
        tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
        assert tl.device_status() == 0
        outs.append(Y1.cpu().numpy().view(np.uint16).copy())
    for o_ in outs[1:]:
        assert np.array_equal(o_, outs[0])
    o = oracle.get()
    ref0 = o.linear(T0, X0, a0, nthreads=8)
    y0 = Y0.cpu().numpy()
    assert (np.abs(y0.astype(np.float64) - ref0) <= oracle.tolerance(ref0, X0, a0)).all()
    ref1 = o.linear(T1, y0, a1, nthreads=8)
    ulp = np.spacing(np.abs(y0)).astype(np.float64)
    tol = oracle.tolerance(ref1, y0, a1) + abs(a1) * ulp.sum(axis=1)[:, None]
    got = Y1[:, :300].float().cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref1) <= tol).all()
    for T, X, Y in small:
        ref = o.linear(T, X, 0.05)
        assert (np.abs(Y.float().cpu().numpy() - ref) <= oracle.tolerance(ref, X, 0.05)).all()


@pytest.mark.parametrize("fmt", [2, 16])
@pytest.mark.parametrize("M", [2, 5])
def test_interleaved_chains(fmt, M):
    """Dependencies follow the data: a dependent layer waits for the earlier
    layers whose Y overlaps its X, not for every earlier layer.  Two chains
    interleave (a0, b0, a1 reads a0, b1 reads b0's output plus 500 more
    columns of the same buffer), and a flagged SwiGLU layer whose [gate | up]
    input no layer of the batch writes runs without waiting.  Each layer
    against the oracle on the inputs as stored; two runs agree bit for bit.
    At M = 5 the dependent layers convert their X once per launch (fp16
    engine), the SwiGLU layer without waiting for any layer."""
    import torch
    import ternary_weight_03_b200 as tl
    K0 = 3000
    X0, X1 = synth.activations(130, M, K0), synth.activations(131, M, K0)
    GUc = synth.activations(132, M, 2 * 800)
    Ta0, Tb0 = synth.trits(133, 1000, K0), synth.trits(134, 2000, K0)
    Ta1, Tb1, Tc = synth.trits(135, 700, 1000), synth.trits(136, 900, 2500), synth.trits(137, 600, 800)
    aa0, ab0, aa1, ab1, ac = 0.02, 0.013, 0.031, 0.017, 0.025
    dX0, dX1, dGU = (torch.from_numpy(v).cuda() for v in (X0, X1, GUc))
    bufA = torch.full((M, 1000), float("nan"), dtype=torch.float16, device="cuda")
    tail = synth.activations(138, M, 500)
    bufB = torch.full((M, 2504), float("nan"), dtype=torch.float16, device="cuda")
    bufB[:, 2000:2500] = torch.from_numpy(tail).cuda()
    Za = torch.full((M, 704), float("nan"), dtype=torch.float16, device="cuda")
    Zb = torch.full((M, 904), float("nan"), dtype=torch.float16, device="cuda")
    Zc = torch.full((M, 600), float("nan"), dtype=torch.float16, device="cuda")
    pk = lambda T: torch.from_numpy(tl.pack(fmt, T)).cuda()
    RE, SW = tl.LAYER_READS_EARLIER, tl.LAYER_SWIGLU_INPUT
    specs = [(pk(Ta0), aa0, dX0, K0, bufA), (pk(Tb0), ab0, dX1, K0, bufB[:, :2000]),
             (pk(Ta1), aa1, bufA, 1000, Za, RE), (pk(Tb1), ab1, bufB[:, :2500], 2500, Zb, RE),
             (pk(Tc), ac, dGU, 800, Zc, RE | SW)]
    layers = tl.make_layers(fmt, specs)
    plan, ws = _plan(fmt, layers)
    outs = []
    for _ in range(2):
        for z in (Za, Zb, Zc):
            z.fill_(float("nan"))
        tl.gemv_batch_run(plan, flags=tl.FLAG_PDL)
        assert tl.device_status() == 0
        outs.append([z.cpu().numpy().view(np.uint16).copy() for z in (Za, Zb, Zc)])
    assert all(np.array_equal(u, v) for u, v in zip(*outs)), "not deterministic"
    o = oracle.get()

    def check(T, x, a, got, stored):
        ref = o.linear(T, x, a, nthreads=8)
        tol = oracle.tolerance(ref, x, a)
        if stored:  # x was stored as binary16 by an earlier layer (or rounded once here)
            tol = tol + abs(a) * np.spacing(np.abs(x).astype(np.float16)).astype(np.float64).sum(axis=1)[:, None]
        err = np.abs(got.astype(np.float64) - ref)
        assert (err <= tol).all(), f"{int((err > tol).sum())} of {err.size} outside tolerance"

    A, B = bufA.cpu().numpy(), bufB.cpu().numpy()
    check(Ta0, X0, aa0, A, False)
    check(Tb0, X1, ab0, B[:, :2000], False)
    check(Ta1, A, aa1, Za[:, :700].cpu().numpy(), True)
    check(Tb1, B[:, :2500], ab1, Zb[:, :900].cpu().numpy(), True)
    assert np.array_equal(B[:, 2000:2500], tail), "the columns no layer writes changed"
    x = _silu_glu(GUc, 800).astype(np.float16)
    check(Tc, x, ac, Zc.cpu().numpy(), True)
