#!/usr/bin/env python3
"""Benchmark of the ternary linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Headline workload (one "step"): the decode GEMV sweep with 2-bit packing:
(K, N) in {(3072,3072), (3072,8192), (8192,3072), (4096,4096), (4096,14336),
(14336,4096)}, M in {1, 8}: twelve tl_gemv calls, fp16 activations ~ N(0,1),
uniform trits, one alpha ~ U(0.01, 0.05) per matrix, seeds 0..5.  Every call
reads a different copy of its packed matrix; the copies rotate through more
than three times the L2 size, so every weight byte comes from HBM.  A step is
one CUDA-graph replay of the twelve calls (event records between them give
the per-launch kernel times).

Metric: packed-weight bytes streamed per second (GB/s), whole job, i.e. the
sum over ranks of bytes divided by the slowest rank's time.  Under torchrun
every rank runs the same sweep on its own GPU (weak scaling; the layer needs
no collective).  Secondary measurements (1.6-bit sweep, batched GEMM,
30-layer decode step) are appended under "secondary".

--impl reference times the CPU oracle (the definition of the layer, in
double) on a bounded sample of the same workload; it is the baseline arm.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

SWEEP = [(3072, 3072), (3072, 8192), (8192, 3072), (4096, 4096), (4096, 14336), (14336, 4096)]
SWEEP_M = (1, 8)
L2_BYTES = 126 << 20
METRIC = "packed-ternary GEMV HBM GB/s (% of peak); batched GEMM TFLOP/s (% peak)"
WORKLOAD = ("decode GEMV sweep, 2-bit packing, M in {1,8}, (K,N) in (3072,3072) (3072,8192) "
            "(8192,3072) (4096,4096) (4096,14336) (14336,4096), fp16 x ~ N(0,1), uniform trits, "
            "alpha ~ U(0.01,0.05) per matrix, seeds 0..5")
DECODE_LAYER = [("q", 3072, 3072), ("k", 3072, 3072), ("v", 3072, 3072), ("o", 3072, 3072),
                ("gate", 3072, 8192), ("up", 3072, 8192), ("down", 8192, 3072)]


# ---------------------------------------------------------------------------
# distributed plumbing (testable with gloo on CPU)
# ---------------------------------------------------------------------------
def dist_env():
    """(rank, local_rank, world) from the torchrun environment, else (0, 0, 1)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def reduce_step_time(ms: float, units: float, group=None):
    """Max of the per-rank elapsed time and sum of per-rank work units."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return ms, units
    t = torch.tensor([ms], dtype=torch.float64)
    u = torch.tensor([units], dtype=torch.float64)
    if dist.get_backend(group) == "nccl":
        t, u = t.cuda(), u.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(u, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), float(u.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------------------
# measured peaks and clocks
# ---------------------------------------------------------------------------
def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------
def make_matrix(fmt: int, K: int, N: int, seed: int, p0: float = 1.0 / 3.0,
                codec: str = "product"):
    """Packed weights, trits and alpha of one seeded matrix.  codec="product"
    packs with the library (the GPU arm's inputs); codec="oracle" with the
    CPU oracle's own packer (the CPU arms, which load nothing of the library)."""
    import synth
    T = synth.trits(seed, N, K, p0=p0)
    if codec == "oracle":
        import oracle
        return oracle.get().pack(fmt, T), T, synth.alpha_for(seed)
    import ternary_weight_03_b200 as tl
    return tl.pack(fmt, T), T, synth.alpha_for(seed)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
class Sweep:
    """Device-resident inputs of the GEMV sweep with rotating weight copies."""

    def __init__(self, fmt: int, dev, shapes=SWEEP, ms=SWEEP_M, p0=1.0 / 3.0, seed0=0,
                 min_rotation_bytes=3 * L2_BYTES):
        import torch
        import synth
        import ternary_weight_03_b200 as tl
        self.fmt, self.dev, self.ms = fmt, dev, ms
        self.items = []  # (K, N, packed host, alpha, X per M)
        per_set = 0
        for i, (K, N) in enumerate(shapes):
            P, _, alpha = make_matrix(fmt, K, N, seed0 + i, p0)
            xs = {M: torch.from_numpy(synth.activations(seed0 + i, M, K)).to(dev) for M in ms}
            self.items.append((K, N, P, alpha, xs))
            per_set += P.nbytes
        self.copies = max(2 * len(ms), -(-min_rotation_bytes // per_set))
        self.dP = [[torch.from_numpy(P).to(dev) for (_, _, P, _, _) in self.items]
                   for _ in range(self.copies)]
        self.Y = {M: [torch.empty((M, N + (-N) % 8), dtype=torch.float16, device=dev)
                      for (_, N, _, _, _) in self.items] for M in ms}
        self.bytes_per_pass = sum(N * tl.row_bytes(fmt, K) for (K, N, _, _, _) in self.items)
        self.bytes_per_step = self.bytes_per_pass * len(ms)
        self.launches_per_step = len(self.items) * len(ms)
        self.rotation_bytes = self.copies * per_set
        self.batch = False
        self.plans, self.workspaces = [], []

    def use_batch(self):
        """Switch to one tl_gemv_batch_run per step: every layer of the step in a
        single launch.  Phase ph's plan reads the M-th token count's weights from
        copy (len(ms) * ph + m) % copies, the same rotation as the per-call steps."""
        import torch
        import ternary_weight_03_b200 as tl
        nm = len(self.ms)
        nphase = self.copies // nm if self.copies % nm == 0 else self.copies
        for ph in range(nphase):
            specs = []
            for mi, M in enumerate(self.ms):
                copy = (nm * ph + mi) % self.copies
                for i, (K, N, _, alpha, xs) in enumerate(self.items):
                    specs.append((self.dP[copy][i], alpha, xs[M], K, self.Y[M][i]))
            layers = tl.make_layers(self.fmt, specs)
            ws = torch.zeros(tl.gemv_batch_bytes(self.fmt, layers), dtype=torch.uint8,
                             device=self.dev)
            self.plans.append(tl.gemv_batch_plan(self.fmt, layers, ws))
            self.workspaces.append(ws)
        self.batch = True
        self.launches_per_step = 1

    def enqueue(self, step: int, stream, events=None, flags: int = 1):
        """Enqueue the calls of one step on `stream` (optionally recording an
        event after each call for per-launch timing).  flags = TL_FLAG_PDL:
        each call may start streaming its (static) weights while the previous
        call drains."""
        import ternary_weight_03_b200 as tl
        if self.batch:
            if events is not None:
                events[0].record(stream)
            tl.gemv_batch_run(self.plans[step % len(self.plans)], stream=stream, flags=flags)
            if events is not None:
                events[1].record(stream)
            return
        L = tl.lib()
        s = stream.cuda_stream
        j = 0
        if events is not None:
            events[0].record(stream)
        for mi, M in enumerate(self.ms):
            copy = (len(self.ms) * step + mi) % self.copies
            for i, (K, N, _, alpha, xs) in enumerate(self.items):
                dP, X, Y = self.dP[copy][i], xs[M], self.Y[M][i]
                rc = L.tl_gemv_ex(self.fmt, dP.data_ptr(), dP.stride(0), alpha, X.data_ptr(),
                                  X.stride(0), Y.data_ptr(), Y.stride(0), M, N, K, flags, s)
                if rc != 0:
                    raise RuntimeError(f"tl_gemv -> {tl.status_str(rc)}")
                j += 1
                if events is not None:
                    events[j].record(stream)


# steps per CUDA graph in the timed region: consecutive launches inside one
# graph are chained by programmatic dependent launch (a launch streams its
# first weights while its predecessor drains); between graph replays they are not
GRAPH_STEPS = 45


def time_graphs(sweep: Sweep, steps: int, warmup: int, stream, clock_gpu: int | None = None,
                flags: int = 1):
    """Warm up with `warmup` steps, then time exactly `steps` steps with CUDA
    events on the launch stream.  Steps are captured into CUDA graphs of up to
    GRAPH_STEPS consecutive steps (the rotation phases advance from step to
    step), so the timed region replays steps // GRAPH_STEPS such graphs and one
    graph of the remaining steps.  The timed graphs hold the layer calls only.
    Afterwards one untimed replay of graphs with event records between the
    calls, launched without PDL, gives a per-call breakdown.  Returns (total
    ms, per-call ms list, clocks summary)."""
    import torch
    nm = len(sweep.ms)
    nphase = sweep.copies // nm if sweep.copies % nm == 0 else sweep.copies
    if sweep.batch:
        nphase = len(sweep.plans)

    def capture(first, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                sweep.enqueue((first + i) % nphase, stream, flags=flags)
        return g

    with torch.cuda.stream(stream):
        sweep.enqueue(0, stream, flags=flags)  # per-device setup outside capture
        torch.cuda.synchronize()
        g_warm = capture(0, warmup)
        full, rem = divmod(steps, GRAPH_STEPS)
        g_full = capture(warmup % nphase, GRAPH_STEPS) if full else None
        g_rem = capture((warmup + full * GRAPH_STEPS) % nphase, rem) if rem else None
        g_warm.replay()
    torch.cuda.synchronize()
    barrier()
    sampler = ClockSampler(clock_gpu) if clock_gpu is not None else None
    if sampler:
        sampler.__enter__()
    try:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(full):
                g_full.replay()
            if g_rem is not None:
                g_rem.replay()
            end.record(stream)
        torch.cuda.synchronize()
        total_ms = start.elapsed_time(end)
    finally:
        if sampler:
            sampler.__exit__(None, None, None)
    del g_warm, g_full, g_rem
    # per-call breakdown (untimed): external event records between calls
    per_call = [0.0] * sweep.launches_per_step
    with torch.cuda.stream(stream):
        for ph in range(min(nphase, 2)):
            evs = [torch.cuda.Event(enable_timing=True, external=True)
                   for _ in range(sweep.launches_per_step + 1)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                sweep.enqueue(ph, stream, evs, flags=0)
            g.replay()
            torch.cuda.synchronize()
            for j in range(sweep.launches_per_step):
                per_call[j] += evs[j].elapsed_time(evs[j + 1]) / min(nphase, 2)
    return total_ms, per_call, (sampler.summary() if sampler else None)


def time_e2e(sweep: Sweep, steps: int, warmup: int, stream):
    """End to end through the C ABI from pinned host buffers: every step
    copies its packed weights and activations host -> device, runs the step's
    layers in one tl_gemv_batch_run (planned once on these buffers) and copies
    the outputs back.  Returns (ms, h2d bytes, d2h bytes)."""
    import torch
    import ternary_weight_03_b200 as tl
    hP = [torch.from_numpy(P).pin_memory() for (_, _, P, _, _) in sweep.items]
    hX = {M: [xs[M].cpu().pin_memory() for (_, _, _, _, xs) in sweep.items] for M in sweep.ms}
    hY = {M: [torch.empty(tuple(y.shape), dtype=torch.float16).pin_memory() for y in sweep.Y[M]]
          for M in sweep.ms}
    # one device copy of the weights per token count, as in the device-resident step
    dP = {M: [torch.empty_like(p, device=sweep.dev) for p in hP] for M in sweep.ms}
    dX = {M: [torch.empty_like(x, device=sweep.dev) for x in hX[M]] for M in sweep.ms}
    specs = [(dP[M][i], alpha, dX[M][i], K, sweep.Y[M][i])
             for M in sweep.ms for i, (K, N, _, alpha, _) in enumerate(sweep.items)]
    layers = tl.make_layers(sweep.fmt, specs)
    ws = torch.zeros(tl.gemv_batch_bytes(sweep.fmt, layers), dtype=torch.uint8, device=sweep.dev)
    plan = tl.gemv_batch_plan(sweep.fmt, layers, ws)
    h2d = sum(p.numel() for p in hP) * len(sweep.ms) + sum(
        x.numel() * 2 for M in sweep.ms for x in hX[M])
    d2h = sum(y.numel() * 2 for M in sweep.ms for y in hY[M])

    def one_step():
        for M in sweep.ms:
            for i in range(len(sweep.items)):
                dP[M][i].copy_(hP[i], non_blocking=True)
                dX[M][i].copy_(hX[M][i], non_blocking=True)
        tl.gemv_batch_run(plan, stream=stream)
        for M in sweep.ms:
            for i, Y in enumerate(sweep.Y[M]):
                hY[M][i].copy_(Y, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            one_step()
        b.record(stream)
        torch.cuda.synchronize()
    return a.elapsed_time(b), h2d, d2h


def check_outputs(sweep: Sweep, samples: int = 64):
    """Spot-check the last outputs of every call against the oracle."""
    import oracle
    import synth
    o = oracle.get()
    worst = 0.0
    rng = np.random.default_rng(0)
    for i, (K, N, P, alpha, xs) in enumerate(sweep.items):
        T = synth.trits(i, N, K)
        for M in sweep.ms:
            X = xs[M].cpu().numpy()
            Y = sweep.Y[M][i][:, :N].float().cpu().numpy().astype(np.float64)
            ms = rng.integers(0, M, samples)
            ns = rng.integers(0, N, samples)
            ref = o.linear_at(T, X, alpha, ms, ns)
            tol = oracle.tolerance(ref, X[ms], alpha)
            err = np.abs(Y[ms, ns] - ref) / tol
            if not (err <= 1.0).all():
                raise AssertionError(f"bench output outside tolerance for shape {(K, N)} M={M}")
            worst = max(worst, float(err.max()))
    return worst


def cpu_baseline(seconds: float = 10.0, threads: int | None = None):
    """The oracle (unpack + double-precision layer) on a bounded sample of the
    sweep: for every (shape, M), the first rows of the matrix, sized so the
    whole sample takes about `seconds` with all host threads; the same sample
    is then timed with one thread.  Inputs are packed by the oracle's own
    codec.  Returns packed bytes/s and details."""
    import oracle
    import synth
    o = oracle.get()
    threads = threads or os.cpu_count() or 1
    # calibrate on a small slice
    K, N = SWEEP[0]
    P, T, alpha = make_matrix(2, K, 64, 0, codec="oracle")
    X = synth.activations(0, 8, K)
    t0 = time.perf_counter()
    rc, Tu, _ = o.unpack(2, P, K)
    o.linear(Tu, X, alpha, nthreads=threads)
    per_trit_m = (time.perf_counter() - t0) / (64 * K * 8)
    total_trit_m = sum(K * N for (K, N) in SWEEP) * sum(SWEEP_M)
    frac = min(1.0, seconds / max(per_trit_m * total_trit_m, 1e-9))
    mats, rows_used = [], []
    for i, (K, N) in enumerate(SWEEP):
        rows = min(N, max(threads, int(N * frac)))
        Pm, _, alpha = make_matrix(2, K, rows, i, codec="oracle")
        mats.append((K, rows, Pm, alpha, {M: synth.activations(i, M, K) for M in SWEEP_M}))
        rows_used.append(rows)

    def timed(nthreads, sample):
        done, el = 0, 0.0
        for (K, rows, Pm, alpha, xs) in sample:
            for M in SWEEP_M:
                t0 = time.perf_counter()
                rc, Tu, _ = o.unpack(2, Pm, K)
                o.linear(Tu, xs[M], alpha, nthreads=nthreads)
                el += time.perf_counter() - t0
                done += rows * ((K + 3) // 4)
        return done, el

    done, elapsed = timed(threads, mats)
    # one thread: a twentieth of the rows (the rate is per byte)
    small = [(K, max(1, rows // 20), Pm[:max(1, rows // 20)], a, xs)
             for (K, rows, Pm, a, xs) in mats]
    done1, el1 = timed(1, small)
    return {"value": round(done / elapsed / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"first {rows_used} rows of each sweep matrix (both M), unpack + double "
                      f"accumulation, {elapsed:.1f} s",
            "one_thread": {"value": round(done1 / el1 / 1e9, 5), "unit": "GB/s", "cores": 1,
                           "sample": f"first {[m[1] for m in small]} rows, {el1:.1f} s"}}


def decode_step(dev, stream, fmts=(2, 16), ms=(1, 8), steps: int = 20, warmup: int = 3):
    """All linear layers of one decode step of a 30-layer LLaMA-style SwiGLU
    decoder (hidden 3072, intermediate 8192): per layer q, k, v, o
    (3072 -> 3072), gate, up (3072 -> 8192), down (8192 -> 3072), i.e. 210
    distinct seeded matrices (p0 = 1/3, alpha ~ U(0.01, 0.05)), each with its
    own seeded activation vector(s), run as ONE tl_gemv_batch_run per step
    (graph-captured, programmatic dependent launch).  "chained" reruns the
    2-bit M = 1 step as one chain: layer i reads (the first K_i columns of)
    the buffer whose first N_{i-1} columns layer i - 1 writes, flagged
    TL_LAYER_READS_EARLIER (a serial dependency per layer; alpha =
    1 / sqrt(2K/3) keeps the chained values in range).  "fused" (2-bit) runs the step
    as a decoder would: q, k and v on one shared X (converted once), gate
    and up on another, writing the two halves of one buffer, and down
    reading silu(gate) * up from it (TL_LAYER_SWIGLU_INPUT, a dependency on
    the earlier layers).  Returns GB/s of packed weights."""
    import torch
    import synth
    import ternary_weight_03_b200 as tl
    mats = []  # (K, N, seed)
    for layer in range(30):
        for j, (_, K, N) in enumerate(DECODE_LAYER):
            mats.append((K, N, 1000 + 7 * layer + j))
    out = {}

    def timed(plan):
        # one graph holds `steps` consecutive decode steps (each one launch over
        # the 210 layers, chained by programmatic dependent launch)
        with torch.cuda.stream(stream):
            tl.gemv_batch_run(plan, stream=stream, flags=1)
            torch.cuda.synchronize()
            gw, g = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(gw, stream=stream):
                for _ in range(warmup):
                    tl.gemv_batch_run(plan, stream=stream, flags=1)
            with torch.cuda.graph(g, stream=stream):
                for _ in range(steps):
                    tl.gemv_batch_run(plan, stream=stream, flags=1)
            gw.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    for fmt in fmts:
        dev_mats, total = [], 0
        for (K, N, seed) in mats:
            P = tl.pack(fmt, synth.trits(seed, N, K))
            dev_mats.append((K, N, torch.from_numpy(P).to(dev), synth.alpha_for(seed)))
            total += N * tl.row_bytes(fmt, K)
        for M in ms:
            xs = [torch.from_numpy(synth.activations(seed, M, K)).to(dev)
                  for (K, N, seed) in mats]
            ys = [torch.empty((M, N), dtype=torch.float16, device=dev) for (K, N, _) in mats]
            variants = [("", 0)] + ([("_chained", tl.LAYER_READS_EARLIER)]
                                    if fmt == 2 and M == 1 else [])
            for suffix, flag in variants:
                if flag:
                    # buffer i holds layer i's input; layer i - 1 writes its first columns
                    bufs = []
                    for i, (K, N, seed) in enumerate(mats):
                        w = max(K, mats[i - 1][1] if i else 0)
                        w += (-w) % 8
                        bufs.append(torch.from_numpy(synth.activations(seed, M, w)).to(dev))
                    specs = [(dP, 1.0 / math.sqrt(2.0 * K / 3.0), bufs[i][:, :K], K,
                              bufs[i + 1][:, :N] if i + 1 < len(bufs) else ys[i], flag if i else 0)
                             for i, (K, N, dP, alpha) in enumerate(dev_mats)]
                else:
                    specs = [(dP, alpha, X, K, Y)
                             for (K, N, dP, alpha), X, Y in zip(dev_mats, xs, ys)]
                layers = tl.make_layers(fmt, specs)
                ws = torch.zeros(tl.gemv_batch_bytes(fmt, layers), dtype=torch.uint8, device=dev)
                plan = tl.gemv_batch_plan(fmt, layers, ws)
                ms_step = timed(plan)
                gbs = total / (ms_step * 1e-3) / 1e9
                out[f"fmt{fmt}_M{M}{suffix}"] = {
                    "packed_bytes": total, "us_per_step": round(ms_step * 1e3, 2),
                    "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks()["hbm_gbs"], 4)}
                del plan, ws
            if fmt == 2:
                # the fused step: per decoder layer q, k, v share X; gate and up
                # share another X and fill [gate | up]; down reads silu(gate) * up
                specs = []
                for layer in range(30):
                    base = 7 * layer
                    xa, xo, xf = xs[base], xs[base + 3], xs[base + 4]
                    gu = torch.empty((M, 2 * 8192), dtype=torch.float16, device=dev)
                    for j in range(7):
                        K, N, dP, alpha = dev_mats[base + j]
                        if j < 3:
                            specs.append((dP, alpha, xa, K, ys[base + j]))
                        elif j == 3:
                            specs.append((dP, alpha, xo, K, ys[base + j]))
                        elif j < 6:
                            half = gu[:, :8192] if j == 4 else gu[:, 8192:]
                            specs.append((dP, alpha, xf, K, half))
                        else:
                            specs.append((dP, alpha, gu, K, ys[base + j],
                                          tl.LAYER_READS_EARLIER | tl.LAYER_SWIGLU_INPUT))
                layers = tl.make_layers(fmt, specs)
                ws = torch.zeros(tl.gemv_batch_bytes(fmt, layers), dtype=torch.uint8, device=dev)
                plan = tl.gemv_batch_plan(fmt, layers, ws)
                ms_step = timed(plan)
                gbs = total / (ms_step * 1e-3) / 1e9
                out[f"fmt{fmt}_M{M}_fused"] = {
                    "packed_bytes": total, "us_per_step": round(ms_step * 1e3, 2),
                    "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks()["hbm_gbs"], 4)}
                del plan, ws, specs
            del xs, ys
        del dev_mats
        torch.cuda.empty_cache()
    return out


def time_single_cold(dev, stream, pk):
    """K = N = 1024, M = 1, 2-bit, alpha = 0.02 (262,144 packed bytes): one
    tl_gemv_ex call at a time, L2 flushed by a 256 MiB write before each,
    median of 20 calls.  Latency-bound: the figure is the call's latency."""
    import numpy as np
    import torch
    import synth
    import ternary_weight_03_b200 as tl
    P, _, _ = make_matrix(2, 1024, 1024, 0)
    dP = torch.from_numpy(P).to(dev)
    X = torch.from_numpy(synth.activations(0, 1, 1024)).to(dev)
    Y = torch.empty((1, 1024), dtype=torch.float16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    with torch.cuda.stream(stream):
        for i in range(23):
            flush.fill_(i & 255)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            rc = tl.lib().tl_gemv_ex(2, dP.data_ptr(), dP.stride(0), 0.02, X.data_ptr(), 1024,
                                     Y.data_ptr(), 1024, 1, 1024, 1024, 0, stream.cuda_stream)
            b.record(stream)
            torch.cuda.synchronize()
            if rc != 0:
                return {"status": tl.status_str(rc)}
            if i >= 3:
                times.append(a.elapsed_time(b) * 1e3)
    us = float(np.median(times))
    gbs = 1024 * 256 / (us * 1e-6) / 1e9
    return {"us_median": round(us, 2), "GB/s": round(gbs, 1),
            "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
            "l2": "flushed by a 256 MiB write before every call"}


def time_ternarise(dev, stream, pk):
    """Device ternariser on the largest sweep shapes: fp16 W read twice (the
    exact |W| sum, then quantise + pack) and the packed rows written once."""
    import torch
    import ternary_weight_03_b200 as tl
    res = {}
    for fmt in (2, 16):
        for (N, K) in ((14336, 4096), (4096, 14336)):
            g = torch.Generator(device=dev).manual_seed(N + K)
            W = (torch.randn((N, K), generator=g, device=dev) * 0.02).half()
            P = torch.empty((N, tl.padded_ldp(fmt, K)), dtype=torch.uint8, device=dev)
            alpha = torch.empty(1, dtype=torch.float32, device=dev)
            ws = torch.empty(tl.TERNARISE_WORKSPACE_BYTES, dtype=torch.uint8, device=dev)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    tl.ternarise(fmt, W, out=P, alpha=alpha, workspace=ws, stream=stream)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                reps = 10
                a.record(stream)
                for _ in range(reps):
                    tl.ternarise(fmt, W, out=P, alpha=alpha, workspace=ws, stream=stream)
                b.record(stream)
                torch.cuda.synchronize()
            us = a.elapsed_time(b) * 1e3 / reps
            moved = 2 * (2 * N * K) + N * tl.row_bytes(fmt, K)
            gbs = moved / (us * 1e-6) / 1e9
            res[f"fmt{fmt}_N{N}_K{K}"] = {"us": round(us, 2), "GB/s": round(gbs, 1),
                                         "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
                                         "bytes": moved}
            del W, P
    return res


def secondary(dev, stream):
    """1.6-bit sweep (p0 = 1/3), batched GEMM (both formats), the 30-layer
    decode step, the device ternariser, the cold 1024 x 1024 single call and
    the sweep as separate per-layer calls."""
    import torch
    import ternary_weight_03_b200 as tl
    out = {}
    pk = peaks()
    # the 2-bit sweep at one token count only (M = 1: the decode GEMV of a
    # single sequence), one launch per step
    for ms_, key in (((1,), "gemv_2bit_sweep_M1"), ((8,), "gemv_2bit_sweep_M8")):
        sw = Sweep(2, dev, ms=ms_)
        sw.use_batch()
        n = 90
        ms, _, _ = time_graphs(sw, n, 5, stream)
        gbs = sw.bytes_per_step * n / (ms * 1e-3) / 1e9
        out[key] = {"GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
                    "us_per_step": round(ms / n * 1e3, 2), "packed_bytes": sw.bytes_per_step}
        del sw
        torch.cuda.empty_cache()
    # 1.6-bit sweep (config 3) at three trit sparsities, one launch per step
    for p0 in (0.2, 1.0 / 3.0, 0.6):
        sw = Sweep(16, dev, p0=p0)
        sw.use_batch()
        n = 45
        ms, per_launch, _ = time_graphs(sw, n, 5, stream)
        gbs = sw.bytes_per_step * n / (ms * 1e-3) / 1e9
        out[f"gemv_1p6bit_sweep_p0_{p0:.2f}"] = {
            "GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
            "us_per_step": round(ms / n * 1e3, 2)}
        del sw
        torch.cuda.empty_cache()
    # batched GEMM, both formats
    import synth
    for fmt, key in ((2, "gemm_2bit"), (16, "gemm_1p6bit")):
        gemm = {}
        for (K, N) in ((4096, 14336), (14336, 4096)):
            P, _, alpha = make_matrix(fmt, K, N, 0)
            dP = torch.from_numpy(P).to(dev)
            for M in (16, 64, 256, 1024, 4096):
                X = torch.from_numpy(synth.activations(1, M, K)).to(dev)
                Y = torch.empty((M, N), dtype=torch.float16, device=dev)

                def call():
                    return tl.lib().tl_gemm(fmt, dP.data_ptr(), dP.stride(0), alpha, X.data_ptr(),
                                            K, Y.data_ptr(), N, M, N, K, stream.cuda_stream)
                rc = call()
                if rc != 0:
                    gemm[f"M{M}_K{K}_N{N}"] = {"status": tl.status_str(rc)}
                    continue
                with torch.cuda.stream(stream):
                    for _ in range(3):
                        call()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    reps = 10
                    a.record(stream)
                    for _ in range(reps):
                        call()
                    b.record(stream)
                    torch.cuda.synchronize()
                us = a.elapsed_time(b) * 1e3 / reps
                tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
                # small M is bound by HBM: packed weights + X + Y once
                moved = N * tl.row_bytes(fmt, K) + 2 * M * K + 2 * M * N
                gbs = moved / (us * 1e-6) / 1e9
                gemm[f"M{M}_K{K}_N{N}"] = {"us": round(us, 2), "TFLOP/s": round(tf, 1),
                                           "frac_tensor": round(tf / pk["bf16_tflops"], 4),
                                           "GB/s": round(gbs, 1),
                                           "frac_hbm": round(gbs / pk["hbm_gbs"], 4)}
            del dP
        out[key] = gemm
    out["decode_step_30_layers"] = decode_step(dev, stream)
    for key, fn in (("ternarise", time_ternarise),
                    ("gemv_2bit_1024x1024_m1_cold", time_single_cold)):
        try:  # a failure here must not cost the other lines
            out[key] = fn(dev, stream, pk)
        except Exception as e:  # noqa: BLE001
            out[key] = {"error": f"{type(e).__name__}: {e}"}
    # the same 2-bit sweep as twelve tl_gemv_ex calls per step (with and without PDL)
    sw = Sweep(2, dev)
    for flags, key in ((1, "gemv_2bit_sweep_per_call_pdl"), (0, "gemv_2bit_sweep_per_call")):
        ms, _, _ = time_graphs(sw, 45, 3, stream, flags=flags)
        gbs = sw.bytes_per_step * 45 / (ms * 1e-3) / 1e9
        out[key] = {"GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
                    "us_per_step": round(ms / 45 * 1e3, 2)}
    return out


def run_gpu(args):
    import torch
    rank, local_rank, world = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    from ternary_weight_03_b200 import build
    build.build()
    import ternary_weight_03_b200 as tl
    tl.lib()
    stream = torch.cuda.Stream(device=dev)
    pk = peaks()

    sweep = Sweep(2, dev)
    sweep.use_batch()
    total_ms, per_call, clocks = time_graphs(sweep, args.steps, args.warmup, stream,
                                             clock_gpu=local_rank)
    worst = check_outputs(sweep)
    max_ms, total_bytes = reduce_step_time(total_ms, sweep.bytes_per_step * args.steps)
    value = total_bytes / (max_ms * 1e-3) / 1e9
    # average launch duration over the timed region: the step is nothing but
    # the dominant kernel's launches (back to back, overlapping under PDL)
    avg_launch_ms = total_ms / (args.steps * sweep.launches_per_step)
    achieved = (sweep.bytes_per_step / sweep.launches_per_step) / (avg_launch_ms * 1e-3) / 1e9
    e2e_ms, h2d, d2h = time_e2e(sweep, max(1, min(args.steps, 5)), 1, stream)
    e2e_steps = max(1, min(args.steps, 5))
    e2e_max, e2e_bytes = reduce_step_time(e2e_ms, sweep.bytes_per_step * e2e_steps)
    traffic = traffic_per_launch()
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16 inputs, f32 accumulation",
        "data": "synthetic (seeded SplitMix64 trits and N(0,1) fp16 activations)",
        "config": {
            "workload": WORKLOAD,
            "packed_bytes_per_step": sweep.bytes_per_step,
            "layers_per_step": len(sweep.items) * len(sweep.ms),
            "launches_per_step": sweep.launches_per_step,
            "l2": f"inputs larger than L2: {sweep.copies} rotating copies of the packed "
                  f"matrices ({sweep.rotation_bytes / 2**20:.0f} MiB) so every call reads HBM",
            "timing": f"CUDA graphs of up to {GRAPH_STEPS} consecutive steps, CUDA events on "
                      "the launch stream",
            "launch": "one tl_gemv_batch_run per step (all 12 independent layers in one "
                      "persistent launch) with TL_FLAG_PDL",
            "parallelism": f"replicas x{world}",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "tlk::decode2_kernel",
            "achieved": round(achieved, 2),
            "peak": pk["hbm_gbs"],
            "unit": "GB/s",
            "frac": round(achieved / pk["hbm_gbs"], 4),
            "traffic": traffic,
            "algorithmic_bytes_per_launch": sweep.bytes_per_step // sweep.launches_per_step,
            "avg_launch_us": round(avg_launch_ms * 1e3, 3),
            "launch_us_without_pdl": [round(t * 1e3, 2) for t in per_call],
            "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({pk['source']})",
        },
        "e2e": {"value": round(e2e_bytes / (e2e_max * 1e-3) / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": sweep.launches_per_step * args.steps,
        "clocks": clocks,
        "max_err_over_tol": round(worst, 4),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if not args.no_secondary:
        try:  # context lines: an error there is recorded, the headline line still prints
            line["secondary"] = secondary(dev, stream)
        except Exception as e:  # noqa: BLE001
            line["secondary"] = {"error": f"{type(e).__name__}: {e}"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def traffic_per_launch():
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel sources (else None)."""
    p = ROOT / "profiles" / "decode2_sweep_traffic.json"
    if not p.exists():
        return None
    try:
        d = json.loads(p.read_text())
        import hashlib
        # the kernel's own sources: its header and the headers it includes
        h = hashlib.sha256()
        for f in d["sources"]:
            h.update((ROOT / f).read_bytes())
        if d.get("sources_sha256") != h.hexdigest():
            return None
        return d.get("dram_bytes_per_launch")
    except (OSError, ValueError, KeyError, TypeError):
        return None


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------
def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return
    import oracle
    import synth
    o = oracle.get()
    threads = os.cpu_count() or 1
    # each step: the first `rows` rows of every sweep matrix, both M, sized so
    # that warmup + steps take about a minute in total
    budget_s = 60.0 / max(1, args.steps + args.warmup)
    K, N = SWEEP[0]
    P, T, alpha = make_matrix(2, K, 64, 0, codec="oracle")
    X = synth.activations(0, 8, K)
    t0 = time.perf_counter()
    o.linear(o.unpack(2, P, K)[1], X, alpha, nthreads=threads)
    per = (time.perf_counter() - t0) / (64 * K * 8)
    frac = min(1.0, budget_s / max(per * sum(K * N for K, N in SWEEP) * sum(SWEEP_M), 1e-9))
    mats = []
    for i, (K, N) in enumerate(SWEEP):
        rows = min(N, max(threads, int(N * frac)))
        Pm, _, alpha = make_matrix(2, K, rows, i, codec="oracle")
        mats.append((K, rows, Pm, alpha, {M: synth.activations(i, M, K) for M in SWEEP_M}))
    step_bytes = sum(rows * ((K + 3) // 4) for (K, rows, _, _, _) in mats) * len(SWEEP_M)

    def step():
        for (K, rows, Pm, alpha, xs) in mats:
            for M in SWEEP_M:
                o.linear(o.unpack(2, Pm, K)[1], xs[M], alpha, nthreads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = step_bytes * args.steps / el / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (oracle)", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "sample": f"first rows {[m[1] for m in mats]} of each "
                   "matrix per step", "parallelism": "host threads"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"first rows {[m[1] for m in mats]} of each sweep matrix, "
                                   "both M, per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_single(fmt: int, K: int, N: int, M: int, reps: int = 4):
    """One seeded layer shape, `reps` calls through the C ABI (tl_gemv for
    M <= 8, tl_gemm otherwise), nothing else on the device."""
    import torch
    import synth
    import ternary_weight_03_b200 as tl
    from ternary_weight_03_b200 import build
    build.build()
    P, _, alpha = make_matrix(fmt, K, N, 0)
    dP = torch.from_numpy(P).cuda()
    X = torch.from_numpy(synth.activations(1, M, K)).cuda()
    for _ in range(reps):
        Y = tl.linear(fmt, dP, alpha, X, K)
    torch.cuda.synchronize()
    print(json.dumps({"single": [fmt, K, N, M], "checksum": float(Y.float().abs().sum())}))


def run_batch_once(fmt: int, M: int, reps: int = 3):
    """The six sweep shapes at M tokens planned as one batch and run `reps`
    times through tl_gemv_batch_run, nothing else on the device (for ncu)."""
    import torch
    import synth
    import ternary_weight_03_b200 as tl
    from ternary_weight_03_b200 import build
    build.build()
    specs = []
    for i, (K, N) in enumerate(SWEEP):
        P, _, alpha = make_matrix(fmt, K, N, i)
        specs.append((torch.from_numpy(P).cuda(), alpha,
                      torch.from_numpy(synth.activations(i, M, K)).cuda(), K,
                      torch.empty((M, N), dtype=torch.float16, device="cuda")))
    layers = tl.make_layers(fmt, specs)
    ws = torch.zeros(tl.gemv_batch_bytes(fmt, layers), dtype=torch.uint8, device="cuda")
    plan = tl.gemv_batch_plan(fmt, layers, ws)
    for _ in range(reps):
        tl.gemv_batch_run(plan)
    torch.cuda.synchronize()
    print(json.dumps({"batch_once": [fmt, M], "status": tl.device_status(),
                      "checksum": float(sum(sp[4].float().abs().sum() for sp in specs))}))


def run_ternarise_once(fmt: int, N: int, K: int, reps: int = 3):
    """tl_ternarise on one seeded N x K fp16 weight matrix, `reps` times,
    nothing else on the device (for ncu)."""
    import torch
    import ternary_weight_03_b200 as tl
    from ternary_weight_03_b200 import build
    build.build()
    g = torch.Generator(device="cuda").manual_seed(N * 7 + K)
    W = (torch.randn((N, K), generator=g, device="cuda") * 0.02).half()
    for _ in range(reps):
        P, alpha = tl.ternarise(fmt, W)
    torch.cuda.synchronize()
    print(json.dumps({"ternarise_once": [fmt, N, K], "alpha": float(alpha.item()),
                      "checksum": int(P.sum().item())}))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--batch-once", metavar="FMT,M",
                    help="plan the six sweep shapes at M tokens as one batch and run it 3 times "
                         "(a small case for profiling the batch kernel)")
    ap.add_argument("--single", metavar="FMT,K,N,M",
                    help="run one seeded layer call 4 times and exit (for ncu captures)")
    ap.add_argument("--ternarise-once", metavar="FMT,N,K",
                    help="ternarise one seeded N x K fp16 matrix 3 times and exit (for ncu)")
    args = ap.parse_args(argv)
    if args.ternarise_once:
        run_ternarise_once(*[int(v) for v in args.ternarise_once.split(",")])
        return
    if args.batch_once:
        run_batch_once(*[int(v) for v in args.batch_once.split(",")])
        return
    if args.single:
        run_single(*[int(v) for v in args.single.split(",")])
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
