"""Benchmark of the weight-only low-bit linear layer on B200.

Headline workload (one "step"): the Llama-3-8B-shaped ternary decode sweep -- 32 distinct layers
x 7 linears (q, k, v, o, gate, up, down) x M in {1, 4, 16} tokens, x ~ N(0,1) fp16, weights
~ N(0, 0.02) ternarised and packed by tq_quantize_pack (1.745 GB packed, larger than L2, so no
L2 flush is needed between steps).  Each layer and M is one tq_gemm_batch C-ABI call (its 7
linears in one persistent launch); the 96 calls of a step are captured in one CUDA graph.

metric: decode packed-weight GB/s (algorithmic bytes: packed weights + scales + x + y) ; the
other hot-path rows (prefill TFLOP/s, W4A16, pack) are measured after the headline step and
reported under "rows", each with its own roofline fraction.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--detail]

With N > 1 (torchrun), every rank runs the same per-GPU workload on its own seeded weights
(replicas, weak scaling; the path has no exchange step); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode packed-weight GB/s & prefill TFLOP/s vs B200 roofline (1 GPU)"
LLAMA = [("q_proj", 4096, 4096), ("k_proj", 1024, 4096), ("v_proj", 1024, 4096),
         ("o_proj", 4096, 4096), ("gate_proj", 14336, 4096), ("up_proj", 14336, 4096),
         ("down_proj", 4096, 14336)]
DECODE_M = (1, 4, 16)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def decode_bytes(M, N, K, bias=False):
    return N * K // 4 + 2 * N + 2 * M * K + 2 * M * N + (2 * N if bias else 0)


def w4g_decode_bytes(M, N, K):
    return N * K // 2 + 2 * N * (K // 128) + 2 * M * K + 2 * M * N


class ClockSampler:
    """Samples nvidia-smi clocks / throttle reasons while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.th = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()
        t0 = time.time()  # nvidia-smi takes a moment to start: wait for its first sample
        while not self.lines and time.time() - t0 < 3.0:
            time.sleep(0.02)
        self.lines.clear()  # keep only samples taken while the timed region runs

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # a timed region shorter than the sampling interval: take the first sample after it
        t0 = time.time()
        while not self.lines and time.time() - t0 < 0.5:
            time.sleep(0.005)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.th:
            self.th.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier_sync(world):
    import torch
    import torch.distributed as dist

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(v, world, device="cuda"):
    """Max of a per-rank scalar over all ranks (the job time is the slowest rank's)."""
    import torch
    import torch.distributed as dist

    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed_offset(rank: int) -> int:
    """Every replica packs its own, distinct weights (weak scaling over independent replicas)."""
    return 100003 * rank


def weak_scaling_value(bytes_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job GB/s: the bytes all ranks processed over the slowest rank's step time."""
    return bytes_per_rank * world / (ms_max * 1e-3) / 1e9


# ------------------------------------------------------------------------------------------------
# our implementation
# ------------------------------------------------------------------------------------------------
def build_ternary_layers(rank, n_layers, config=1, shapes=LLAMA, dtype=None):
    import torch

    import bit_weight_only_tq_b200 as tq
    import tq_inputs as I

    layers = []
    for l in range(n_layers):
        row = []
        for mid, (name, N, K) in enumerate(shapes):
            w = I.weights(N, K, I.seed_for(config, l, mid) + rank_seed_offset(rank), device="cuda")
            p, s = tq.tq_quantize_pack(w)
            row.append((name, N, K, p, s))
            del w
        layers.append(row)
    torch.cuda.synchronize()
    return layers


def layer_calls(gemm, grouped, row, xs, ys, bs=None):
    """The seven linears of one Llama layer as a serving engine issues them: q/k/v and gate/up
    each through one grouped call (they read the same x), o and down alone."""
    d = {name: (N, K, w, s) for name, N, K, w, s in row}

    def grp(names):
        grouped(xs[d[names[0]][1]], [d[n][2] for n in names], [d[n][3] for n in names],
                None if bs is None else [bs[d[n][0]] for n in names], [ys[n] for n in names])

    grp(("q_proj", "k_proj", "v_proj"))
    N, K, w, s = d["o_proj"]
    gemm(xs[K], w, s, None if bs is None else bs[N], ys["o_proj"])
    grp(("gate_proj", "up_proj"))
    N, K, w, s = d["down_proj"]
    gemm(xs[K], w, s, None if bs is None else bs[N], ys["down_proj"])


def capture(fn):
    import torch

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm-up (also sets kernel attributes outside capture)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, iters, warm=3):
    import torch

    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(True), torch.cuda.Event(True)
    a.record()
    for _ in range(iters):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def run_ours(args, world, rank, local):
    import torch

    import bit_weight_only_tq_b200 as tq
    import tq_inputs as I

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    n_layers = 32
    layers = build_ternary_layers(rank, n_layers)

    # inputs / outputs of a step: one x per (M, K); one output buffer per M (slices per GEMM)
    Ks = sorted({K for _, _, K in LLAMA})
    xs = {(M, K): I.activations(M, K, I.seed_for(1, 99, M) + K, device="cuda") for M in DECODE_M for K in Ks}
    out_cols = n_layers * sum(N for _, N, _ in LLAMA)
    ys = {M: torch.empty(M * out_cols, dtype=torch.float16, device="cuda") for M in DECODE_M}

    # y slices of one output buffer per M, in the order of LLAMA within each layer
    yv = {}
    for M in DECODE_M:
        off = 0
        for li in range(n_layers):
            for mid, (_, N, _) in enumerate(LLAMA):
                yv[(M, li, mid)] = ys[M][off: off + M * N].view(M, N)
                off += M * N

    def step_grouped():
        # per layer: q/k/v share x (one grouped launch), o, gate/up share x (grouped), down
        for M in DECODE_M:
            for li, row in enumerate(layers):
                P = [r[3] for r in row]
                S = [r[4] for r in row]
                Y = [yv[(M, li, j)] for j in range(len(row))]
                tq.tq_gemm_grouped(xs[(M, 4096)], P[0:3], S[0:3], None, Y[0:3])
                tq.tq_gemm(xs[(M, 4096)], P[3], S[3], None, Y[3])
                tq.tq_gemm_grouped(xs[(M, 4096)], P[4:6], S[4:6], None, Y[4:6])
                tq.tq_gemm(xs[(M, 14336)], P[6], S[6], None, Y[6])

    def step_separate():
        for M in DECODE_M:
            for li, row in enumerate(layers):
                for mid, (name, N, K, p, s) in enumerate(row):
                    tq.tq_gemm(xs[(M, K)], p, s, None, yv[(M, li, mid)])

    ws = tq.batch_workspace()
    # per layer and M: one persistent launch over the layer's 7 linears (each with its own x)
    batch_args = []
    for M in DECODE_M:
        for li, row in enumerate(layers):
            X = [xs[(M, K)] for (_, _, K, _, _) in row]
            P = [r[3] for r in row]
            S = [r[4] for r in row]
            Y = [yv[(M, li, j)] for j in range(len(row))]
            batch_args.append((X, P, S, Y))

    # every call names the call after it (the first of the next step after the last), whose
    # first weight tiles it prefetches into L2 (tq_gemm_batch_next)
    def step_batch():
        for i, (X, P, S, Y) in enumerate(batch_args):
            Xn, Pn, _, _ = batch_args[(i + 1) % len(batch_args)]
            tq.tq_gemm_batch(X, P, S, None, Y, workspace=ws, next_packed=Pn, next_M=Xn[0].shape[0])

    steps = {"batch": (step_batch, 1), "grouped": (step_grouped, 4), "separate": (step_separate, len(LLAMA))}
    step_fn, per_layer = steps[args.calls]

    bytes_step = sum(decode_bytes(M, N, K) for M in DECODE_M for _ in range(n_layers) for _, N, K in LLAMA)
    launches_step = len(DECODE_M) * n_layers * per_layer
    g = capture(step_fn)
    for _ in range(args.warmup):
        g.replay()
    barrier_sync(world)
    clk = ClockSampler(local)
    clk.start()
    ev0, ev1 = torch.cuda.Event(True), torch.cuda.Event(True)
    ev0.record()
    for _ in range(args.steps):
        g.replay()
    ev1.record()
    barrier_sync(world)
    clocks = clk.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, world)
    value = weak_scaling_value(bytes_step, world, ms_max)

    # end-to-end through the public API: pinned-host x in, y out, every step
    h_x = {k: v.cpu().pin_memory() for k, v in xs.items()}
    h_y = {M: torch.empty(ys[M].numel(), dtype=torch.float16).pin_memory() for M in DECODE_M}
    bi = sum(v.numel() * 2 for v in h_x.values())
    bo = sum(v.numel() * 2 for v in h_y.values())

    # one CUDA graph: x copied in, then the step's calls, the largest M first; the outputs of
    # every 8 layers are copied out on a second stream while the next 8 layers compute (only the
    # last chunk's copy, M = 1, is not hidden), and the step ends when every copy has landed
    copy_stream = torch.cuda.Stream()
    chunk = 8
    per_m = len(batch_args) // len(DECODE_M) if args.calls == "batch" else 0
    # the end-to-end order (largest M first): the index of the call that follows each call
    e2e_order = [mi * per_m + li for mi in reversed(range(len(DECODE_M))) for li in range(per_m)]
    e2e_next = {a: e2e_order[(i + 1) % len(e2e_order)] for i, a in enumerate(e2e_order)}

    def e2e_fn():
        cs = torch.cuda.current_stream()
        for k, v in h_x.items():
            xs[k].copy_(v, non_blocking=True)
        if args.calls != "batch":
            step_fn()
            for M in DECODE_M:
                h_y[M].copy_(ys[M], non_blocking=True)
            return
        cols = out_cols // n_layers
        for mi, M in reversed(list(enumerate(DECODE_M))):
            for l0 in range(0, n_layers, chunk):
                l1 = min(l0 + chunk, n_layers)
                for li in range(l0, l1):
                    X, P, S, Y = batch_args[mi * per_m + li]
                    Xn, Pn, _, _ = batch_args[e2e_next[mi * per_m + li]]
                    tq.tq_gemm_batch(X, P, S, None, Y, workspace=ws, next_packed=Pn, next_M=Xn[0].shape[0])
                ev = torch.cuda.Event()
                ev.record(cs)
                copy_stream.wait_event(ev)
                a, b = l0 * M * cols, l1 * M * cols
                with torch.cuda.stream(copy_stream):
                    h_y[M][a:b].copy_(ys[M][a:b], non_blocking=True)
        cs.wait_stream(copy_stream)

    g_e2e = capture(e2e_fn)

    def e2e_step():
        g_e2e.replay()

    for _ in range(2):
        e2e_step()
    barrier_sync(world)
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    e0.record()
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    barrier_sync(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    e2e_val = weak_scaling_value(bytes_step, world, e2e_ms)

    # the same, with every GEMM call issued eagerly through the C ABI (argument checks, tensor
    # map encoding and the launch itself on the host inside the timed region), no CUDA graph
    eager_calls = step_fn
    if args.calls == "batch":
        # the C ABI called directly with prebuilt descriptor arrays: the timed host work is the
        # library's own (argument checks, tensor-map encoding, launch), not Python marshalling
        import ctypes

        stream_h = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        prebuilt = []
        for X, P, S, Y in batch_args:
            arr = (tq.TqLinear * len(P))()
            for j in range(len(P)):
                arr[j] = tq.TqLinear(X[j].data_ptr(), P[j].data_ptr(), S[j].data_ptr(), None, Y[j].data_ptr(),
                                     P[j].shape[0], X[j].shape[1])
            prebuilt.append((arr, len(P), X[0].shape[0]))
        ws_p, ws_n = ctypes.c_void_p(ws.data_ptr()), ws.numel()
        # each call with the call after it in that order (tq_gemm_batch_next)
        def batch_call(a, nxt):
            arr, n, M = prebuilt[a]
            narr, nn, nM = prebuilt[nxt]
            return tq.lib.tq_gemm_batch_next(arr, n, M, ws_p, ws_n, 0, narr, nn, nM, stream_h)

        def eager_calls():
            for a in range(len(prebuilt)):
                st = batch_call(a, (a + 1) % len(prebuilt))
                if st != 0:
                    raise RuntimeError(tq.tq_status_string(st))

    def e2e_eager_step():
        for k, v in h_x.items():
            xs[k].copy_(v, non_blocking=True)
        if args.calls != "batch":
            eager_calls()
            for M in DECODE_M:
                h_y[M].copy_(ys[M], non_blocking=True)
            return
        # as in the graph: largest M first, outputs of every 8 layers copied out on the second
        # stream under the next layers' calls
        cs = torch.cuda.current_stream()
        cols = out_cols // n_layers
        for mi, M in reversed(list(enumerate(DECODE_M))):
            for l0 in range(0, n_layers, chunk):
                l1 = min(l0 + chunk, n_layers)
                for a in range(mi * per_m + l0, mi * per_m + l1):
                    st = batch_call(a, e2e_next[a])
                    if st != 0:
                        raise RuntimeError(tq.tq_status_string(st))
                ev = torch.cuda.Event()
                ev.record(cs)
                copy_stream.wait_event(ev)
                a, b = l0 * M * cols, l1 * M * cols
                with torch.cuda.stream(copy_stream):
                    h_y[M][a:b].copy_(ys[M][a:b], non_blocking=True)
        cs.wait_stream(copy_stream)

    for _ in range(2):
        e2e_eager_step()
    barrier_sync(world)
    n_eager = max(3, min(args.steps, 50))
    e0.record()
    for _ in range(n_eager):
        e2e_eager_step()
    e1.record()
    barrier_sync(world)
    eager_ms = max_over_ranks(e0.elapsed_time(e1) / n_eager, world)
    eager_val = weak_scaling_value(bytes_step, world, eager_ms)

    # roofline of the dominant kernel (the decode GEMM is every launch of the step)
    per_launch_us = ms * 1e3 / launches_step
    achieved = bytes_step / launches_step / (per_launch_us * 1e-6) / 1e9
    traffic = load_traffic()
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "traffic": traffic,
            "kernel": "batch_decode_kernel" if args.calls == "batch" else "decode_gemm_kernel",
            "peak_source": f"{peak_src} hbm_gbs"}

    detail = {}
    if args.detail and rank == 0:
        detail = per_shape_detail(layers, xs)

    rows = {}
    samples = {"batch": "one tq_gemm_batch launch per layer (7 linears)",
               "grouped": "per layer: grouped q/k/v, o, grouped gate/up, down (4 launches)",
               "separate": "7 single-matrix tq_gemm calls per layer"}
    for other in ("batch", "grouped", "separate"):
        if other == args.calls:
            continue
        g2 = capture(steps[other][0])
        ms2 = time_graph(g2, max(3, min(args.steps, 20)))
        del g2
        rows[f"ternary_decode_{other}"] = {
            "value": round(bytes_step / (ms2 * 1e-3) / 1e9, 1), "unit": "GB/s",
            "frac": round(bytes_step / (ms2 * 1e-3) / 1e9 / hbm, 4), "peak": hbm, "bound": "hbm",
            "ms_per_step": round(ms2, 4), "sample": "same sweep, " + samples[other]}
    if not args.no_rows:
        rows.update(secondary_rows(args, rank, layers, peaks))

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded N(0,0.02) weights ternarised on the GPU; x ~ N(0,1) fp16)",
        "config": dict(decode_config(args, world), launches_per_step=launches_step),
        "roofline": roof,
        "e2e": {"value": round(e2e_val, 1), "unit": "GB/s", "h2d_bytes_per_step": bi,
                "d2h_bytes_per_step": bo, "ms_per_step": round(e2e_ms, 4),
                "calls": ("graph; y of each 8 layers copied out on a 2nd stream under the next"
                          if args.calls == "batch" else "graph replay"),
                "eager_value": round(eager_val, 1), "eager_ms_per_step": round(eager_ms, 4)},
        "gpu_launches": launches_step * args.steps,
        "clocks": clocks,
        "rows": rows,
    }
    if detail:
        result["detail"] = detail
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    return result


def per_shape_detail(layers, xs):
    import torch

    import bit_weight_only_tq_b200 as tq

    out = {}
    for mid, (name, N, K) in enumerate(LLAMA):
        for M in DECODE_M:
            y = torch.empty(M, N, dtype=torch.float16, device="cuda")

            def fn():
                for row in layers:
                    _, _, _, p, s = row[mid]
                    tq.tq_gemm(xs[(M, K)], p, s, None, y)

            g = capture(fn)
            ms = time_graph(g, 10)
            per = ms * 1e3 / len(layers)
            ent = {"us": round(per, 2), "GB/s": round(decode_bytes(M, N, K) / (per * 1e-6) / 1e9, 1)}
            del g
            # the same matrices, eight layers' copies per tq_gemm_batch launch (4 launches)
            ys8 = [torch.empty(M, N, dtype=torch.float16, device="cuda") for _ in range(8)]
            ws = tq.batch_workspace()

            def fb():
                for l0 in range(0, len(layers), 8):
                    grp = layers[l0:l0 + 8]
                    tq.tq_gemm_batch([xs[(M, K)]] * len(grp), [r[mid][3] for r in grp], [r[mid][4] for r in grp],
                                     None, ys8[:len(grp)], workspace=ws)

            g = capture(fb)
            ms = time_graph(g, 10)
            per = ms * 1e3 / len(layers)
            ent["batch8_us"] = round(per, 2)
            ent["batch8_GB/s"] = round(decode_bytes(M, N, K) / (per * 1e-6) / 1e9, 1)
            ent["hbm_floor_us"] = round(decode_bytes(M, N, K) / (float(load_peaks()[0]["hbm_gbs"]) * 1e3), 2)
            out[f"{name} M={M}"] = ent
            del g
    return out


def secondary_rows(args, rank, layers, peaks):
    """One measurement per remaining hot-path row (prefill, W4A16, pack), each timed on the GPU
    with CUDA events over several launches of the public API."""
    import torch

    import bit_weight_only_tq_b200 as tq
    import tq_inputs as I

    hbm = float(peaks["hbm_gbs"])
    tc = float(peaks["bf16_tflops"])
    rows = {}
    # ---- ternary prefill (config 2): 4 layers x 7 shapes, M in {2048, 512, 8192}, bias, outlier
    # tokens
    bs = {N: I.bias(N, I.seed_for(2, 1, N), device="cuda") for N in (1024, 4096, 14336)}
    sub = layers[:4]
    for M in (2048, 512, 8192):
        xs = {K: I.activations(M, K, I.seed_for(2, 0, K), device="cuda", outlier_row_frac=0.01)
              for K in (4096, 14336)}
        ys = {name: torch.empty(M, N, dtype=torch.float16, device="cuda") for name, N, _ in LLAMA}

        def pf():
            for row in sub:
                layer_calls(tq.tq_gemm, tq.tq_gemm_grouped, row, xs, ys, bs)

        g = capture(pf)
        ms = time_graph(g, 10)
        flops = sum(2 * M * N * K for row in sub for _, N, K, _, _ in row)
        tf = flops / (ms * 1e-3) / 1e12
        rows[f"ternary_prefill_M{M}"] = {"value": round(tf, 1), "unit": "TFLOP/s", "frac": round(tf / tc, 4),
                                         "peak": tc, "bound": "tensor",
                                         "sample": f"4 layers x 7 shapes, M={M}; q/k/v and gate/up grouped"}
        del g, xs, ys
    # ---- W4A16 pack (config 3 weights, fp32): 2 layers x 7 shapes, 1.75 GB read
    wf = [[I.weights(N, K, I.seed_for(3, l, mid) + rank_seed_offset(rank), device="cuda", outlier_frac=0.001)
           for mid, (name, N, K) in enumerate(LLAMA)] for l in range(2)]
    po = [[(torch.empty(N, K // 8, dtype=torch.int32, device="cuda"),
            torch.empty(N, K // 128, dtype=torch.float16, device="cuda")) for (name, N, K) in LLAMA] for _ in range(2)]

    def pack4():
        for l in range(2):
            for mid in range(len(LLAMA)):
                tq.w4g_quantize_pack(wf[l][mid], po[l][mid][0], po[l][mid][1])

    pack4()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(True), torch.cuda.Event(True)
    a.record()
    pack4()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    byts = 2 * sum(N * K * 4 + N * K // 2 + 2 * N * (K // 128) for _, N, K in LLAMA)
    gbs = byts / (ms * 1e-3) / 1e9
    rows["w4g_quantize_pack_llama_fp32"] = {"value": round(gbs, 1), "unit": "GB/s", "frac": round(gbs / hbm, 4),
                                            "peak": hbm, "bound": "hbm", "ms": round(ms, 3),
                                            "sample": f"2 Llama-3-8B layers x 7 shapes, fp32 in "
                                                      f"({byts / 1e9:.2f} GB moved), inputs larger than L2"}
    del wf, po
    # ---- W4A16 decode / prefill (config 3): 8 layers
    w4 = []
    for l in range(8):
        row = []
        for mid, (name, N, K) in enumerate(LLAMA):
            w = I.weights(N, K, I.seed_for(3, l, mid) + rank_seed_offset(rank), device="cuda", outlier_frac=0.001)
            qw, sc = tq.w4g_quantize_pack(w)
            row.append((name, N, K, qw, sc))
            del w
        w4.append(row)
    ws = tq.batch_workspace()
    for M in (1, 16):
        xq = {K: I.activations(M, K, I.seed_for(3, 2, K) + M, device="cuda") for K in (4096, 14336)}
        yq = {N: torch.empty(M, N, dtype=torch.float16, device="cuda") for N in (1024, 4096, 14336)}

        def wd():  # one w4g_gemm_batch launch per layer (its 7 linears), each naming the next
            for li, row in enumerate(w4):
                nxt = w4[(li + 1) % len(w4)]
                tq.w4g_gemm_batch([xq[K] for _, _, K, _, _ in row], [r[3] for r in row], [r[4] for r in row],
                                  None, [yq[N] for _, N, _, _, _ in row], workspace=ws,
                                  next_qweight=[r[3] for r in nxt], next_M=M)

        def wc():  # one w4g_gemm call per linear
            for row in w4:
                for name, N, K, qw, sc in row:
                    tq.w4g_gemm(xq[K], qw, sc, None, yq[N])

        byts = sum(w4g_decode_bytes(M, N, K) for row in w4 for _, N, K, _, _ in row)
        for key, fn, what in ((f"w4g_decode_M{M}", wd, "one batch launch per layer"),
                              (f"w4g_decode_M{M}_calls", wc, "one call per linear")):
            g = capture(fn)
            ms = time_graph(g, 20)
            gbs = byts / (ms * 1e-3) / 1e9
            rows[key] = {"value": round(gbs, 1), "unit": "GB/s", "frac": round(gbs / hbm, 4),
                         "peak": hbm, "bound": "hbm", "sample": f"8 layers x 7 shapes, {what}"}
            del g
    for M, wl in ((4096, w4[:1]), (256, w4)):
        xq = {K: I.activations(M, K, I.seed_for(3, 3, K), device="cuda") for K in (4096, 14336)}
        yq = {name: torch.empty(M, N, dtype=torch.float16, device="cuda") for name, N, _ in LLAMA}

        def wp():
            for row in wl:
                layer_calls(tq.w4g_gemm, tq.w4g_gemm_grouped, row, xq, yq)

        g = capture(wp)
        ms = time_graph(g, 10)
        flops = sum(2 * M * N * K for row in wl for _, N, K, _, _ in row)
        tf = flops / (ms * 1e-3) / 1e12
        rows[f"w4g_prefill_M{M}"] = {"value": round(tf, 1), "unit": "TFLOP/s", "frac": round(tf / tc, 4),
                                     "peak": tc, "bound": "tensor",
                                     "sample": f"{len(wl)} layer{'s' if len(wl) > 1 else ''} x 7 shapes, M={M}; "
                                               "q/k/v and gate/up grouped"}
        del g, xq, yq
    del w4
    # ---- config 0: one ternary linear 1024x1024 at M = 1 (L2-resident: the time of one call)
    w = I.weights(1024, 1024, I.seed_for(0, 0, 0), device="cuda")
    p0, s0 = tq.tq_quantize_pack(w)
    del w
    x0 = I.activations(1, 1024, I.seed_for(0, 0, 0), device="cuda")
    y0 = torch.empty(1, 1024, dtype=torch.float16, device="cuda")
    g = capture(lambda: [tq.tq_gemm(x0, p0, s0, None, y0) for _ in range(32)])
    ms = time_graph(g, 20) / 32
    rows["config0_decode_1024x1024_M1"] = {"value": round(ms * 1e3, 2), "unit": "us/call",
                                           "sample": "32 calls in a CUDA graph; weights L2-resident (256 KiB), "
                                                     "so no roofline fraction"}
    del g
    # ---- config 4: Qwen2-7B, 28 layers x {qkv 4608x3584, o 3584x3584, gate_up 37888x3584,
    # down 3584x18944}: tq_quantize_pack of all fp16 weights (13.05 GB read), then the M sweep
    qshapes = [(4608, 3584), (3584, 3584), (37888, 3584), (3584, 18944)]
    nl = 28
    wq = [[I.weights(N, K, I.seed_for(4, l, mid) + rank_seed_offset(rank), device="cuda", dtype=torch.float16)
           for mid, (N, K) in enumerate(qshapes)] for l in range(nl)]
    pq = [[(torch.empty(N, K // 4, dtype=torch.uint8, device="cuda"), torch.empty(N, dtype=torch.float16, device="cuda"))
           for (N, K) in qshapes] for _ in range(nl)]

    def pack_all():
        for l in range(nl):
            for mid in range(len(qshapes)):
                tq.tq_quantize_pack(wq[l][mid], pq[l][mid][0], pq[l][mid][1])

    pack_all()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(True), torch.cuda.Event(True)
    a.record()
    pack_all()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    byts = nl * sum(N * K * 2 + N * K // 4 + 2 * N for N, K in qshapes)
    gbs = byts / (ms * 1e-3) / 1e9
    rows["tq_quantize_pack_qwen2_fp16"] = {"value": round(gbs, 1), "unit": "GB/s", "frac": round(gbs / hbm, 4),
                                           "peak": hbm, "bound": "hbm", "ms": round(ms, 3),
                                           "sample": f"all {nl} Qwen2-7B layers x 4 shapes, fp16 in "
                                                     f"({byts / 1e9:.2f} GB moved), inputs larger than L2"}
    del wq
    sweep = {}
    for M in (1, 2, 8, 32, 128, 512, 2048, 8192):
        xk = {K: I.activations(M, K, I.seed_for(4, 99, M) + K, device="cuda") for K in (3584, 18944)}
        yn = {N: torch.empty(M, N, dtype=torch.float16, device="cuda") for N, _ in qshapes}

        def qs():
            for l in range(nl):
                for mid, (N, K) in enumerate(qshapes):
                    tq.tq_gemm(xk[K], pq[l][mid][0], pq[l][mid][1], None, yn[N])

        g = capture(qs)
        ms = time_graph(g, 10)
        byts = nl * sum(decode_bytes(M, N, K) for N, K in qshapes)
        flops = nl * sum(2 * M * N * K for N, K in qshapes)
        t_att = max(byts / (hbm * 1e9), flops / (tc * 1e12)) * 1e3  # ms at the attainable roofline
        ent = {"ms": round(ms, 4), "GB/s": round(byts / (ms * 1e-3) / 1e9, 1),
               "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1), "attainable_frac": round(t_att / ms, 4),
               "path": "decode" if tq.tq_select_path(0, M, 3584, 3584, 1) == tq.PATH_DECODE else "prefill"}
        sweep[f"M{M}"] = ent
        del g, xk, yn
    rows["qwen2_sweep_28_layers"] = {"unit": "per M: ms for 28 layers x 4 shapes; attainable_frac = "
                                             "max(bytes / HBM, flops / fp16 peak) / time", "values": sweep}
    rows["dispatch_crossover_qwen2"] = dispatch_crossover(tq, I, pq[:8], qshapes)
    del pq
    torch.cuda.synchronize()
    return rows


def dispatch_crossover(tq, I, pq, qshapes):
    """Both GEMM paths forced at M around the ridge, on Qwen2-7B shapes (ternary: the given
    packed layers; W4A16: four layers packed here), to place the automatic decode/prefill
    switch by measurement."""
    import torch

    nl = len(pq)
    p4 = []
    for l in range(4):
        row = []
        for mid, (N, K) in enumerate(qshapes):
            w = I.weights(N, K, I.seed_for(4, 50 + l, mid), device="cuda", outlier_frac=0.001)
            row.append(tq.w4g_quantize_pack(w))
            del w
        p4.append(row)
    out = {"unit": "ms per pass (ternary: %d layers, W4A16: 4 layers) x 4 shapes" % nl, "values": {}}
    for M in (16, 24, 32, 40, 48, 64):
        xk = {K: I.activations(M, K, I.seed_for(4, 98, M) + K, device="cuda") for K in (3584, 18944)}
        yn = {N: torch.empty(M, N, dtype=torch.float16, device="cuda") for N, _ in qshapes}
        ent = {}
        for fmt, layers, fn in (("ternary", pq, tq.tq_gemm), ("w4g", p4, tq.w4g_gemm)):
            for name, path in (("decode", tq.PATH_DECODE), ("prefill", tq.PATH_PREFILL)):
                def run():
                    for lay in layers:
                        for mid, (N, K) in enumerate(qshapes):
                            fn(xk[K], lay[mid][0], lay[mid][1], None, yn[N], path=path)

                g = capture(run)
                ent[f"{fmt}_{name}_ms"] = round(time_graph(g, 10), 4)
                del g
            fcode = 0 if fmt == "ternary" else 1
            ent[f"{fmt}_auto"] = "decode" if tq.tq_select_path(fcode, M, 3584, 3584, 1) == tq.PATH_DECODE else "prefill"
        out["values"][f"M{M}"] = ent
        del xk, yn
    del p4
    return out


TRAFFIC_SOURCES = ("tq_batch.cu", "tq_decode.cu", "tq_ptx.cuh", "tq_common.cuh")


def kernel_source_sha():
    """SHA-256 over the sources of the batch decode kernel (the headline's dominant kernel)."""
    import hashlib

    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "bit_weight_only_tq_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def load_traffic():
    """DRAM bytes per batch-decode launch from the committed ncu summary, only if it was taken on
    this kernel source (the summary records the SHA-256 of the kernel's source files)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        sha = kernel_source_sha()
    except (OSError, ValueError):
        return None
    if d.get("kernel_source_sha256") != sha:
        return None
    return d.get("batch_decode_bytes_per_launch")


# ------------------------------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ------------------------------------------------------------------------------------------------
def decode_config(args, world):
    """`config` of the headline decode workload (both arms)."""
    return {"workload": "Llama-3-8B-shaped ternary decode linears, 32 layers x {q,k,v,o,gate,up,down} "
                        "x M in {1,4,16}",
            "calls": {"batch": "per layer and M: one tq_gemm_batch launch over its 7 linears",
                      "grouped": "per layer: grouped q/k/v, o, grouped gate/up, down",
                      "separate": "7 tq_gemm per layer"}[args.calls],
            "layers": 32, "M": list(DECODE_M),
            "bytes_per_step": sum(decode_bytes(M, N, K) for M in DECODE_M for _ in range(32) for _, N, K in LLAMA),
            "l2": "inputs > L2 (1.745 GB packed)",
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
            "graph": "one CUDA graph per step, PDL"}


ORACLE_SAMPLE_ROWS = 1024


def oracle_sample_setup():
    """The bounded sample of the decode workload the oracle is timed on: the first 1024 output
    rows of each layer-0 Llama linear (q, k, v, o, gate, up, down), packed by the oracle."""
    import oracle as O
    import tq_inputs as I

    mats = []
    for mid, (name, N, K) in enumerate(LLAMA):
        w = I.weights(N, K, I.seed_for(1, 0, mid))[:ORACLE_SAMPLE_ROWS].numpy()
        p, s = O.tq_quantize_pack(w)
        mats.append((name, min(N, ORACLE_SAMPLE_ROWS), K, p, s))
    xs = {(M, K): I.activations(M, K, 1).numpy() for M in DECODE_M for K in {4096, 14336}}
    return mats, xs


def oracle_sample_run(sample, seconds, start=0):
    """Oracle tq_gemm at M = 1, 4, 16 over the sample's linears, cycled until `seconds` of GEMM
    time (at least one call). Returns (bytes, seconds, calls)."""
    import oracle as O

    mats, xs = sample
    done_b, gemm_time, n_items = 0, 0.0, 0
    while gemm_time < seconds or n_items == 0:
        i = start + n_items
        name, N, K, p, s = mats[i % len(mats)]
        M = DECODE_M[(i // len(mats)) % len(DECODE_M)]
        t1 = time.perf_counter()
        O.tq_gemm(xs[(M, K)], p, s, None, K)
        gemm_time += time.perf_counter() - t1
        done_b += decode_bytes(M, N, K)
        n_items += 1
    return done_b, gemm_time, n_items


def oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_baseline(seconds=12.0):
    """The oracle as it stands, on the host cores, on the bounded sample of the decode workload
    (`oracle_sample_setup`), timed for `seconds` of GEMM; then a quarter of that time with the
    BLAS pool limited to one thread (the single-core figure)."""
    sample = oracle_sample_setup()
    done_b, gemm_time, n_items = oracle_sample_run(sample, seconds)
    out = {"value": round(done_b / gemm_time / 1e9, 4), "unit": "GB/s", "cores": oracle_cores(), "kind": "oracle",
           "sample": f"{n_items} oracle tq_gemm calls on the first {ORACLE_SAMPLE_ROWS} output rows of each "
                     f"layer-0 Llama linear, M cycling 1/4/16 ({gemm_time:.1f} s of GEMM)"}
    try:
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=1):
            b1, t1, n1 = oracle_sample_run(sample, seconds / 4)
        out["single_core_value"] = round(b1 / t1 / 1e9, 4)
    except Exception:  # noqa: BLE001  (threadpoolctl missing: no single-core figure)
        pass
    return out


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle timed on this host on the GPU arm's metric and config; each
    step is a bounded sample of the workload (oracle GEMMs on the sample of `oracle_sample_setup`),
    sized so that warm-up + timed steps take about `--cpu-seconds` of GEMM in total."""
    t0 = time.perf_counter()
    sample = oracle_sample_setup()
    per_step_s = min(2.0, max(0.02, args.cpu_seconds / max(1, args.steps + args.warmup)))
    tot_b, tot_s, calls, step_ms = 0, 0.0, 0, []
    for i in range(args.warmup + args.steps):
        b, sec, n = oracle_sample_run(sample, per_step_s, start=calls)
        calls += n
        if i >= args.warmup:
            tot_b += b
            tot_s += sec
            step_ms.append(sec * 1e3)
    val = round(tot_b / tot_s / 1e9, 4) if tot_s > 0 else 0.0
    timed_calls = calls
    return {
        "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(statistics.median(step_ms), 3) if step_ms else None,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeds as the GPU arm)",
        "config": decode_config(args, world),
        "impl": "reference",
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": oracle_cores(), "kind": "oracle",
                         "sample": f"each step: oracle tq_gemm calls for ~{per_step_s:.2f} s on the first "
                                   f"{ORACLE_SAMPLE_ROWS} output rows of each layer-0 Llama linear, M cycling "
                                   f"1/4/16 ({timed_calls} calls in warm-up and timed steps)"},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t0, 1),
    }


# ------------------------------------------------------------------------------------------------
# small fixed cases for profiler captures (a few launches each, a few GB on the device at most)
# ------------------------------------------------------------------------------------------------
PROFILE_CASES = {
    "decode": "ternary gate_proj 14336x4096 at M=1, 3 launches; q/k/v group (4096+1024+1024)x4096 at M=16, 3 launches",
    "prefill": "ternary q_proj 4096x4096 at M=2048 (1 % outlier rows), 3 launches; W4A16 gate+up (2x14336)x4096 "
               "grouped at M=256, 3 launches; ternary q/k/v (4096+1024+1024)x4096 grouped at M=512, 3 launches",
    "pack": "tq_quantize_pack of an fp16 Qwen2-7B gate_up 37888x3584 (2 launches) and an fp32 4096x4096 (2 launches); w4g_quantize_pack of the latter (2 launches)",
    "prefill_mid": "ternary Qwen2-7B down 3584x18944 at M=128, 3 launches; gate_up 37888x3584 at M=32, 3 launches",
    "batch": "tq_gemm_batch over the 7 ternary linears of a Llama-3-8B layer (54.5 MB packed; four layers in "
             "turn, 218 MB, each call naming the next) at M=1, 6 launches; then at M=16, 6 launches",
    "w4g_batch": "w4g_gemm_batch over one Llama-3-8B layer's 7 W4A16 linears (109 MB) at M=1, 3 launches; "
                 "then at M=16, 3 launches",
}


def run_profile_case(name):
    import torch

    import bit_weight_only_tq_b200 as tq
    import tq_inputs as I

    if name == "decode":
        w = I.weights(14336, 4096, 1, device="cuda")
        p, s = tq.tq_quantize_pack(w)
        del w
        x = I.activations(1, 4096, 2, device="cuda")
        for _ in range(3):
            tq.tq_gemm(x, p, s)
        ws = [tq.tq_quantize_pack(I.weights(N, 4096, 3 + i, device="cuda")) for i, N in enumerate((4096, 1024, 1024))]
        x16 = I.activations(16, 4096, 4, device="cuda")
        for _ in range(3):
            tq.tq_gemm_grouped(x16, [a for a, _ in ws], [b for _, b in ws])
    elif name == "prefill":
        w = I.weights(4096, 4096, 1, device="cuda")
        p, s = tq.tq_quantize_pack(w)
        del w
        x = I.activations(2048, 4096, 2, device="cuda", outlier_row_frac=0.01)
        for _ in range(3):
            tq.tq_gemm(x, p, s)
        gu = []
        for i in range(2):
            w = I.weights(14336, 4096, 5 + i, device="cuda")
            gu.append(tq.w4g_quantize_pack(w))
            del w
        x = I.activations(256, 4096, 6, device="cuda")
        for _ in range(3):
            tq.w4g_gemm_grouped(x, [q for q, _ in gu], [sc for _, sc in gu])
        qkv = []
        for i, N in enumerate((4096, 1024, 1024)):
            w = I.weights(N, 4096, 8 + i, device="cuda")
            qkv.append(tq.tq_quantize_pack(w))
            del w
        x = I.activations(512, 4096, 9, device="cuda", outlier_row_frac=0.01)
        for _ in range(3):
            tq.tq_gemm_grouped(x, [p for p, _ in qkv], [sc for _, sc in qkv])
    elif name == "prefill_mid":
        w = I.weights(3584, 18944, 1, device="cuda")
        p, s = tq.tq_quantize_pack(w)
        del w
        x = I.activations(128, 18944, 2, device="cuda")
        for _ in range(3):
            tq.tq_gemm(x, p, s)
        w = I.weights(37888, 3584, 3, device="cuda")
        p2, s2 = tq.tq_quantize_pack(w)
        del w
        x2 = I.activations(32, 3584, 4, device="cuda")
        for _ in range(3):
            tq.tq_gemm(x2, p2, s2)
    elif name in ("batch", "w4g_batch"):
        int4 = name == "w4g_batch"
        ws = tq.batch_workspace()
        nl = 1 if int4 else 4
        layers = []
        for li in range(nl):
            mats = []
            for mid, (_, N, K) in enumerate(LLAMA):
                w = I.weights(N, K, 10 + 7 * li + mid, device="cuda", outlier_frac=0.001 if int4 else 0.0)
                mats.append((tq.w4g_quantize_pack(w) if int4 else tq.tq_quantize_pack(w)) + (K,))
                del w
            layers.append(mats)
        calls = [(M, i % nl) for M in (1, 16) for i in range(3)] if int4 else \
            [(1 if i < 6 else 16, i % nl) for i in range(12)]
        xs = {(M, K): I.activations(M, K, 20 + K, device="cuda") for M in (1, 16) for K in (4096, 14336)}
        for i, (M, li) in enumerate(calls):
            mats = layers[li]
            args3 = ([xs[(M, K)] for _, _, K in mats], [p for p, _, _ in mats], [s for _, s, _ in mats])
            if int4:
                tq.w4g_gemm_batch(*args3, workspace=ws)
            else:
                nxt = calls[i + 1] if i + 1 < len(calls) else None
                tq.tq_gemm_batch(*args3, workspace=ws, next_packed=None if nxt is None else
                                 [p for p, _, _ in layers[nxt[1]]], next_M=0 if nxt is None else nxt[0])
    elif name == "pack":
        w = I.weights(37888, 3584, 1, device="cuda", dtype=torch.float16)
        for _ in range(2):
            tq.tq_quantize_pack(w)
        w = I.weights(4096, 4096, 2, device="cuda")
        for _ in range(2):
            tq.tq_quantize_pack(w)
        for _ in range(2):
            tq.w4g_quantize_pack(w)
    torch.cuda.synchronize()
    assert tq.tq_device_status() == 0
    print(f"profile case {name} done: {PROFILE_CASES[name]}", flush=True)


DATASHEET_TFLOPS = 2250.0  # B200 dense fp16/bf16 tensor peak (NVIDIA datasheet), secondary fraction


def compact_rows(rows):
    """Each secondary row as [value, unit, fraction of the measured peak] (tensor rows add the
    fraction of the datasheet peak); the Qwen2 sweep as its attainable fraction per M."""
    out = {}
    for k, v in rows.items():
        if "values" in v and k.startswith("qwen2_sweep"):
            out["qwen2_sweep_att_frac"] = {m[1:]: e["attainable_frac"] for m, e in v["values"].items()}
        elif "values" in v:
            continue  # long tables (crossover) stay in the stderr record
        else:
            e = [v.get("value"), v.get("unit")]
            if "frac" in v:
                e.append(v["frac"])
            if v.get("bound") == "tensor":
                e.append(round(v["value"] / DATASHEET_TFLOPS, 4))
            out[k] = e
    return out


def compact_result(res):
    r = dict(res)
    if "rows" in r:
        r["rows"] = compact_rows(r["rows"])
        r["rows_format"] = "[value, unit, frac of measured peak(, frac of datasheet 2250 TF/s)]"
    r.pop("detail", None)
    return r


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=sorted(PROFILE_CASES),
                    help="run one small fixed case for a profiler capture and exit (no timing)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--detail", action="store_true", help="per-shape decode breakdown")
    ap.add_argument("--calls", choices=["batch", "grouped", "separate"], default="batch",
                    help="how the headline step calls the library: one batch launch per layer (default), "
                         "grouped q/k/v and gate/up calls, or one call per linear")
    ap.add_argument("--no-rows", action="store_true", help="skip the secondary hot-path rows")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.case:
        run_profile_case(args.case)
        return 0

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0

    world, rank, local = dist_setup()
    res = run_ours(args, world, rank, local)
    if rank == 0:
        # the full record (every row with its sample description) on stderr; the one JSON line
        # on stdout stays short enough to survive a 1500-character tail
        print("bench detail: " + json.dumps(res), file=sys.stderr, flush=True)
        print(json.dumps(compact_result(res)), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
