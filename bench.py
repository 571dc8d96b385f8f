#!/usr/bin/env python3
"""Benchmark of the AWQ W4A16 linear layer on B200.

Headline: the Mistral-7B-shaped decode set (M = 1; K x N = 4096 x 6144 QKV,
4096 x 4096 O, 4096 x 28672 gate+up, 14336 x 4096 down).  One step is one
decode pass through a layer: the four fused-dequantization GEMVs, each
reading that layer's packed weights once.  Layers rotate (distinct weights,
footprint above twice the L2 size) so the weights always come from HBM.
The metric is packed-weight bytes (4-bit codes + binary16 steps + 4-bit zero
points, 0.5195 B per weight) per second.

Also reported on the same line: the prefill GEMM (7B shapes, M = 4096) in
TFLOP/s, the one-off quantization pass (act_stats + compute_scales +
quantize_pack) in GB/s of fp16 weights read, the end-to-end number through
the public API with host buffers, and the CPU oracle timed on the host cores.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       (N > 1: launch under torch.distributed.run; each rank runs its own
       replica of the workload, value = all ranks' bytes / max-over-ranks time)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W4A16 matmul: weight GB/s (M=1) & TFLOP/s (M>=256) vs B200 roofline"
WORKLOAD_ID = 2
BYTES_PER_WEIGHT = 0.5 + 2 / 128 + 0.5 / 128  # codes + steps + zero points
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The files the decode GEMV kernel is compiled from: a stored ncu traffic figure
# stays valid while none of them changes.
GEMV_SOURCES = ("weight_only_quantization_quantize_b200/csrc/gemv.cu",
                "weight_only_quantization_quantize_b200/csrc/awq_common.cuh",
                "weight_only_quantization_quantize_b200/csrc/awq_kernels.cuh",
                "include/awq_b200.h")


def _code_only(text: str) -> str:
    """C/C++ source with comments and blank runs removed (what the compiler sees)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash():
    """Hash of the decode GEMV's code (comments and layout ignored)."""
    h = hashlib.sha256()
    for rel in GEMV_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(rel.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def stored_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if taken on this source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5], f[6], f[7], f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
def build_layers(awq, nlayers, device, workload=WORKLOAD_ID, zero_point=True, M=1, first=0):
    """Quantize `nlayers` distinct synthetic layers on the GPU (kept packed).

    zero_point=False: symmetric weights (no zeros tensor; p["z"] is None)."""
    wl = synth.WORKLOADS[workload]
    layers = []
    for li in range(first, first + nlayers):
        projs = []
        for si, (K, N, label) in enumerate(wl.shapes):
            L = synth.make_layer(workload, li, M=M, K=K, N=N, R=wl.R, device=device, shape_id=si)
            s = awq.compute_scales(awq.act_stats(L.Xcal))
            Q, sc, z = awq.quantize_pack(L.W, s, zero_point=zero_point)
            projs.append(dict(K=K, N=N, label=label, X=L.X, s=s, Q=Q, sc=sc, z=z,
                              Y=torch.empty(M, N, dtype=torch.float16, device=device)))
            del L
        layers.append(projs)
    torch.cuda.synchronize()
    return layers


def max_over_ranks(x, device):
    """The maximum of x over all ranks (x itself outside a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, bytes_per_step, steps, ms):
    """Whole-job GB/s: every rank's bytes over the slowest rank's time (weak scaling)."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def weight_bytes(K, N):
    return K * N * BYTES_PER_WEIGHT


def algorithmic_bytes(M, K, N):
    return weight_bytes(K, N) + 2 * M * K + 2 * K + 2 * M * N


def zeroed_workspace(awq, device, shapes, Ms):
    """One zero-filled workspace large enough for every (M, K, N) call of a run."""
    need = max(awq.gemm_workspace_size(M, K, N) for M in Ms for K, N in shapes)
    return torch.zeros(need, dtype=torch.uint8, device=device)


def graph_time(step, steps, warmup, stream):
    """Warm up, capture `steps` calls of step(i) in one CUDA graph, replay once
    untimed, then time one replay with CUDA events; ms for the whole replay."""
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            step(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    return ms


def run_ours(args, rank, world, device):
    import weight_only_quantization_quantize_b200 as awq
    awq.lib()
    peaks, peak_src = load_peaks()
    L2 = torch.cuda.get_device_properties(device).L2_cache_size
    wl = synth.WORKLOADS[WORKLOAD_ID]
    layer_bytes = sum(weight_bytes(K, N) for K, N, _ in wl.shapes)
    nlayers = max(2, math.ceil(2 * L2 / layer_bytes) + 1)
    layers = build_layers(awq, nlayers, device)
    stream = torch.cuda.current_stream(device)
    ws = zeroed_workspace(awq, device, [(K, N) for K, N, _ in wl.shapes], [1])

    def step(i):
        for p in layers[i % nlayers]:
            awq.w4a16_gemv(p["X"], p["s"], p["Q"], p["sc"], p["z"], out=p["Y"], workspace=ws)

    # warm-up, then capture K steps in one CUDA graph (launch-bound decode loop)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(args.steps):
            step(i)
    g.replay()  # one untimed replay
    torch.cuda.synchronize()

    dist = world > 1
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # The timed region lasts milliseconds, shorter than the 200 ms sampling
    # period, so clocks are sampled over ~1 s of the same load that ends with
    # the timed replay.
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t_end = time.time() + 1.0
        while time.time() < t_end:
            g.replay()
            torch.cuda.synchronize()
        if dist:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), device)
    if dist:
        torch.distributed.barrier()
    del g

    bytes_step = layer_bytes
    value = whole_job_value(world, bytes_step, args.steps, ms)
    alg_step = sum(algorithmic_bytes(1, K, N) for K, N, _ in wl.shapes)
    achieved = alg_step * args.steps / (ms * 1e-3) / 1e9
    launches = 4 * args.steps
    traffic = stored_traffic("gemv_decode_7b")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic, "peak_source": f"{peak_src} HBM copy bandwidth",
                "kernel": "gemv_kernel",
                "bytes_per_launch_avg": round(alg_step / 4)}

    # ---- end to end through the public API: pinned host X in, host Y out, every step
    e2e = run_e2e(awq, layers, args, device)

    extra = {}
    if not args.quick and rank == 0:
        del layers
        torch.cuda.empty_cache()
        extra.update(run_config_sweep(awq, device, peaks, peak_src))
        qlayers = build_layers(awq, 1, device)
        extra["quantize_7b_layer"] = run_quantize(awq, device, qlayers, peaks)
        extra["quantize_7b_layer_symmetric"] = run_quantize(awq, device, qlayers, peaks, zero_point=False)
        del qlayers
        extra["decode_7b_symmetric"] = run_decode_variant(awq, device, peaks, nlayers)
        extra["decode_7b_prescaled"] = run_decode_variant(awq, device, peaks, nlayers, prescaled=True)
        extra.update(run_calibration(awq, device))

    cpu = run_cpu_baseline(rank, world) if rank == 0 else None
    return dict(value=value, ms=ms, roofline=roofline, e2e=e2e, launches=launches,
                clocks=clk.summary(), extra=extra, cpu=cpu, nlayers=nlayers, L2=L2)


def run_e2e(awq, layers, args, device):
    """The decode step through the public API with host buffers: every step
    copies that layer's four activation rows from pinned host memory (one
    copy), runs the four projections (QuantLinear layers, eager) and reads the
    four outputs back (one copy).  The copies run on their own streams, one
    step ahead (inputs) and one step behind (outputs) of the compute stream,
    with events ordering each buffer's reuse, as a serving loop overlaps them;
    the timed steps are captured once in a CUDA graph and replayed."""
    stream = torch.cuda.current_stream(device)
    up = torch.cuda.Stream(device)    # host -> device
    down = torch.cuda.Stream(device)  # device -> host
    nl = len(layers)
    ks = [p["K"] for p in layers[0]]
    ns = [p["N"] for p in layers[0]]
    xo = np.cumsum([0] + ks)
    yo = np.cumsum([0] + ns)
    hx = [torch.empty(int(xo[-1]), dtype=torch.float16).pin_memory() for _ in layers]
    hy = [torch.empty(int(yo[-1]), dtype=torch.float16).pin_memory() for _ in layers]
    dx = [torch.empty(int(xo[-1]), dtype=torch.float16, device=device) for _ in layers]
    dy = [torch.empty(int(yo[-1]), dtype=torch.float16, device=device) for _ in layers]
    for li, layer in enumerate(layers):
        for pi, p in enumerate(layer):
            hx[li][xo[pi]:xo[pi + 1]].copy_(p["X"].view(-1).cpu())
    xv = [[dx[li][xo[pi]:xo[pi + 1]].view(1, -1) for pi in range(len(ks))] for li in range(nl)]
    yv = [[dy[li][yo[pi]:yo[pi + 1]].view(1, -1) for pi in range(len(ns))] for li in range(nl)]
    lin = [[awq.QuantLinear(p["Q"], p["sc"], p["z"], p["s"]) for p in layer] for layer in layers]
    ws = zeroed_workspace(awq, device, [(p["K"], p["N"]) for p in layers[0]], [1])
    h2d = 2 * int(xo[-1])
    d2h = 2 * int(yo[-1])

    def make_events():
        return {k: [torch.cuda.Event() for _ in range(nl)] for k in ("in_ready", "computed", "out_read")}

    def run(n, first, evs, cur):
        """Steps first .. first + n - 1 on stream `cur`; events ordering each
        buffer's reuse are waited on only once recorded in this run."""
        recorded = set()

        def wait(strm, kind, li):
            if (kind, li) in recorded:
                strm.wait_event(evs[kind][li])

        def record(strm, kind, li):
            evs[kind][li].record(strm)
            recorded.add((kind, li))

        def upload(i):
            li = i % nl
            with torch.cuda.stream(up):
                wait(up, "computed", li)       # the previous step on dx[li] is done with it
                dx[li].copy_(hx[li], non_blocking=True)
                record(up, "in_ready", li)

        up.wait_stream(cur)
        down.wait_stream(cur)
        upload(first)
        for i in range(first, first + n):
            li = i % nl
            if i + 1 < first + n:
                upload(i + 1)
            wait(cur, "in_ready", li)
            wait(cur, "out_read", li)         # dy[li] of the previous step on it was read out
            for pi, f in enumerate(lin[li]):
                f(xv[li][pi], out=yv[li][pi], workspace=ws)
            record(cur, "computed", li)
            with torch.cuda.stream(down):
                wait(down, "computed", li)
                hy[li].copy_(dy[li], non_blocking=True)
                record(down, "out_read", li)
        cur.wait_stream(up)
        cur.wait_stream(down)

    run(args.warmup, 0, make_events(), stream)
    torch.cuda.synchronize()
    # The timed steps go through the same public calls, captured once into a
    # CUDA graph so that host-side submission (Python, ctypes) is not what is
    # timed; every step still copies its inputs in and its outputs out.
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(args.steps, args.warmup, make_events(), torch.cuda.current_stream(device))
    g.replay()
    torch.cuda.synchronize()
    wb = sum(weight_bytes(p["K"], p["N"]) for p in layers[0])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    return {"value": round(wb * args.steps / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / args.steps, 4),
            "path": "QuantLinear (python binding -> C ABI), the timed steps captured in one CUDA graph; "
                    "per step one H2D copy of its 4 activation rows from pinned host memory and one D2H "
                    "copy of its 4 outputs, on copy streams overlapping the neighbouring steps' compute"}


def flush_l2(buf):
    buf.add_(1)


def _sweep_entry(kind, M, wl, ms_per_pass, passes_bytes, flops, peaks, peak_src, layers_note):
    """One sweep key: weight GB/s for the HBM-bound token counts, TFLOP/s (and
    GB/s) for the tensor-bound ones, each as a fraction of the named peak."""
    gbs = passes_bytes / (ms_per_pass * 1e-3) / 1e9
    tf = flops / (ms_per_pass * 1e-3) / 1e12
    e = {"M": M, "shapes": [list(x[:2]) for x in wl.shapes], "ms_per_pass": round(ms_per_pass, 5),
         "weight_gbs": round(gbs, 1), "tflops": round(tf, 1), "layers": layers_note}
    if kind == "hbm":
        e.update(bound="hbm", frac=round(gbs / peaks["hbm_gbs"], 4), peak=peaks["hbm_gbs"],
                 peak_name=f"{peak_src} HBM copy bandwidth (GB/s)")
    else:
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        e.update(bound="tensor", frac=round(tf / peak, 4), peak=peak,
                 peak_name=f"{peak_src} dense bf16 burst (TFLOP/s; fp16 runs at the bf16 rate); "
                           "each pass is a few ms timed alone")
    return e


def run_sweep(awq, device, peaks, peak_src, wid, Ms, reps, kinds):
    """Time `reps` passes over distinct layers of workload `wid` for each token
    count in Ms, each captured in one CUDA graph (layers rotate so the weights
    come from HBM).  The layers are quantized once, with activations for the
    largest M; smaller M use the leading rows."""
    wl = synth.WORKLOADS[wid]
    L2 = torch.cuda.get_device_properties(device).L2_cache_size
    layer_bytes = sum(weight_bytes(K, N) for K, N, _ in wl.shapes)
    nlayers = wl.layers if wl.layers > 1 else max(2, math.ceil(2 * L2 / layer_bytes) + 1)
    Mmax = max(Ms)
    layers = build_layers(awq, nlayers, device, workload=wid, M=Mmax)
    ws = zeroed_workspace(awq, device, [(K, N) for K, N, _ in wl.shapes], Ms)
    stream = torch.cuda.current_stream(device)
    note = (f"{nlayers} distinct layers, each pass one layer's 4 projections" if wl.layers > 1 else
            f"{nlayers} distinct layers rotated ({nlayers * layer_bytes / 1e6:.0f} MB packed > 2 x L2)")
    out = {}
    for M, kind in zip(Ms, kinds):
        views = [[(p, p["X"][:M], p["Y"][:M]) for p in layer] for layer in layers]

        def step(i):
            for p, X, Y in views[i % nlayers]:
                awq.w4a16_gemm(X, p["s"], p["Q"], p["sc"], p["z"], out=Y, workspace=ws)

        steps = reps * nlayers if wl.layers > 1 else max(reps, nlayers)
        ms = graph_time(step, steps, 3, stream) / steps
        flops = sum(2 * M * K * N for K, N, _ in wl.shapes)
        out[M] = _sweep_entry(kind, M, wl, ms, layer_bytes, flops, peaks, peak_src, note)
    del layers, ws
    torch.cuda.empty_cache()
    return out


def run_config_sweep(awq, device, peaks, peak_src):
    """Every workload and token count of the benchmark configuration list."""
    out = {}
    out["single_layer_1024_m1"] = run_sweep(awq, device, peaks, peak_src, 1, [1], 200, ["hbm"])[1]
    r = run_sweep(awq, device, peaks, peak_src, 3, [8, 16, 32, 48], 20, ["hbm"] * 4)
    out.update({f"small_batch_13b_m{M}": e for M, e in r.items()})
    r = run_sweep(awq, device, peaks, peak_src, 4, [512, 2048, 4096], 5, ["tensor"] * 3)
    out.update({f"prefill_7b_m{M}": e for M, e in r.items()})
    r = run_sweep(awq, device, peaks, peak_src, 5, [1, 32, 256], 2, ["hbm", "hbm", "tensor"])
    out.update({f"stack_70b_m{M}": e for M, e in r.items()})
    return out


def run_calibration(awq, device, reps=3):
    """The two calibration searches on one 7B projection (O, 4096 x 4096, 256
    calibration rows): the scale search over alpha = j/8 and weight clipping
    (11 candidate ranges).  Calibration runs once per layer, offline."""
    wl = synth.WORKLOADS[WORKLOAD_ID]
    K, N, _ = wl.shapes[1]
    L = synth.make_layer(WORKLOAD_ID, 0, M=1, K=K, N=N, R=wl.R, device=device, shape_id=1)
    R = wl.R
    ws = torch.zeros(awq.scale_search_workspace_size(R, K, N), dtype=torch.uint8, device=device)
    s = awq.compute_scales(awq.act_stats(L.Xcal))

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        t = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            t.append(e0.elapsed_time(e1))
        return statistics.median(t)

    ms_search = timed(lambda: awq.scale_search(L.Xcal, L.W, workspace=ws))
    ms_clip = timed(lambda: awq.quantize_pack_clip(L.W, s, L.Xcal, 11))
    gemm_flops = 10 * 2 * R * K * N          # the unquantized X W and 9 quantized products
    clip_flops = 11 * 2 * R * K * N          # candidate error vectors applied to the rows
    return {"scale_search_7b_o": {"ms": round(ms_search, 3), "grid": "alpha = j/8, j = 0..8",
                                  "calib_rows": R, "matmul_tflops": round(gemm_flops / (ms_search * 1e-3) / 1e12, 1),
                                  "includes": "statistics, W transpose, X W (tcgen05), 9 x (scales, quantize_pack, "
                                              "W4A16 matmul at M = R, loss), argmin"},
            "quantize_clip_7b_o": {"ms": round(ms_clip, 3), "candidates": 11, "calib_rows": R,
                                   "fp32_tflops": round(clip_flops / (ms_clip * 1e-3) / 1e12, 1),
                                   "includes": "per (group, column) 11 ranges scored on the calibration rows, "
                                               "codes of the best"}}


def run_decode_variant(awq, device, peaks, nlayers, steps=200, warmup=5, prescaled=False):
    """A decode-step variant, timed like the headline.

    prescaled=False: symmetric weights (zeros = NULL); algorithmic bytes 0.5 B
    per weight + 2 B per 128 weights (no zero points).
    prescaled=True: the headline's asymmetric weights with 1/s folded upstream
    (X already holds X/s, s = NULL); 0.5195 B per weight."""
    wl = synth.WORKLOADS[WORKLOAD_ID]
    layers = build_layers(awq, nlayers, device, zero_point=prescaled)
    if prescaled:
        for lp in layers:
            for p in lp:
                p["X"] = awq.fold_inverse_scale(p["X"], p["s"])
        torch.cuda.synchronize()
    ws = zeroed_workspace(awq, device, [(K, N) for K, N, _ in wl.shapes], [1])

    def step(i):
        for p in layers[i % nlayers]:
            if prescaled:
                awq.w4a16_gemv(p["X"], None, p["Q"], p["sc"], p["z"], out=p["Y"], workspace=ws)
            else:
                awq.w4a16_gemv(p["X"], p["s"], p["Q"], p["sc"], None, out=p["Y"], workspace=ws)

    ms = graph_time(step, steps, warmup, torch.cuda.current_stream(device))
    del layers
    per_weight = BYTES_PER_WEIGHT if prescaled else 0.5 + 2 / 128
    wbytes = sum(K * N * per_weight for K, N, _ in wl.shapes)
    gbs = wbytes * steps / (ms * 1e-3) / 1e9
    return {"ms_per_step": round(ms / steps, 5), "weight_gbs": round(gbs, 1),
            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "bytes": ("0.5195 B/weight (codes, steps, zeros); X already divided by s" if prescaled
                      else "0.5 B/weight codes + fp16 step per 128 weights; no zero points"),
            "l2": f"{nlayers} distinct layers rotated", "timing": "CUDA graph, CUDA events"}


def run_quantize(awq, device, layers, peaks, reps=5, zero_point=True):
    """act_stats + compute_scales + quantize_pack over one 7B layer (fp16 W read once).

    zero_point=False times the symmetric quantizer (no zero points written)."""
    wl = synth.WORKLOADS[WORKLOAD_ID]
    ins = []
    for si, (K, N, label) in enumerate(wl.shapes):
        L = synth.make_layer(WORKLOAD_ID, 99, M=1, K=K, N=N, R=wl.R, device=device, shape_id=si)
        ins.append(L)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    times = []
    for r in range(reps + 2):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for L in ins:
            s = awq.compute_scales(awq.act_stats(L.Xcal))
            awq.quantize_pack(L.W, s, zero_point=zero_point)
        e1.record()
        torch.cuda.synchronize()
        if r >= 2:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    packed = weight_bytes if zero_point else (lambda K, N: K * N * (0.5 + 2 / 128))
    moved = sum(2 * L.K * L.N + packed(L.K, L.N) + 2 * L.R * L.K for L in ins)
    gbs = moved / (ms * 1e-3) / 1e9
    return {"ms_per_layer": round(ms, 4), "gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "bytes": "fp16 W read + packed write + calibration rows"}


def _oracle_sample(oracle, K, N, label, si, frac, offset=0):
    """Oracle inputs for a column sample of one projection (quantization is per column)."""
    wl = synth.WORKLOADS[WORKLOAD_ID]
    L = synth.make_layer(WORKLOAD_ID, 0, M=1, K=K, N=N, R=wl.R, device="cpu", shape_id=si)
    ncols = max(8, (int(N * frac) // 8) * 8)
    cols = (np.arange(ncols, dtype=np.int64) * (N // ncols) + offset) % N
    s = oracle.compute_scales(oracle.act_stats(L.Xcal.numpy()))
    Wsub = np.ascontiguousarray(L.W.numpy()[:, cols])
    Q, sc, z = oracle.quantize_pack(Wsub, s)
    return L.X.numpy(), s, Q, sc, z, K, ncols


def run_cpu_baseline(rank, world, fraction=0.25):
    """The oracle (dequantise-then-float matmul) on the host cores: a bounded sample."""
    import oracle
    wl = synth.WORKLOADS[WORKLOAD_ID]
    cores = os.cpu_count() or 1
    total_bytes, total_s = 0.0, 0.0
    for si, (K, N, label) in enumerate(wl.shapes):
        X, s, Q, sc, z, K, ncols = _oracle_sample(oracle, K, N, label, si, fraction)
        t0 = time.perf_counter()
        oracle.matmul(X, s, Q, sc, z, precision=32, nthreads=cores)
        total_s += time.perf_counter() - t0
        total_bytes += weight_bytes(K, ncols)
    return {"value": round(total_bytes / total_s / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"7B decode layer, M=1, {int(fraction * 100)}% of each projection's columns "
                      f"(all K), float dequantise-then-matmul, {cores} threads"}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle, as it stands, on bounded samples of the same workload."""
    if rank != 0:
        return
    import oracle
    wl = synth.WORKLOADS[WORKLOAD_ID]
    cores = os.cpu_count() or 1
    frac = 1 / 16
    prepared = [_oracle_sample(oracle, K, N, label, si, frac)
                for si, (K, N, label) in enumerate(wl.shapes)]

    def step(i):
        b = 0.0
        for X, s, Q, sc, z, K, ncols in prepared:
            oracle.matmul(X, s, Q, sc, z, precision=32, nthreads=cores)
            b += weight_bytes(K, ncols)
        return b

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    tot = 0.0
    for i in range(args.steps):
        tot += step(i)
    sec = time.perf_counter() - t0
    value = tot / sec / 1e9
    sample = (f"7B decode layer, M=1, 1/16 of each projection's columns per step (all K), "
              f"float dequantise-then-matmul oracle, {cores} threads")
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3 / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "shapes": [list(x[:2]) for x in wl.shapes], "M": 1},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile(workload, M, reps):
    """One synthetic layer of `workload`, each projection called `reps` times (for ncu)."""
    import weight_only_quantization_quantize_b200 as awq
    torch.cuda.set_device(0)
    wl = synth.WORKLOADS[workload]
    projs = []
    for si, (K, N, label) in enumerate(wl.shapes):
        L = synth.make_layer(workload, 0, M=M, K=K, N=N, R=wl.R, device="cuda", shape_id=si)
        s = awq.compute_scales(awq.act_stats(L.Xcal))
        Q, sc, z = awq.quantize_pack(L.W, s)
        ws = torch.zeros(max(awq.gemm_workspace_size(M, K, N), 16), dtype=torch.uint8, device="cuda")
        projs.append((L.X, s, Q, sc, z, ws))
        del L
    torch.cuda.synchronize()
    for _ in range(reps):
        for X, s, Q, sc, z, ws in projs:
            if M == 1:
                awq.w4a16_gemv(X, s, Q, sc, z)
            else:
                awq.w4a16_gemm(X, s, Q, sc, z, workspace=ws)
    torch.cuda.synchronize()
    print(f"profile driver done: workload {workload}, M={M}, reps={reps}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="headline only (no extra sections)")
    ap.add_argument("--profile", nargs=3, type=int, metavar=("WORKLOAD", "M", "REPS"),
                    help="profiling driver: one layer of WORKLOAD, every projection REPS times")
    args = ap.parse_args()
    if args.profile:
        run_profile(*args.profile)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        r = run_ours(args, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rank != 0:
        return
    wl = synth.WORKLOADS[WORKLOAD_ID]
    line = {
        "metric": METRIC, "value": round(r["value"], 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms"] / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": wl.name, "shapes": [list(x[:2]) for x in wl.shapes], "M": 1,
                   "layers_rotated": r["nlayers"],
                   "l2": f"inputs larger than L2: {r['nlayers']} distinct layers rotated "
                         f"({r['nlayers'] * 113.3:.0f} MB of packed weights > 2 x {r['L2'] / 2**20:.0f} MiB L2)",
                   "parallelism": f"replicas x{world}", "timing": "CUDA graph of all timed steps, CUDA events",
                   "clocks_window": "nvidia-smi every 200 ms over ~1 s of identical load ending with the timed replay"},
        "roofline": r["roofline"], "cpu_baseline": r["cpu"], "e2e": r["e2e"],
        "gpu_launches": r["launches"], "clocks": r["clocks"],
    }
    line.update(r["extra"])
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
