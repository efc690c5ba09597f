#!/usr/bin/env python3
"""Benchmark of the ternary GEMM (TQ2/TQ1 packed weights x fp16 activations).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--sweep]

One step = one pass of the ternary linear layers of the workload over one
batch of synthetic activations (weights are prepared once: at inference
only the ternary weights and their scales are kept).  The default
workload is the decode GEMV of the 70B-like down projection (W 8192x28672,
M = 1, TQ2), the shape the memory-bound target is stated on; the same line
carries, under "targets", the compute-regime shape (W 8192x8192, M = 256,
TQ2) and the LLaMA-7B-like single-layer decode set (W in {4096x4096,
11008x4096, 4096x11008}, M = 1), each timed the same way.  Weights are
absmean-ternarized from N(0, 0.02) latent weights by this library, then
cloned into enough rotating copies that every timed step reads weights that
are not in L2 (the copies total > 3x the L2 size).  The timed region is one
CUDA graph holding all K steps, timed with CUDA events around its replay;
the average GEMM launch takes that time over the number of launches.

Prints ONE JSON line (rank 0).  With --sweep, writes a table of lines for
the batch sweep, the 70B-like block and the sparsity stress workloads.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# ------------------------------------------------------------------ workloads
WORKLOADS = {
    # single-layer decode GEMV, LLaMA-7B-like shapes, M = 1 (N, K per layer)
    "llama7b_decode_m1": dict(layers=[(4096, 4096), (11008, 4096), (4096, 11008)], M=1, fmt="tq2",
                              seeds=[2, 3, 4]),
    "down_8192x28672_m1": dict(layers=[(8192, 28672)], M=1, fmt="tq2", seeds=[16]),
    "square_8192_m256": dict(layers=[(8192, 8192)], M=256, fmt="tq2", seeds=[5]),
    # 70B-like block linears at batch 16: q, k, v, o, gate, up, down
    "block70b_m16": dict(layers=[(8192, 8192), (1024, 8192), (1024, 8192), (8192, 8192),
                                 (28672, 8192), (28672, 8192), (8192, 28672)], M=16, fmt="tq2",
                         seeds=[10, 11, 12, 13, 14, 15, 16]),
    # the same block with q/k/v concatenated into one GEMM and gate/up fused
    # with the SwiGLU epilogue (2 x 28672 interleaved rows -> 28672 outputs)
    "block70b_m16_fused": dict(layers=[(10240, 8192), (8192, 8192), (57344, 8192), (8192, 28672)],
                               M=16, fmt="tq2", seeds=[10, 13, 14, 16], swiglu=[2]),
}
def kernels_per_call(path, M, fmt, swiglu=False):
    """Launches of this library's kernels for one call: prep + main for the
    mma.sync path and for the integer path at 3 <= M <= 16, one kernel
    otherwise; TQ1 adds its transcode on the tensor-core paths except the
    integer path at M <= 2, which reads TQ1 planes directly; an unfused
    SwiGLU call adds its combine kernel."""
    n = 2 if path == 2 or (path == 4 and M >= 3) else 1
    if fmt == "tq1" and path != 1 and not (path == 4 and M <= 2):
        n += 1
    if swiglu and not (path == 4 and 3 <= M <= 16):
        n += 1
    return n


def workload_from_args(name, M=None, fmt=None):
    w = dict(WORKLOADS[name])
    if M is not None:
        w["M"] = M
    if fmt is not None:
        w["fmt"] = fmt
    w["name"] = name
    return w


def algo_bytes(fmt, M, N, K):
    from bit_mixed_precision_tri_b200.api import packed_row_bytes
    return N * packed_row_bytes(fmt, K) + N * (K // 256) * 2 + M * K * 2 + M * N * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {k: float(j[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "bit_mixed_precision_tri_b200", "csrc")
    for fn in sorted(os.listdir(cs)):
        with open(os.path.join(cs, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if taken on the
    current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    src = kernel_source_hash()
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel \
                    and parts[1] == src and parts[3] == workload:
                return float(parts[2])
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 8:
                continue
            try:
                sm.append(float(p[0]))
                mx.append(float(p[1]))
            except ValueError:
                continue
            for nm, v in zip(names, p[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm
def prepare_layers(w, device, copies):
    import bit_mixed_precision_tri_b200 as tri
    from bit_mixed_precision_tri_b200 import inputs
    layers = []
    for (N, K), seed in zip(w["layers"], w["seeds"]):
        if w.get("p_zero") is None:
            W = inputs.latent_weights(N, K, seed).to(device)
            trits, g = tri.ternarize(W, 1e-6)
            qs, d = tri.pack(trits, g, w["fmt"])
            del W
        else:   # format stress: i.i.d. trits, one scale per 256-block
            trits = inputs.random_trits(N, K, w["p_zero"], seed).to(device)
            g = inputs.block_scales(N, K, seed + 1).to(device)
            qs, d = tri.pack(trits, g, w["fmt"])
            g = g.max()
        del trits
        reps = [(qs, d)] + [(qs.clone(), d.clone()) for _ in range(copies - 1)]
        X = inputs.activations(w["M"], K, 6 + w["M"] + seed).to(device)
        sw = len(layers) in w.get("swiglu", ())
        Y = torch.empty(w["M"], N // 2 if sw else N, dtype=torch.float16, device=device)
        layers.append(dict(N=N, K=K, reps=reps, X=X, Y=Y, gamma=float(g.item()), swiglu=sw))
    torch.cuda.synchronize(device)
    return layers


def run_ours(args, rank, world, device, w=None):
    import bit_mixed_precision_tri_b200 as tri
    if w is None:
        w = workload_from_args(args.workload, args.M, args.fmt)
    M, fmt = w["M"], w["fmt"]
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    step_bytes = sum(algo_bytes(fmt, M, N, K) - (M * N if i in w.get("swiglu", ()) else 0)
                     for i, (N, K) in enumerate(w["layers"]))
    weight_bytes = sum(N * tri.packed_row_bytes(fmt, K) + N * (K // 256) * 2 for N, K in w["layers"])
    copies = max(args.steps, int(np.ceil(3 * l2 / max(weight_bytes, 1))) + 1)
    layers = prepare_layers(w, device, copies)
    paths = [tri.auto_path(fmt, M, L["N"], L["K"]) for L in layers]
    ws = tri.Workspace(device)
    from bit_mixed_precision_tri_b200 import _lib as _tl
    ws.get(max(max(tri.gemm_workspace_bytes(fmt, M, L["N"], L["K"]),
                   int(_tl.lib().tri_gemm_swiglu_workspace_bytes(tri.api.FORMATS[fmt], M, L["N"] // 2, L["K"]))
                   if L["swiglu"] else 0) for L in layers))
    stream = torch.cuda.Stream(device)

    def call(L, X, qs, d, Y):
        if L["swiglu"]:
            tri.gemm_swiglu(X, qs, d, L["N"] // 2, L["K"], fmt, out=Y, workspace=ws, stream=stream)
        else:
            tri.gemm(X, qs, d, L["N"], L["K"], fmt, out=Y, workspace=ws, stream=stream)

    def step(c):
        for L in layers:
            qs, d = L["reps"][c]
            call(L, L["X"], qs, d, L["Y"])

    # eager warm-up (also allocates), then the warm-up and the timed steps are
    # each captured as one CUDA graph (one launch for the whole region; the
    # kernels of consecutive GEMMs overlap through programmatic dependent launch)
    with torch.cuda.stream(stream):
        for c in range(min(copies, 2)):
            step(c)
    torch.cuda.synchronize(device)
    g_warm, g_steps = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream):
        for i in range(args.warmup):
            step((copies - 1 - i) % copies)
    with torch.cuda.graph(g_steps, stream=stream):
        for s in range(args.steps):
            step(s % copies)
    torch.cuda.synchronize(device)
    upload_graph(g_steps, stream)
    g_warm.replay()
    torch.cuda.synchronize(device)

    clocks = ClockSampler(device.index if device.index is not None else 0)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        g_steps.replay()
        t1.record(stream)
    torch.cuda.synchronize(device)
    barrier(world)
    clk = clocks.stop() if rank == 0 else None
    elapsed_ms = t0.elapsed_time(t1)
    # every launch of the timed region is one of this library's GEMMs, back to
    # back on one stream: the average launch takes elapsed / launches
    n_launch = args.steps * len(layers)
    kernel_ms = elapsed_ms
    kernel_bytes = args.steps * sum(algo_bytes(fmt, M, L["N"], L["K"]) - (M * L["N"] if L["swiglu"] else 0)
                                    for L in layers)
    max_ms = allreduce_max(elapsed_ms, world, device)

    # end-to-end through the public API: every step copies its inputs (the X
    # of every layer, one pinned host buffer) to the device, runs the GEMMs
    # with eager calls, and reads all outputs back (one pinned host buffer)
    xsz = [M * L["K"] for L in layers]
    ysz = [L["Y"].numel() for L in layers]
    xh = torch.cat([L["X"].flatten().cpu() for L in layers]).pin_memory()
    yh = torch.empty(sum(ysz), dtype=torch.float16).pin_memory()
    xd_all = torch.empty(sum(xsz), dtype=torch.float16, device=device)
    yd_all = torch.empty(sum(ysz), dtype=torch.float16, device=device)
    xd = list(torch.split(xd_all, xsz))
    yd = list(torch.split(yd_all, ysz))
    xd = [x.view(M, L["K"]) for x, L in zip(xd, layers)]
    yd = [y.view(M, -1) for y, L in zip(yd, layers)]
    h2d, d2h = xh.numel() * 2, yh.numel() * 2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for rep in range(2):   # first pass warms, second is timed
            if rep == 1:
                barrier(world)
                torch.cuda.synchronize(device)
                e0.record(stream)
            for s in range(args.steps):
                c = s % copies
                xd_all.copy_(xh, non_blocking=True)
                for i, L in enumerate(layers):
                    qs, d = L["reps"][c]
                    call(L, xd[i], qs, d, yd[i])
                yh.copy_(yd_all, non_blocking=True)
            if rep == 1:
                e1.record(stream)
            torch.cuda.synchronize(device)
    e2e_ms = allreduce_max(e0.elapsed_time(e1), world, device)
    del g_warm, g_steps
    launches = args.steps * sum(kernels_per_call(p, M, fmt, L["swiglu"]) for p, L in zip(paths, layers))
    unit = "GB/s" if M <= 32 else "TFLOP/s"
    flops = sum(2.0 * M * N * K for N, K in w["layers"])

    def metric_value(ms, steps):
        if unit == "GB/s":
            return world * steps * step_bytes / (ms * 1e-3) / 1e9
        return world * steps * flops / (ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    if unit == "GB/s":
        achieved = kernel_bytes / (kernel_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": peak_src,
                "traffic": recorded_traffic("gemm", w["name"])}
    else:
        kflops = sum(2.0 * M * L["N"] * L["K"] for L in layers) * args.steps
        achieved = kflops / (kernel_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "peak_source": peak_src,
                "traffic": recorded_traffic("gemm", w["name"])}
    roof["kernel_launches_timed"] = n_launch
    roof["kernel_ms_per_launch"] = kernel_ms / max(n_launch, 1)
    res = {
        "metric": "TQ2/TQ1 ternary GEMM: HBM GB/s (M<=16) and TFLOP/s (M>=64) vs roofline",
        "value": metric_value(max_ms, args.steps),
        "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16xternary->f32acc",
        "data": "synthetic",
        "config": {"workload": w["name"], "layers_NxK": [f"{N}x{K}" for N, K in w["layers"]],
                   "M": M, "format": fmt, "global_batch": M * world,
                   "paths": paths, "weight_copies": copies,
                   "l2_policy": f"rotating {copies} weight copies ({copies * weight_bytes / 1e6:.0f} MB > 3x L2)",
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "roofline": roof,
        "e2e": {"value": metric_value(e2e_ms, args.steps), "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": launches,
        "clocks": clk,
    }
    return res


def upload_graph(g, stream):
    """Upload an instantiated graph to the device without running it, so that
    its first (timed) replay is not slowed by the one-time upload."""
    try:
        from cuda.bindings import runtime as cudart
        cudart.cudaGraphUpload(g.raw_cuda_graph_exec(), stream.cuda_stream)
    except Exception:   # older bindings: the first replay then includes the upload
        pass


def measure_cublas_fp16(w, device, steps, warmup):
    """The same layer sequence as a dense fp16 GEMM (torch.matmul -> cuBLAS),
    timed the same way (one CUDA graph of K steps over rotating weight copies
    larger than L2).  Context for the ternary path, not part of it."""
    M = w["M"]
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    dense_bytes = sum(2 * N * K for N, K in w["layers"])
    copies = max(2, int(np.ceil(3 * l2 / dense_bytes)) + 1)
    g = torch.Generator(device="cpu").manual_seed(1234)
    mats = [[(torch.randn(N, K, generator=g) * 0.02).half().to(device) for N, K in w["layers"]]]
    for _ in range(copies - 1):
        mats.append([t.clone() for t in mats[0]])
    xs = [torch.randn(M, K, generator=g).half().to(device) for _, K in w["layers"]]
    ys = [torch.empty(M, N, dtype=torch.float16, device=device) for N, _ in w["layers"]]
    stream = torch.cuda.Stream(device)

    def step(c):
        for i in range(len(w["layers"])):
            torch.matmul(xs[i], mats[c][i].t(), out=ys[i])

    with torch.cuda.stream(stream):
        for c in range(2):
            step(c)
    torch.cuda.synchronize(device)
    gw, gs = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gw, stream=stream):
        for i in range(warmup):
            step(i % copies)
    with torch.cuda.graph(gs, stream=stream):
        for i in range(steps):
            step(i % copies)
    upload_graph(gs, stream)
    gw.replay()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        gs.replay()
        t1.record(stream)
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1) / steps
    bytes_step = dense_bytes + sum(2 * M * K + 2 * M * N for N, K in w["layers"])
    del gw, gs, mats
    return {"ms_per_step": ms, "GB/s": bytes_step / (ms * 1e-3) / 1e9,
            "TFLOP/s": sum(2.0 * M * N * K for N, K in w["layers"]) / (ms * 1e-3) / 1e12,
            "weight_copies": copies}


TARGET_WORKLOADS = ("square_8192_m256", "llama7b_decode_m1")


def measure_targets(args, rank, world, device):
    """The other stated shapes, each timed like the main line (one CUDA graph
    of K steps over rotating weight copies larger than L2), with its own
    roofline; the compute-regime shape reports its tensor fraction against
    both the burst and the sustained measured bf16/fp16 peak."""
    out = {}
    peaks, _ = load_peaks()
    for name in TARGET_WORKLOADS:
        a = argparse.Namespace(**vars(args))
        a.steps, a.warmup = min(args.steps, 20), max(3, min(args.warmup, 5))
        w = workload_from_args(name)
        r = run_ours(a, rank, world, device, w=w)
        roof = dict(r["roofline"])
        if roof["bound"] == "tensor":
            roof["frac_of_sustained"] = roof["achieved"] / peaks["bf16_tflops_sustained"]
            roof["peak_sustained"] = peaks["bf16_tflops_sustained"]
        t = {"value": r["value"], "unit": r["unit"], "ms_per_step": r["ms_per_step"],
             "steps": a.steps, "warmup": a.warmup, "config": r["config"], "roofline": roof,
             "e2e": r["e2e"], "gpu_launches": r["gpu_launches"], "clocks": r["clocks"]}
        if not args.no_cublas:
            cb = measure_cublas_fp16(w, device, a.steps, a.warmup)
            cb["speedup_of_ternary"] = cb["ms_per_step"] / r["ms_per_step"]
            t["cublas_fp16"] = cb
        out[name] = t
    return out


# ------------------------------------------------------------------ decode step (f3)
DECODE_BLOCK = {"D": 8192, "H": 64, "Hkv": 8, "F": 28672}   # the 70B-like block's shapes


def measure_decode_block(device, M=1, context=4096, steps=20, warmup=5, fmt="tq2"):
    """One transformer-block decode step (RMSNorm, fused QKV, QK-Norm + RoPE
    with cache append, grouped-query attention over `context` cached
    positions, O, RMSNorm, fused gate/up SwiGLU, down, residuals) at the
    70B-like shapes for M sequences, random ternary weights (P(0) = 0.31,
    gamma 0.0159) and random caches; K steps captured in one CUDA graph and
    timed with CUDA events.  Every step streams the block's packed weights
    (220 MB TQ2) and the sequences' cached K and V (> L2), so no flush is
    needed between steps."""
    import bit_mixed_precision_tri_b200 as tri
    from bit_mixed_precision_tri_b200 import decode as dec
    from bit_mixed_precision_tri_b200 import inputs
    Dm, H, Hkv, F = (DECODE_BLOCK[k] for k in ("D", "H", "Hkv", "F"))
    hd = dec.HEAD_DIM
    shapes = {"qkv": ((H + 2 * Hkv) * hd, Dm), "o": (Dm, H * hd), "gate": (F, Dm), "up": (F, Dm), "down": (Dm, F)}
    w = {}
    for i, (name, (n, k)) in enumerate(shapes.items()):
        w[name] = (inputs.random_trits_on(device, n, k, 0.31, 200 + i),
                   torch.tensor([0.0159], dtype=torch.float32, device=device))
    for i, (name, n) in enumerate((("g_attn", Dm), ("g_mlp", Dm), ("gq", hd), ("gk", hd))):
        w[name] = (1.0 + 0.25 * inputs.fp16_normal_on(device, (n,), 210 + i).float()).to(torch.float16)
    Lmax = context + 1
    blk = dec.DecodeBlock(w, Dm, H, Hkv, F, M, Lmax, device, fmt=fmt)
    del w
    blk.kcache.copy_(inputs.fp16_normal_on(device, tuple(blk.kcache.shape), 220))
    blk.vcache.copy_(inputs.fp16_normal_on(device, tuple(blk.vcache.shape), 221))
    x = inputs.fp16_normal_on(device, (M, Dm), 222)
    pos = torch.full((M,), context, dtype=torch.int32, device=device)   # the new token follows `context` cached ones
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for _ in range(2):
            blk.step(x, pos, context + 1)
    torch.cuda.synchronize(device)
    g_warm, g_steps = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream):
        for _ in range(warmup):
            blk.step(x, pos, context + 1)
    with torch.cuda.graph(g_steps, stream=stream):
        for _ in range(steps):
            blk.step(x, pos, context + 1)
    torch.cuda.synchronize(device)
    g_warm.replay()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        g_steps.replay()
        t1.record(stream)
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1) / steps
    kv_bytes = M * Hkv * (context + 1) * hd * 2 * 2
    act_bytes = 2 * M * (Dm * 12 + (H + 2 * Hkv) * hd + F * 3)           # fp16 activations in and out, roughly
    step_bytes = blk.weight_bytes + kv_bytes + act_bytes
    peaks, _ = load_peaks()
    g = 1 if M <= 2 else 2                  # integer GEMM launches per call (3 <= M <= 16: prep + main)
    # rmsnorm, qkv, qknorm_rope, attention (2), o, rmsnorm, gate/up SwiGLU (2), down, residual
    launches = 1 + g + 1 + 2 + g + 1 + 2 + g + 1
    res = {"M": M, "context": context, "fmt": fmt, "shapes": dict(DECODE_BLOCK, head_dim=hd),
           "us_per_step": round(ms * 1e3, 2), "tokens_per_s": round(M / (ms * 1e-3), 1),
           "bytes_per_step": step_bytes, "weight_bytes": blk.weight_bytes, "kv_bytes": kv_bytes,
           "GB/s": round(step_bytes / (ms * 1e-3) / 1e9, 1),
           "frac_of_hbm": round(step_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
           "steps": steps, "warmup": warmup, "gpu_launches_per_step": launches,
           "data": "synthetic: random ternary weights (P(0) = 0.31), random fp16 caches and input"}
    del blk
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ other rows
def measure_rows(device, N=28672, K=8192, reps=5):
    """Time the offline rows of the path (absmean, ternarize, pack, unpack) on
    the largest weight of the 70B-like block (inputs larger than L2), with
    CUDA events; algorithmic bytes per element are stated per row."""
    import bit_mixed_precision_tri_b200 as tri
    from bit_mixed_precision_tri_b200 import inputs
    n = N * K
    W = inputs.latent_weights(N, K, 12).to(device)
    L = tri._lib.lib()
    ws = torch.zeros(L.tri_absmean_workspace_bytes(N, K), dtype=torch.uint8, device=device)
    g = torch.empty(1, dtype=torch.float32, device=device)
    trits = torch.empty(N, K, dtype=torch.int8, device=device)
    q2 = torch.empty(N, K // 4, dtype=torch.uint8, device=device)
    q1 = torch.empty(N, (K // 256) * 52, dtype=torch.uint8, device=device)
    dd = torch.empty(N, K // 256, dtype=torch.float16, device=device)
    out = torch.empty(N, K, dtype=torch.int8, device=device)
    st = torch.cuda.current_stream(device).cuda_stream
    P = lambda t: t.data_ptr()
    ops = {
        "absmean": (lambda: L.tri_absmean(P(W), N, K, 1e-6, P(g), P(ws), ws.numel(), st), 4.0),
        "ternarize": (lambda: L.tri_ternarize(P(W), N, K, 1e-6, P(trits), P(g), P(ws), ws.numel(), st),
                      9.0),
        "pack_tq2": (lambda: L.tri_pack_tq2(P(trits), N, K, P(g), 1, P(q2), P(dd), None, st),
                     1.0 + 0.25 + 2 / 256),
        "pack_tq1": (lambda: L.tri_pack_tq1(P(trits), N, K, P(g), 1, P(q1), P(dd), None, st),
                     1.0 + 52 / 256 + 2 / 256),
        "unpack_tq2": (lambda: L.tri_unpack(2, P(q2), N, K, P(out), None, st), 0.25 + 1.0),
        "unpack_tq1": (lambda: L.tri_unpack(1, P(q1), N, K, P(out), None, st), 52 / 256 + 1.0),
    }
    res = {}
    for name, (fn, bpe) in ops.items():
        for _ in range(2):
            assert fn() == 0, name
        times = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            assert fn() == 0, name
            b.record()
            torch.cuda.synchronize(device)
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        res[name] = {"us": round(ms * 1e3, 1), "GB/s": round(n * bpe / (ms * 1e-3) / 1e9, 1),
                     "bytes_per_weight": round(bpe, 4)}
    res["shape"] = f"{N}x{K}"
    del W, trits, q2, q1, dd, out
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ oracle arm
def blas_threads() -> int:
    """Threads of the BLAS pool that numpy's float64 matmul (the oracle's
    block products) runs on."""
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return 1


def oracle_sample(w, budget_s=12.0, threads=None):
    """Time the CPU oracle (as it stands) on a bounded sample of the workload:
    whole layers (unpack + fp64 GEMM) until ~budget_s of CPU work.  With
    ``threads`` the BLAS pool is limited to that many threads for the timing.
    Returns a dict: value (the workload's unit), unit, sample description,
    threads used, elapsed seconds."""
    import contextlib
    from bit_mixed_precision_tri_b200 import inputs
    from oracle import tri_oracle as O
    M, fmt = w["M"], w["fmt"]
    unit = "GB/s" if M <= 32 else "TFLOP/s"
    prepared = []
    for (N, K), seed in zip(w["layers"], w["seeds"]):
        rows = min(N, 2048)
        W = inputs.latent_weights(rows, K, seed).numpy()
        t, g = O.absmean_ternarize(W, 1e-6)
        qs, d = O.pack(fmt, t, np.array([g], np.float32))
        X = inputs.activations(M, K, 6 + M + seed).numpy()
        prepared.append((rows, K, qs, d, X))
    limit = contextlib.nullcontext()
    if threads is not None:
        try:
            from threadpoolctl import threadpool_limits
            limit = threadpool_limits(limits=threads, user_api="blas")
        except Exception:
            pass
    with limit:
        used = blas_threads()
        done_bytes = done_flops = 0.0
        t0 = time.perf_counter()
        n = 0
        while True:
            for rows, K, qs, d, X in prepared:
                O.gemm_packed_f64(fmt, X, qs, d, rows, K)
                done_bytes += algo_bytes(fmt, M, rows, K)
                done_flops += 2.0 * M * rows * K
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
    val = done_bytes / dt / 1e9 if unit == "GB/s" else done_flops / dt / 1e12
    desc = (f"{n} passes over the first min(N, 2048) rows of each layer "
            f"({'+'.join(str(min(N, 2048)) + 'x' + str(K) for N, K in w['layers'])}), "
            f"unpack + float64 GEMM (numpy, BLAS on {used} thread(s)), {dt:.1f} s")
    return {"value": val, "unit": unit, "sample": desc, "threads": used, "elapsed_s": dt}


def run_reference(args, rank, world):
    w = workload_from_args(args.workload, args.M, args.fmt)
    if rank != 0:
        return None
    budget = max(3.0, 60.0 / max(args.steps + args.warmup, 1))
    samples = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(w, budget_s=budget)
        if i >= args.warmup:
            samples.append(r)
    value = statistics.mean(r["value"] for r in samples)
    unit = samples[0]["unit"]
    return {
        "impl": "reference",
        "metric": "TQ2/TQ1 ternary GEMM: HBM GB/s (M<=16) and TFLOP/s (M>=64) vs roofline",
        "value": value, "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        # measured: the mean wall time of one step (one bounded oracle sample)
        "ms_per_step": statistics.mean(r["elapsed_s"] for r in samples) * 1e3,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w["name"], "layers_NxK": [f"{N}x{K}" for N, K in w["layers"]],
                   "M": w["M"], "format": w["fmt"]},
        "cpu_baseline": {"value": value, "unit": unit, "cores": samples[0]["threads"], "kind": "oracle",
                         "sample": samples[0]["sample"]},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ dist utils
def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def allreduce_max(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


SWEEP_M = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512]


def run_sweep(args, rank, world, device):
    """Batch sweep on W 8192x8192 (TQ2 and TQ1), the 70B-like block at M = 16
    and the format stress set on W 14336x4096 (P(0) in {0.3, 0.5, 0.7, 0.9},
    per-block scales, M in {1, 16, 128}); one JSON line each, with the cuBLAS
    fp16 time of the same shapes beside it."""
    jobs = []
    for fmt in ("tq2", "tq1"):
        for M in SWEEP_M:
            jobs.append(dict(name=f"sweep_8192_{fmt}_m{M}", layers=[(8192, 8192)], M=M, fmt=fmt, seeds=[5]))
    jobs.append(dict(WORKLOADS["block70b_m16"], name="block70b_m16"))
    jobs.append(dict(WORKLOADS["block70b_m16_fused"], name="block70b_m16_fused"))
    for fmt in ("tq2", "tq1"):
        for p0 in (0.3, 0.5, 0.7, 0.9):
            for M in (1, 16, 128):
                jobs.append(dict(name=f"stress_14336x4096_{fmt}_p{p0}_m{M}", layers=[(14336, 4096)], M=M,
                                 fmt=fmt, seeds=[20 + int(10 * p0)], p_zero=p0))
    cublas_cache = {}
    for job in jobs:
        a = argparse.Namespace(**vars(args))
        a.steps, a.warmup = min(args.steps, 10), max(3, min(args.warmup, 3))
        res = run_ours(a, rank, world, device, w=job)
        key = (tuple(job["layers"]), job["M"])
        if not args.no_cublas:
            if key not in cublas_cache:
                cublas_cache[key] = measure_cublas_fp16(job, device, a.steps, a.warmup)
            cb = dict(cublas_cache[key])
            cb["speedup_of_ternary"] = cb["ms_per_step"] / res["ms_per_step"]
            res["cublas_fp16"] = cb
        if rank == 0:
            print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="down_8192x28672_m1", choices=sorted(WORKLOADS))
    ap.add_argument("--M", type=int, default=None)
    ap.add_argument("--fmt", default=None, choices=[None, "tq2", "tq1"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip timing the offline rows")
    ap.add_argument("--no-cublas", action="store_true", help="skip the cuBLAS fp16 comparison")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the extra target workloads of the default line")
    ap.add_argument("--sweep", action="store_true",
                    help="print one line per batch-sweep, block and format-stress workload")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the one-block decode step (70B-like shapes, M = 1 and 16, "
                         "4096 cached positions) and print it")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-step lines of the default run")
    ap.add_argument("--rows-only", action="store_true",
                    help="time only the offline rows (absmean, ternarize, pack, unpack) on the "
                         "28672x8192 weight, --steps timed calls each, and print them")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if world > 1 and rank != 0:
            return
        res = run_reference(args, 0, world)
        print(json.dumps(res), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        if args.sweep:
            run_sweep(args, rank, world, device)
            return
        if args.decode_only:
            if rank == 0:
                out = {f"decode_block70b_m{M}": measure_decode_block(device, M=M, steps=max(1, args.steps),
                                                                     warmup=args.warmup) for M in (1, 16)}
                print(json.dumps(out), flush=True)
            return
        if args.rows_only:
            if rank == 0:
                print(json.dumps({"rows": measure_rows(device, reps=max(1, args.steps))}), flush=True)
            return
        res = run_ours(args, rank, world, device)
        if not args.no_cublas:
            w = workload_from_args(args.workload, args.M, args.fmt)
            cb = measure_cublas_fp16(w, device, args.steps, args.warmup)
            cb["speedup_of_ternary"] = cb["ms_per_step"] / res["ms_per_step"]
            res["cublas_fp16"] = cb
        if not args.no_targets and args.workload == "down_8192x28672_m1" and args.M is None \
                and args.fmt is None:
            res["targets"] = measure_targets(args, rank, world, device)
        if not args.no_rows:
            res["rows"] = measure_rows(device)
        if not args.no_decode and args.workload == "down_8192x28672_m1" and args.M is None and args.fmt is None:
            res["decode_block70b"] = {f"m{M}": measure_decode_block(device, M=M, steps=min(args.steps, 20),
                                                                    warmup=max(3, min(args.warmup, 5)))
                                      for M in (1, 16)}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            w = workload_from_args(args.workload, args.M, args.fmt)
            r = oracle_sample(w, budget_s=8.0)
            r1 = oracle_sample(w, budget_s=4.0, threads=1)
            res["cpu_baseline"] = {"value": r["value"], "unit": r["unit"], "cores": r["threads"],
                                   "kind": "oracle", "sample": r["sample"],
                                   "single_core": {"value": r1["value"], "unit": r1["unit"], "cores": 1,
                                                   "sample": r1["sample"]}}
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
