#!/usr/bin/env python
"""Benchmark of the dynamic-convolution hot path on B200.

One step = routing + forward of one dynamic-convolution layer over one batch
(default: the ResNet-18-style 3x3 layer, B=64, 128->128 channels, 28x28, bf16,
n=4 experts, softmax routing). Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--variant V]
  python bench.py --config effnet_block   # the chained 1x1 -> depthwise block, one GPU
  python bench.py --impl reference ...     # the fp64 CPU oracle on the host cores

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of the
same layer (weak scaling, no collective on the data path); the time is the max
over ranks.

Timing: inputs are rotated over enough x/alpha/y buffer sets that their total
footprint exceeds the 126 MB L2, so each step starts cold in L2. The K timed
steps run as CUDA-graph replays (8 steps per graph, each step routing then
forward of one set), bracketed by a barrier and a device synchronisation. A
second timed pass of K/4 steps replays 8 routing launches, then 8 forward
launches, with CUDA events between the graphs: it gives the per-call average
durations used for the roofline and the route/forward breakdown.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=None)
    ap.add_argument("--variant", default="auto",
                    choices=["auto", "fused", "outside", "premix", "direct", "depthwise"])
    ap.add_argument("--batch", type=int, default=0,
                    help="override the configuration's batch size (small profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the layer's backward step (weight, router and input gradients)")
    ap.add_argument("--cells", type=int, default=0,
                    help="time the layer with its kernel assembled from this many warehouse cells")
    ap.add_argument("--warehouse", type=int, default=128, help="warehouse cells for --cells")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--per-config", default="all",
                    help="comma-separated configurations measured into the line's per_config "
                         "object ('all', or 'none' to skip); one GPU only")
    ap.add_argument("--hooks", default="",
                    help="implementation knobs for comparisons, e.g. '6=0,5=0' "
                         "(see dynconv_test_hook in include/dynconv.h)")
    return ap.parse_args()


def dist_env():
    from dynamic_convolution_b200 import multi
    return multi.dist_env()


def workload_name(cfg) -> str:
    return cfg.name


def config_dict(cfg, extra=None):
    d = {"workload": cfg.name, "B": cfg.B, "C_in": cfg.C_in, "C_out": cfg.C_out,
         "H": cfg.H, "W": cfg.W, "kernel": f"{cfg.KH}x{cfg.KW}", "stride": cfg.stride,
         "pad": cfg.pad, "groups": cfg.groups, "n_experts": cfg.n,
         "routing": "softmax" if cfg.mode == 1 else "sigmoid", "tau": cfg.tau}
    if extra:
        d.update(extra)
    return d


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# --------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- reference arm

def run_reference(args, cfg):
    """The fp64 CPU oracle, as it stands, on the host cores. Each step is a bounded
    sample of the workload: routing of one image plus one output row of its forward."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from dynamic_convolution_b200 import synth
    inp = synth.make_inputs(cfg)
    x = inp.x_f64
    Wr = inp.Wr.astype(np.float64)
    br = inp.br.astype(np.float64)
    E = inp.experts_f64
    bias = inp.bias.astype(np.float64)

    def step(k):
        b = k % cfg.B
        a = oracle.route(x[b:b + 1], Wr, br, cfg.mode, cfg.tau, nthreads=1)
        full_a = np.zeros((cfg.B, cfg.n))
        full_a[b] = a[0]
        oracle.forward_rows(x, E, full_a, bias, b, k % cfg.H_out, 1, stride=cfg.stride,
                            pad=cfg.pad, groups=cfg.groups)

    for k in range(args.warmup):
        step(k)
    t0 = time.perf_counter()
    for k in range(args.steps):
        step(k)
    dt = time.perf_counter() - t0
    images = args.steps / cfg.H_out          # one output row of H_out per step
    value = images / dt
    flops_per_img = cfg.conv_flops / cfg.B
    line = {
        "impl": "reference", "metric": "images/s per dynconv layer (route + forward)",
        "value": value, "unit": "images/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, {"sample": "route 1 image + 1 output row of its forward per step"}),
        "eff_tflops": value * flops_per_img / 1e12,
        "cpu_baseline": {"value": value, "unit": "images/s", "cores": 1, "kind": "oracle",
                         "sample": "per step: routing of one image and one output row of its "
                                   "forward (fp64 C oracle, one thread)"},
        "e2e": {"value": value, "unit": "images/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- our arm

def cpu_baseline(cfg, inp):
    import oracle
    cores = os.cpu_count() or 1
    nb = min(cfg.B, max(16, cores))
    x = inp.x_f64[:nb]
    t0 = time.perf_counter()
    a = oracle.route(x, inp.Wr, inp.br, cfg.mode, cfg.tau, nthreads=0)
    oracle.forward(x, inp.experts_f64, a, inp.bias, stride=cfg.stride, pad=cfg.pad,
                   groups=cfg.groups, nthreads=0)
    dt = time.perf_counter() - t0
    return {"value": nb / dt, "unit": "images/s", "cores": oracle.threads_used(0, nb),
            "kind": "oracle",
            "sample": f"route + forward of {nb} of the {cfg.B} images, fp64 C oracle, "
                      f"threads over images"}


def cpu_baseline_backward(cfg, inp, dy_f64, nb=None):
    """The oracle's backward step (expert, bias, attention, router and input
    gradients) on a bounded sample of the batch, timed on the host cores."""
    import oracle
    cores = os.cpu_count() or 1
    nb = nb or min(cfg.B, max(2, min(cores, 8)))
    x, dy = inp.x_f64[:nb], dy_f64[:nb]
    a = oracle.route(x, inp.Wr, inp.br, cfg.mode, cfg.tau)
    t0 = time.perf_counter()
    oracle.backward(x, dy, inp.experts_f64, a, inp.bias, inp.Wr, cfg.mode, cfg.tau,
                    stride=cfg.stride, pad=cfg.pad, groups=cfg.groups)
    dt = time.perf_counter() - t0
    return {"value": nb / dt, "unit": "images/s", "cores": oracle.threads_used(0, nb),
            "kind": "oracle",
            "sample": f"backward of {nb} of the {cfg.B} images (fp64 C oracle; weight and input "
                      f"gradients threaded over images, router gradients and sums over images "
                      f"on one thread)"}


def cpu_baseline_cells(cfg, ci, cells, n, nb=None):
    """The oracle's cell routing and forward on a bounded sample of the batch."""
    import oracle
    nb = nb or min(cfg.B, 4)
    x = ci.x_f64[:nb]
    t0 = time.perf_counter()
    a = oracle.route_cells(x, ci.Wr, ci.br, cells, cfg.mode, cfg.tau)
    oracle.forward_cells(x, ci.warehouse_f64, a, ci.bias, cfg.C_out, cfg.KH, cfg.KW, cfg.stride,
                         cfg.pad, cfg.groups)
    dt = time.perf_counter() - t0
    return {"value": nb / dt, "unit": "images/s", "cores": 1, "kind": "oracle",
            "sample": f"cell routing + forward of {nb} of the {cfg.B} images "
                      f"(fp64 C oracle, one thread)"}


def profile_traffic(kernel_tag: str, workload: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}__{workload}.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_hash") != src_hash:
        return None
    return d.get("dram_bytes_per_launch")


def _code_only(text: str) -> str:
    """C/C++ source without comments and blank space: what the compiler sees
    of it, so that an edit of a comment does not orphan the captured profiles."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(" ".join(line.split()) for line in text.splitlines() if line.strip())


def kernel_source_hash(csrc: str | None = None) -> str:
    """Hash of the forward translation unit's code: dynconv.cu and every csrc
    header it includes, directly or not (the backward and cell units compile
    separately and cannot change the forward kernels), comments and blank
    space left out."""
    csrc = csrc or os.path.join(ROOT, "dynamic_convolution_b200", "csrc")
    seen, todo = set(), ["dynconv.cu"]
    while todo:
        fn = todo.pop()
        if fn in seen or not os.path.exists(os.path.join(csrc, fn)):
            continue
        seen.add(fn)
        with open(os.path.join(csrc, fn)) as f:
            todo += re.findall(r'^#include "([^"]+)"', f.read(), flags=re.M)
    h = hashlib.sha256()
    for fn in sorted(seen):
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(fn.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def bound_of(cfg, peaks):
    """Roofline bound of a layer: tensor cores when its arithmetic intensity
    (conv FLOP per algorithmic byte, x + y + experts) is above the ridge of the
    two measured peaks and it is a dense bf16 layer, else HBM."""
    from dynamic_convolution_b200 import synth
    algo_bytes = (cfg.B * cfg.H * cfg.W * cfg.C_in + cfg.B * cfg.H_out * cfg.W_out * cfg.C_out
                  + cfg.n * cfg.weight_elems) * cfg.elem_bytes
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    tensor = (cfg.dtype == synth.BF16 and cfg.groups == 1
              and cfg.conv_flops / max(algo_bytes, 1) >= ridge)
    return ("tensor" if tensor else "hbm"), algo_bytes


def roofline_entry(cfg, launch_ms, kernel_label, peaks, peak_kind, traffic):
    bound, algo_bytes = bound_of(cfg, peaks)
    if bound == "tensor":
        achieved = cfg.conv_flops / (launch_ms / 1e3) / 1e12
        peak = float(peaks["bf16_tflops"])
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_kind": f"bf16 dense burst, {peak_kind}",
                "kernel": kernel_label, "traffic": traffic, "launch_ms": launch_ms,
                "algorithmic": f"{cfg.conv_flops} conv FLOP per launch (2*B*HW*Cout*Cin*KH*KW)"}
    achieved = algo_bytes / (launch_ms / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_kind": f"HBM copy, {peak_kind}",
            "kernel": kernel_label, "traffic": traffic, "launch_ms": launch_ms,
            "algorithmic": f"{algo_bytes} bytes per launch (x + y + experts)"}


def kernel_label_of(variant_name, cfg):
    if variant_name == "premix":
        mixer = "premix_small_kernel" if cfg.n <= 8 else "premix_kernel"
        return (f"forward call: {mixer} + the PREMIX convolution (tc_conv_persist_kernel "
                f"or tc_conv_kernel<premix>, as planned)")
    if variant_name in ("fused", "outside"):
        return f"tc_conv_kernel<{variant_name}>"
    return f"{variant_name}_kernel"


class GraphTimer:
    """Per-call device times of captured calls: each call is one CUDA graph;
    cold reps first READ a buffer of twice the L2 size (every input, expert and
    workspace byte of the call then comes from HBM; a read leaves no dirty
    lines that would drain to HBM during the timed call, as a write would),
    warm reps repeat the call back to back. Events are recorded on the stream
    the graphs replay on."""

    def __init__(self, torch, stream):
        self.torch = torch
        self.stream = stream
        self.flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda")
        self.sink = None

    def capture(self, fn):
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g, stream=self.stream):
            fn(self.stream)
        return g

    def median_ms(self, g, reps, cold):
        torch = self.torch
        g.replay()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        with torch.cuda.stream(self.stream):
            for k, (e0, e1) in enumerate(evs):
                if cold:
                    self.sink = self.flush.sum()
                e0.record(self.stream)
                g.replay()
                e1.record(self.stream)
        self.stream.synchronize()
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)


def measure_config(name, args, peaks, peak_kind, src_hash):
    """One layer configuration on one GPU, for the line's per_config object:
    steps of routing + forward as CUDA-graph replays over rotating input sets
    (ms_per_step, with the clocks sampled meanwhile), the median of >= 50 cold
    and of >= 50 warm per-call times of the routing and the forward call (the
    roofline uses the cold forward median), the forward of every variant that
    takes the shape, the oracle on a bounded sample of the batch, and the
    end-to-end rate through the public calls with host buffers."""
    import torch

    import dynamic_convolution_b200 as dc
    from dynamic_convolution_b200 import synth

    cfg = synth.CONFIGS[name]
    reps = max(args.steps, 50)
    med_reps = min(reps, 1000)  # per-call medians: enough samples, bounded run time
    inp = synth.make_inputs(cfg)
    tdt = torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32
    dev = lambda a: (torch.from_numpy(a).view(torch.bfloat16) if cfg.dtype == synth.BF16
                     else torch.from_numpy(a)).cuda()
    x0, E = dev(inp.x_store), dev(inp.experts_store)
    Wr, br, bias = (torch.from_numpy(a).cuda() for a in (inp.Wr, inp.br, inp.bias))
    desc = dc.desc_from_config(cfg)
    ws_bytes = dc.dynconv_workspace_size(desc)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    chosen = dc.dynconv_select_variant(desc, ws_bytes)
    vname = dc.VARIANT_NAMES.get(chosen, str(chosen))
    set_bytes = 2 * x0.numel() * x0.element_size()
    nsets = max(2, min(64, math.ceil(2 * L2_BYTES / set_bytes)))
    xs = [x0] + [x0.clone() for _ in range(nsets - 1)]
    ys = [torch.empty((cfg.B, cfg.H_out, cfg.W_out, cfg.C_out), dtype=tdt, device="cuda")
          for _ in range(nsets)]
    alphas = [torch.empty((cfg.B, cfg.n), device="cuda") for _ in range(nsets)]
    stream = torch.cuda.Stream()
    timer = GraphTimer(torch, stream)

    def route(s, st, d=desc):
        dc.check(dc.dynconv_route(d, xs[s], Wr, br, cfg.mode, cfg.tau, alphas[s], st), "route")

    def forward(s, st, d=desc):
        dc.check(dc.dynconv_forward(d, xs[s], E, alphas[s], bias, ys[s], ws, ws_bytes, st),
                 "forward")

    with torch.cuda.stream(stream):
        for k in range(max(args.warmup, 10)):
            route(k % nsets, stream)
            forward(k % nsets, stream)
    stream.synchronize()
    dc.check(dc.dynconv_device_status(stream), f"{name}: device status after warm-up")

    # steps: graphs of up to 8 (route, forward) pairs over rotating sets
    G = min(8, nsets)
    n0 = dc.dynconv_launch_count()
    graphs = []
    for g0 in range(0, nsets - G + 1, G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for s in range(g0, g0 + G):
                route(s, stream)
                forward(s, stream)
        graphs.append(g)
    launches_per_step = (dc.dynconv_launch_count() - n0) / (len(graphs) * G)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    graphs[0].replay()
    torch.cuda.synchronize()
    est = max(time.perf_counter() - t0, 1e-6)
    n_rep = max(math.ceil(reps / G), min(4000, math.ceil(0.25 / est)))
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.1)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(n_rep):
            graphs[i % len(graphs)].replay()
        e1.record(stream)
    stream.synchronize()
    clocks = sampler.stop()
    step_ms = e0.elapsed_time(e1) / (n_rep * G)
    del graphs

    # per-call medians, cold (L2 flushed first) and warm
    g_route = timer.capture(lambda st: route(0, st))
    g_fwd = timer.capture(lambda st: forward(0, st))
    route_cold = timer.median_ms(g_route, med_reps, True)
    fwd_cold = timer.median_ms(g_fwd, med_reps, True)
    route_warm = timer.median_ms(g_route, med_reps, False)
    fwd_warm = timer.median_ms(g_fwd, med_reps, False)
    del g_route, g_fwd
    dc.check(dc.dynconv_device_status(stream), f"{name}: device status after timing")

    # every variant that takes the shape (cold forward medians)
    variants = {}
    cand = ([dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE, dc.VARIANT_PREMIX]
            if cfg.dtype == synth.BF16 and cfg.groups == 1 else
            [dc.VARIANT_DEPTHWISE] if cfg.groups > 1 else [dc.VARIANT_DIRECT])
    for v in cand:
        dv = dc.desc_from_config(cfg, v)
        # a plain call first: a variant that refuses the shape is skipped
        # (it returns before launching anything)
        if dc.dynconv_forward(dv, xs[0], E, alphas[0], bias, ys[0], ws, ws_bytes, stream) != 0:
            continue
        stream.synchronize()
        g = timer.capture(lambda st, dv=dv: forward(0, st, dv))
        variants[dc.VARIANT_NAMES[v]] = timer.median_ms(g, min(med_reps, 200), True)
        del g
    dc.check(dc.dynconv_device_status(stream), f"{name}: device status after variants")

    # end to end: host x in, y out, copies inside the timed region
    e2e = measure_e2e(torch, dc, cfg, inp, desc, xs, alphas, ys, Wr, br, E, bias, ws_bytes,
                      max(20, min(reps, 200)), tdt, nsets)

    cpu = None if args.no_cpu_baseline else cpu_baseline(cfg, inp)
    traffic = profile_traffic(vname, cfg.name, src_hash)
    label = kernel_label_of(vname, cfg)
    entry = {
        "variant": vname, "dtype": "bf16" if cfg.dtype == synth.BF16 else "f32",
        "ms_per_step": step_ms, "images_per_s": cfg.B / (step_ms / 1e3),
        "forward_ms": fwd_cold, "route_ms": route_cold,
        "forward_ms_warm_l2": fwd_warm, "route_ms_warm_l2": route_warm,
        "forward_images_per_s": cfg.B / (fwd_cold / 1e3),
        "forward_eff_tflops": cfg.conv_flops / (fwd_cold / 1e3) / 1e12,
        "roofline": roofline_entry(cfg, fwd_cold, label, peaks, peak_kind, traffic),
        "variants_forward_ms": variants,
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches_per_step": launches_per_step,
        "timing": (f"ms_per_step: mean over {n_rep * G} graph-replayed steps over {nsets} input "
                   f"sets; *_ms: median of {reps} calls, cold = after reading "
                   f"{2 * L2_BYTES >> 20} MiB (2x L2), warm = back to back"),
    }
    if cfg.dtype == synth.BF16 and cfg.groups == 1:
        entry["mixing_gflop"] = 2.0 * cfg.B * cfg.n * cfg.weight_elems / 1e9
    del xs, ys, alphas, E, ws, timer
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry


def measure_e2e(torch, dc, cfg, inp, desc, xs, alphas, ys, Wr, br, E, bias, ws_bytes, steps,
                tdt, nsets):
    """Routing + forward through the public calls with the input copied in from
    pinned host memory and the output copied back every step, alternating over
    two streams (own buffers and workspace each) so that copies in, kernels and
    copies out of neighbouring steps overlap."""
    from dynamic_convolution_b200 import synth
    xh = torch.from_numpy(inp.x_store).pin_memory()
    if cfg.dtype == synth.BF16:
        xh = xh.view(torch.bfloat16)
    n_e2e = 2
    streams = [torch.cuda.Stream() for _ in range(n_e2e)]
    yhs = [torch.empty(ys[0].shape, dtype=tdt).pin_memory() for _ in range(n_e2e)]
    wss = [torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda") for _ in range(n_e2e)]
    per = max(1, nsets // n_e2e)

    def step(k):
        j = k % n_e2e
        st, s = streams[j], k % (n_e2e * per)
        with torch.cuda.stream(st):
            xs[s].copy_(xh, non_blocking=True)
            dc.check(dc.dynconv_route(desc, xs[s], Wr, br, cfg.mode, cfg.tau, alphas[s], st))
            dc.check(dc.dynconv_forward(desc, xs[s], E, alphas[s], bias, ys[s], wss[j], ws_bytes,
                                        st))
            yhs[j].copy_(ys[s], non_blocking=True)

    for k in range(2 * n_e2e):
        step(k)
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for st in streams:
        st.wait_event(e0)
    for k in range(steps):
        step(k)
    for st in streams:
        main.wait_stream(st)
    e1.record(main)
    main.synchronize()
    ms = e0.elapsed_time(e1)
    return {"value": cfg.B * steps / (ms / 1e3), "unit": "images/s",
            "h2d_bytes_per_step": int(xh.numel() * xh.element_size()),
            "d2h_bytes_per_step": int(yhs[0].numel() * yhs[0].element_size()),
            "streams": n_e2e, "steps": steps}


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    import dynamic_convolution_b200 as dc
    from dynamic_convolution_b200 import build, multi, synth

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.cuda.current_device()
    build.build()
    dc.load()

    variant = {"auto": 0, "fused": 1, "outside": 2, "premix": 3, "direct": 4,
               "depthwise": 5}[args.variant]
    hooks = {}
    for kv in filter(None, args.hooks.split(",")):
        k, v = kv.split("=")
        hooks[int(k)] = int(v)
        dc.check(dc.dynconv_test_hook(int(k), int(v)), f"test hook {kv}")
    inp = synth.make_inputs(cfg, seed=rank)
    desc = dc.desc_from_config(cfg, variant)
    tdt = torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32

    def dev_tensor(a):
        if cfg.dtype == synth.BF16:
            return torch.from_numpy(a).view(torch.bfloat16).cuda()
        return torch.from_numpy(a).cuda()

    x0 = dev_tensor(inp.x_store)
    experts = dev_tensor(inp.experts_store)
    Wr = torch.from_numpy(inp.Wr).cuda()
    br = torch.from_numpy(inp.br).cuda()
    bias = torch.from_numpy(inp.bias).cuda()
    set_bytes = x0.numel() * x0.element_size() * 2
    nsets = max(2, math.ceil(2 * L2_BYTES / set_bytes))
    nsets = min(nsets, 64)
    xs = [x0] + [x0.clone() for _ in range(nsets - 1)]
    ys = [torch.empty((cfg.B, cfg.H_out, cfg.W_out, cfg.C_out), dtype=tdt, device="cuda")
          for _ in range(nsets)]
    alphas = [torch.empty((cfg.B, cfg.n), dtype=torch.float32, device="cuda") for _ in range(nsets)]
    ws_bytes = dc.dynconv_workspace_size(desc)
    workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    chosen = dc.dynconv_select_variant(desc, ws_bytes)

    stream = torch.cuda.Stream()

    def route(s, st):
        dc.check(dc.dynconv_route(desc, xs[s], Wr, br, cfg.mode, cfg.tau, alphas[s], st), "route")

    def forward(s, st):
        dc.check(dc.dynconv_forward(desc, xs[s], experts, alphas[s], bias, ys[s], workspace,
                                    ws_bytes, st), "forward")

    # warm-up outside capture (also sets kernel attributes once)
    with torch.cuda.stream(stream):
        for k in range(max(args.warmup, 3)):
            route(k % nsets, stream)
            forward(k % nsets, stream)
    stream.synchronize()
    st = dc.dynconv_device_status(stream)
    dc.check(st, "device status after warm-up")

    # Timed graphs: each step is route(s) then forward(s) of one input set, as a
    # layer runs in a network (the forward reads x while the routing kernel
    # left it in L2; the routing -> mixing edge is programmatic). A second,
    # shorter timed pass replays all routes of a group, then all forwards, so
    # that CUDA events between the two graphs give each call's duration.
    G = min(8, nsets)
    groups = [list(range(g, min(g + G, nsets))) for g in range(0, nsets, G)]
    steps_graphs, split_graphs = [], []
    n0 = dc.dynconv_launch_count()
    for grp in groups:
        gs = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gs, stream=stream):
            for s in grp:
                route(s, stream)
                forward(s, stream)
        steps_graphs.append((gs, len(grp)))
    launches_per_step = (dc.dynconv_launch_count() - n0) / nsets
    for grp in groups:
        gr, gf = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for s in grp:
                route(s, stream)
        with torch.cuda.graph(gf, stream=stream):
            for s in grp:
                forward(s, stream)
        split_graphs.append((gr, gf, len(grp)))
    tails = {}
    for s in range(nsets):  # single-step graphs for an exact step count
        gt = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gt, stream=stream):
            route(s, stream)
            forward(s, stream)
        tails[s] = gt
    for gs, _ in steps_graphs:  # warm the graphs
        gs.replay()
    for gr, gf, _ in split_graphs:
        gr.replay()
        gf.replay()
    torch.cuda.synchronize()

    # schedule of exactly K steps
    plan = []
    k = 0
    gi = 0
    while k < args.steps:
        gs, m = steps_graphs[gi % len(steps_graphs)]
        if k + m <= args.steps:
            plan.append(gs)
            k += m
        else:
            for s in range(args.steps - k):
                plan.append(tails[s])
            k = args.steps
        gi += 1
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    sampler = ClockSampler(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.2)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for gs in plan:
            gs.replay()
        ev1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    total_ms = ev0.elapsed_time(ev1)
    st = dc.dynconv_device_status(stream)
    dc.check(st, "device status after timing")

    # per-call durations (routing, forward) from the split pass
    split_groups = max(1, (args.steps // 4) // G)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * split_groups + 1)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for i in range(split_groups):
            gr, gf, m = split_graphs[i % len(split_graphs)]
            gr.replay()
            ev[2 * i + 1].record(stream)
            gf.replay()
            ev[2 * i + 2].record(stream)
    stream.synchronize()
    split_steps = sum(split_graphs[i % len(split_graphs)][2] for i in range(split_groups))
    route_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(split_groups))
    fwd_ms = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(split_groups))
    route_ms *= args.steps / split_steps  # scaled to K steps, like total_ms
    fwd_ms *= args.steps / split_steps
    st = dc.dynconv_device_status(stream)
    dc.check(st, "device status after the split pass")

    total_ms, fwd_ms, route_ms = multi.max_over_ranks([total_ms, fwd_ms, route_ms], device="cuda")

    # ---- end to end through the public API, host buffers, copies inside the timed region.
    # Steps alternate over two streams, each with its own device buffers, host
    # output buffer and PREMIX workspace, so that one step's host->device copy,
    # another's kernels and another's device->host copy overlap (the two copy
    # directions use separate copy engines). Every step still copies its own
    # input in and its own output back.
    xh = torch.from_numpy(inp.x_store).pin_memory()
    if cfg.dtype == synth.BF16:
        xh = xh.view(torch.bfloat16)
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    n_e2e = 2
    e2e_streams = [torch.cuda.Stream() for _ in range(n_e2e)]
    yhs = [torch.empty(ys[0].shape, dtype=tdt).pin_memory() for _ in range(n_e2e)]
    wss = [workspace] + [torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
                         for _ in range(n_e2e - 1)]

    def e2e_step(k):
        # set k mod (an even number of sets): every set is used by one stream only
        j = k % n_e2e
        st, s = e2e_streams[j], k % (n_e2e * max(1, nsets // n_e2e))
        with torch.cuda.stream(st):
            xs[s].copy_(xh, non_blocking=True)
            dc.check(dc.dynconv_route(desc, xs[s], Wr, br, cfg.mode, cfg.tau, alphas[s], st))
            dc.check(dc.dynconv_forward(desc, xs[s], experts, alphas[s], bias, ys[s], wss[j],
                                        ws_bytes, st))
            yhs[j].copy_(ys[s], non_blocking=True)

    for k in range(2 * n_e2e):  # warm-up of the copies on both streams
        e2e_step(k)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for st in e2e_streams:
        st.wait_event(e0)
    for k in range(e2e_steps):
        e2e_step(k)
    for st in e2e_streams:
        stream.wait_stream(st)
    e1.record(stream)
    stream.synchronize()
    e2e_ms = multi.max_over_ranks([e0.elapsed_time(e1)], device="cuda")[0]
    if world > 1:
        dist.barrier()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    del steps_graphs, split_graphs, tails, plan
    peaks, peak_kind = measured_peaks()
    K = args.steps
    value = multi.weak_scaling_rate(cfg.B * K, world, total_ms / 1e3)
    fwd_launch_ms = fwd_ms / K
    route_launch_ms = route_ms / K
    conv_flops = cfg.conv_flops
    eb = cfg.elem_bytes
    algo_bytes = (cfg.B * cfg.H * cfg.W * cfg.C_in + cfg.B * cfg.H_out * cfg.W_out * cfg.C_out
                  + cfg.n * cfg.weight_elems) * eb
    src_hash = kernel_source_hash()
    variant_name = dc.VARIANT_NAMES.get(chosen, str(chosen))
    # the bound: tensor cores when the layer's arithmetic intensity (conv FLOP per
    # algorithmic byte) is above the ridge of the two measured peaks, else HBM
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    tensor_bound = (cfg.dtype == synth.BF16 and cfg.groups == 1
                    and conv_flops / max(algo_bytes, 1) >= ridge)
    kernel_label = kernel_label_of(variant_name, cfg)
    if tensor_bound:
        achieved = conv_flops / (fwd_launch_ms / 1e3) / 1e12
        peak = float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_kind": f"bf16 dense burst, {peak_kind}",
                "kernel": kernel_label,
                "algorithmic": f"{conv_flops} conv FLOP per launch (2*B*HW*Cout*Cin*KH*KW)"}
    else:
        achieved = algo_bytes / (fwd_launch_ms / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": f"HBM copy, {peak_kind}",
                "kernel": kernel_label,
                "algorithmic": f"{algo_bytes} bytes per launch (x + y + experts)"}
    roof["traffic"] = profile_traffic(variant_name, cfg.name, src_hash)
    roof["launch_ms"] = fwd_launch_ms

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, inp)

    line = {
        "metric": "images/s per dynconv layer (route + forward)",
        "value": value, "unit": "images/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.dtype == synth.BF16 else "f32",
        "data": "synthetic (seeded normal draws, layer shapes of the configuration)",
        "config": config_dict(cfg, {"variant": variant_name,
                                    "l2": f"inputs rotated over {nsets} x/y sets "
                                          f"({nsets * set_bytes / 2**20:.0f} MiB > 126 MiB L2)",
                                    "parallelism": f"dp{world} (independent batches)"}),
        "eff_tflops": world * conv_flops * K / (total_ms / 1e3) / 1e12,
        "forward_ms": fwd_launch_ms, "route_ms": route_launch_ms,
        "forward_images_per_s": cfg.B / (fwd_launch_ms / 1e3),
        "forward_eff_tflops": conv_flops / (fwd_launch_ms / 1e3) / 1e12,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": multi.weak_scaling_rate(cfg.B * e2e_steps, world, e2e_ms / 1e3),
                "unit": "images/s",
                "h2d_bytes_per_step": int(xh.numel() * xh.element_size()),
                "d2h_bytes_per_step": int(yhs[0].numel() * yhs[0].element_size()),
                "streams": n_e2e,
                "steps": e2e_steps},
        "gpu_launches": int(round(launches_per_step * K)),
        "clocks": clocks,
        "source_hash": src_hash,
        "hooks": hooks or None,
    }
    if world == 1 and args.per_config != "none":
        names = list(synth.CONFIGS) if args.per_config == "all" else args.per_config.split(",")
        line["per_config"] = {nm: measure_config(nm, args, peaks, peak_kind, src_hash)
                              for nm in names}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_block(args):
    """The chained EfficientNet-style block (1x1 expand layer, then the depthwise
    5x5 layer on its output), one GPU. Step = both layers' routing and forward.
    Times the block with the depthwise layer's routing pooled in the expand
    layer's epilogue (dynconv_forward_pooled + dynconv_route_pooled) and, for
    comparison, with the routing kernel reading the intermediate tensor again.
    CUDA graphs of 8 steps over rotating input sets larger than L2."""
    import torch

    import dynamic_convolution_b200 as dc
    from dynamic_convolution_b200 import build, synth

    torch.cuda.set_device(0)
    build.build()
    dc.load()
    up, dw = synth.CONFIGS["effnet_expand_1x1"], synth.CONFIGS["effnet_dw_5x5"]
    ia, ib = synth.make_inputs(up), synth.make_inputs(dw)
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
    Ea, Eb = bf(ia.experts_store), bf(ib.experts_store)
    Wra, bra, biasa = (torch.from_numpy(a).cuda() for a in (ia.Wr, ia.br, ia.bias))
    Wrb, brb, biasb = (torch.from_numpy(a).cuda() for a in (ib.Wr, ib.br, ib.bias))
    da, db = dc.desc_from_config(up), dc.desc_from_config(dw)
    wsa = dc.dynconv_workspace_size(da)
    ws = torch.empty(max(wsa, 16), dtype=torch.uint8, device="cuda")
    parts = dc.dynconv_pool_parts(da, wsa)
    x0 = bf(ia.x_store)
    set_bytes = 2 * x0.numel() * 2 + 2 * up.B * up.H * up.W * up.C_out * 2
    nsets = max(2, min(64, math.ceil(2 * L2_BYTES / set_bytes)))
    xs = [x0.clone() for _ in range(nsets)]
    mids = [torch.empty((up.B, up.H, up.W, up.C_out), dtype=torch.bfloat16, device="cuda")
            for _ in range(nsets)]
    outs = [torch.empty_like(m) for m in mids]
    aa = [torch.empty((up.B, up.n), device="cuda") for _ in range(nsets)]
    ab = [torch.empty((dw.B, dw.n), device="cuda") for _ in range(nsets)]
    ysum = [torch.empty((up.B, parts, up.C_out), device="cuda") for _ in range(nsets)]
    stream = torch.cuda.Stream()

    def step(s, pooled, st):
        dc.check(dc.dynconv_route(da, xs[s], Wra, bra, up.mode, up.tau, aa[s], st))
        if pooled:
            dc.check(dc.dynconv_forward_pooled(da, xs[s], Ea, aa[s], biasa, mids[s], ysum[s], ws,
                                               wsa, st))
            dc.check(dc.dynconv_route_pooled(db, ysum[s], parts, Wrb, brb, dw.mode, dw.tau, ab[s],
                                             st))
        else:
            dc.check(dc.dynconv_forward(da, xs[s], Ea, aa[s], biasa, mids[s], ws, wsa, st))
            dc.check(dc.dynconv_route(db, mids[s], Wrb, brb, dw.mode, dw.tau, ab[s], st))
        dc.check(dc.dynconv_forward(db, mids[s], Eb, ab[s], biasb, outs[s], None, 0, st))

    res = {}
    for pooled in (True, False):
        with torch.cuda.stream(stream):
            for k in range(max(args.warmup, 3)):
                step(k % nsets, pooled, stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for s in range(min(8, nsets)):
                step(s, pooled, stream)
        reps = max(1, args.steps // min(8, nsets))
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        dc.check(dc.dynconv_device_status(stream), "device status")
        res[pooled] = e0.elapsed_time(e1) / (reps * min(8, nsets))
        del g
    ms = res[True]
    line = {"metric": "images/s per block (1x1 expand + depthwise 5x5, routing + forward)",
            "value": up.B / (ms / 1e3), "unit": "images/s", "n_gpus": 1,
            "steps": reps * min(8, nsets), "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal draws, layer shapes of the configuration)",
            "config": {"workload": "effnet_block (effnet_expand_1x1 -> effnet_dw_5x5)",
                       "routing_pool": "depthwise routing pooled in the expand epilogue",
                       "l2": f"inputs rotated over {nsets} sets"},
            "unpooled_ms_per_step": res[False],
            "unpooled_images_per_s": up.B / (res[False] / 1e3)}
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, cfg):
    """One layer's backward step on one GPU: dynconv_backward_weight,
    dynconv_route_backward and dynconv_backward_data, with inputs, upstream
    gradients and dx rotated over sets larger than L2 in total, in CUDA graphs
    of 8 steps. Also times each call alone (same graphs, one call per step).
    Effective TFLOP/s counts the two convolution-sized contractions (weight
    gradient and input gradient): 2 x the forward's conv FLOPs."""
    import torch

    import dynamic_convolution_b200 as dc
    from dynamic_convolution_b200 import build, synth

    torch.cuda.set_device(0)
    build.build()
    dc.load()
    inp = synth.make_inputs(cfg)
    dys, _ = synth.make_upstream_grad(cfg)
    tdt = torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32
    dev = lambda a: (torch.from_numpy(a).view(torch.bfloat16) if cfg.dtype == synth.BF16
                     else torch.from_numpy(a)).cuda()
    x0, dy0, E = dev(inp.x_store), dev(dys), dev(inp.experts_store)
    Wr, br, bias = (torch.from_numpy(a).cuda() for a in (inp.Wr, inp.br, inp.bias))
    d = dc.desc_from_config(cfg)
    wsb = dc.dynconv_backward_workspace_size(d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    set_bytes = (2 * x0.numel() + dy0.numel()) * x0.element_size()
    nsets = max(2, min(64, math.ceil(2 * L2_BYTES / set_bytes)))
    xs = [x0.clone() for _ in range(nsets)]
    dys_ = [dy0.clone() for _ in range(nsets)]
    dxs = [torch.empty_like(x0) for _ in range(nsets)]
    alphas = [torch.empty((cfg.B, cfg.n), device="cuda") for _ in range(nsets)]
    for k in range(nsets):
        dc.check(dc.dynconv_route(d, xs[k], Wr, br, cfg.mode, cfg.tau, alphas[k]))
    dE = torch.empty(E.shape, dtype=torch.float32, device="cuda")
    dbias = torch.empty((cfg.n, cfg.C_out), device="cuda")
    dalpha = torch.empty((cfg.B, cfg.n), device="cuda")
    dWr = torch.empty((cfg.n, cfg.C_in), device="cuda")
    dbr = torch.empty(cfg.n, device="cuda")
    dg = torch.empty((cfg.B, cfg.C_in), device="cuda")
    stream = torch.cuda.Stream()

    def weight(s, st):
        dc.check(dc.dynconv_backward_weight(d, xs[s], dys_[s], E, alphas[s], bias, dE, dbias,
                                            dalpha, ws, wsb, st))

    def router(s, st):
        dc.check(dc.dynconv_route_backward(d, xs[s], Wr, alphas[s], dalpha, cfg.mode, cfg.tau,
                                           dWr, dbr, dg, ws, wsb, st))

    def data(s, st):
        dc.check(dc.dynconv_backward_data(d, dys_[s], E, alphas[s], dg, dxs[s], ws, wsb, st))

    def full(s, st):
        weight(s, st)
        router(s, st)
        data(s, st)

    def timed(fn):
        with torch.cuda.stream(stream):
            for k in range(max(args.warmup, 3)):
                fn(k % nsets, stream)
        stream.synchronize()
        per = min(8, nsets)
        g = torch.cuda.CUDAGraph()
        n0 = dc.dynconv_launch_count()
        with torch.cuda.graph(g, stream=stream):
            for k in range(per):
                fn(k, stream)
        launches = (dc.dynconv_launch_count() - n0) // per
        reps = max(1, args.steps // per)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        dc.check(dc.dynconv_device_status(stream), "device status")
        del g
        return e0.elapsed_time(e1) / (reps * per), reps * per, launches

    ms, steps, launches = timed(full)
    parts = {name: round(timed(fn)[0] * 1e3, 2) for name, fn in
             (("backward_weight", weight), ("route_backward", router), ("backward_data", data))}
    tflops = 2 * cfg.conv_flops / (ms / 1e3) / 1e12
    line = {"metric": "images/s (layer backward: expert, bias, attention, router and input "
                      "gradients)",
            "value": cfg.B / (ms / 1e3), "unit": "images/s", "n_gpus": 1, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if cfg.dtype == synth.BF16 else "f32",
            "data": "synthetic (seeded normal draws, layer shapes of the configuration)",
            "config": {"workload": f"{cfg.name} backward", "l2": f"inputs rotated over {nsets} sets"},
            "effective_tflops": tflops, "us_per_call": parts, "gpu_launches_per_step": launches,
            "cpu_baseline": None if args.no_cpu_baseline else cpu_baseline_backward(
                cfg, inp, synth.make_upstream_grad(cfg)[1]),
            "wgrad_kernel": ("tcgen05" if cfg.dtype == synth.BF16 and cfg.groups == 1
                             and cfg.stride == 1 and cfg.C_in % 8 == 0 and cfg.C_out % 8 == 0
                             else "cuda-core depthwise" if cfg.dtype == synth.BF16
                             and cfg.groups == cfg.C_in == cfg.C_out and cfg.C_in % 8 == 0
                             else "cuda-core")}
    print(json.dumps(line), flush=True)
    return 0


def run_cells(args, cfg):
    """The layer with its kernel assembled from warehouse cells, one GPU: step =
    dynconv_route_cells + dynconv_forward_cells of one batch, CUDA graphs of 8
    steps, inputs rotated over sets larger than L2 in total."""
    import torch

    import dynamic_convolution_b200 as dc
    from dynamic_convolution_b200 import build, synth

    torch.cuda.set_device(0)
    build.build()
    dc.load()
    cells, n = args.cells, args.warehouse
    ci = synth.make_cell_inputs(cfg, cells, n)
    dev = lambda a: (torch.from_numpy(a).view(torch.bfloat16) if cfg.dtype == synth.BF16
                     else torch.from_numpy(a)).cuda()
    x0, E = dev(ci.x_store), dev(ci.warehouse_store)
    Wr, br, bias = (torch.from_numpy(a).cuda() for a in (ci.Wr, ci.br, ci.bias))
    d = dc.make_desc(cfg.B, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.KH, cfg.KW, cfg.stride,
                     cfg.pad, cfg.groups, n, cfg.dtype)
    wsb = dc.dynconv_cells_workspace_size(d, cells)
    if wsb == 0:
        raise SystemExit(f"{cfg.name}: {cells} cells do not divide the kernel into 16-byte cells")
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    tdt = torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32
    set_bytes = x0.numel() * x0.element_size() + cfg.B * cfg.H_out * cfg.W_out * cfg.C_out * 2
    nsets = max(2, min(64, math.ceil(2 * L2_BYTES / set_bytes)))
    xs = [x0.clone() for _ in range(nsets)]
    ys = [torch.empty((cfg.B, cfg.H_out, cfg.W_out, cfg.C_out), dtype=tdt, device="cuda")
          for _ in range(nsets)]
    alphas = [torch.empty((cfg.B, cells, n), device="cuda") for _ in range(nsets)]
    stream = torch.cuda.Stream()

    def step(k, st):
        dc.check(dc.dynconv_route_cells(d, cells, xs[k], Wr, br, cfg.mode, cfg.tau, alphas[k],
                                        ws, wsb, st))
        dc.check(dc.dynconv_forward_cells(d, cells, xs[k], E, alphas[k], bias, ys[k], ws, wsb, st))

    with torch.cuda.stream(stream):
        for k in range(max(args.warmup, 3)):
            step(k % nsets, stream)
    stream.synchronize()
    per = min(8, nsets)
    g = torch.cuda.CUDAGraph()
    n0 = dc.dynconv_launch_count()
    with torch.cuda.graph(g, stream=stream):
        for k in range(per):
            step(k, stream)
    launches = (dc.dynconv_launch_count() - n0) // per
    reps = max(1, args.steps // per)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    dc.check(dc.dynconv_device_status(stream), "device status")
    ms = e0.elapsed_time(e1) / (reps * per)
    del g
    mix_flops = 2.0 * cfg.B * cfg.C_out * cfg.KH * cfg.KW * cfg.Cg * n
    line = {"metric": "images/s (warehouse cells: route + forward)",
            "value": cfg.B / (ms / 1e3), "unit": "images/s", "n_gpus": 1, "steps": reps * per,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if cfg.dtype == synth.BF16 else "f32",
            "data": "synthetic (seeded normal draws, layer shapes of the configuration)",
            "config": {"workload": f"{cfg.name} from {cells} cells, warehouse of {n} cells",
                       "l2": f"inputs rotated over {nsets} sets"},
            "conv_tflops": cfg.conv_flops / (ms / 1e3) / 1e12,
            "mixing_gflop": mix_flops / 1e9, "gpu_launches_per_step": launches,
            "cpu_baseline": None if args.no_cpu_baseline else cpu_baseline_cells(cfg, ci, cells, n)}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    from dynamic_convolution_b200 import synth
    if args.config == "effnet_block":
        return run_block(args)
    if args.backward:
        return run_backward(args, synth.CONFIGS[args.config or synth.HEADLINE])
    if args.cells:
        return run_cells(args, synth.CONFIGS[args.config or synth.HEADLINE])
    name = args.config or synth.HEADLINE
    cfg = synth.CONFIGS[name]
    if args.batch > 0:
        cfg = cfg.scaled(B=args.batch, name=f"{cfg.name}_b{args.batch}")
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
