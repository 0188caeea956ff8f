"""Benchmark of the NVFP4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {native,reference}]

Headline (``value``): W4A16 decode throughput in GB/s on the four linears of a
27B-shaped decoder layer (fused QKV 5120->10240, o_proj 5120->5120, fused
gate+up 5120->34816, down 17408->5120) at M = 1 token.  One step runs the four
linears once.  Bytes per step are algorithmic: packed codes (N*K/2) + E4M3
scales (N*K/16) + bf16 activations (M*K*2) + the fp32 global scale, for each
linear.  Weights are quantized on the device by ``nvfp4_quantize`` and rotated
over two copies (389 MB > the 126 MB L2), so every step streams from HBM.

Also reported in the same JSON line (measured outside the headline's timed
region): the decode sweep M in {1, 2, 4, 8, 16, 32} per shape, prefill W4A4
TFLOP/s, the activation quantizer, one MoE layer, and the 64-layer decode stack
(the four linears per layer chained through the library's rms / silu kernels).

``--impl reference`` times the CPU oracle (the method's plain restatement) on
the same workload and metric, on this host's cores.  With more than one GPU
the runs are replicas (the layer does not shard here): every rank runs the
same workload on its own GPU, the step time is the max over ranks and
``value`` counts all ranks' bytes.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 linear: decode GB/s (% HBM peak); prefill TFLOPS (% FP4 tensor peak)"
SHAPES = (("qkv", 5120, 10240, 1), ("o_proj", 5120, 5120, 2), ("gate_up", 5120, 34816, 3),
          ("down", 17408, 5120, 4))
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
WORKLOAD = ("dense27b decode linears (QKV 5120x10240, o_proj 5120x5120, gate_up 5120x34816, down 17408x5120), "
            "W4A16, M=1")


def decode_bytes(M, K, N):
    return N * K // 2 + N * K // 16 + M * K * 2 + 4


STEP_BYTES = sum(decode_bytes(1, K, N) for _, K, N, _ in SHAPES)


def workload_config(world: int) -> dict:
    """The headline workload, identical in both arms' lines."""
    return {"workload": WORKLOAD, "M": 1, "bytes_per_step": STEP_BYTES,
            "l2": "weights 194.7 MB per step > 126 MB L2 (the native arm rotates 2 copies, 389 MB)",
            "parallelism": f"replicas x{world}"}


def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time (every rank gets it); ``ms`` unchanged on one rank."""
    if not dist:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: int, ms_per_step: float) -> float:
    """Aggregate GB/s of `world` replicas that each stream `bytes_per_step` per step."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic(kernel_src: str, name: str):
    """DRAM bytes of one decode step (the kernel's 4 launches) from a committed
    ncu summary, if it was taken on the current source of the kernel (matched
    by hash); else None."""
    src = os.path.join(ROOT, "bit_linear_moe_b200", "csrc", kernel_src)
    p = os.path.join(ROOT, "profiles", f"{name}.traffic.txt")
    if not (os.path.exists(src) and os.path.exists(p)):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(p):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != h:
        return None
    try:
        return float(vals["dram_bytes_per_step"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ native ----

def run_native(args, rank, world, dist):
    import torch
    import bit_linear_moe_b200 as nv
    from bit_linear_moe_b200 import synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    # weights: fp32 on the host (seeded), quantized on the device, two copies
    layers = []
    for name, K, N, seed in SHAPES:
        w = torch.from_numpy(synth.dense_weight(seed, K, N)).to(dev)
        codes, scales, gs = nv.nvfp4_quantize(w, sf_layout=nv.SF_TILED)
        del w
        copies = [(codes, scales, gs), (codes.clone(), scales.clone(), gs.clone())]
        x = torch.from_numpy(synth.decode_x(seed, 1, K)).to(torch.bfloat16).to(dev)
        y = torch.empty((1, N), dtype=torch.float32, device=dev)
        layers.append((name, K, N, copies, x, y))
    torch.cuda.synchronize()

    ws = {}
    for name, K, N, copies, x, y in layers:
        nbytes = int(nv.lib().nvfp4_linear_workspace(1, K, N, nv.MODE_W4A16))
        ws[name] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev) if nbytes else None

    def call(j, i):
        name, K, N, copies, x, y = layers[j]
        c, s, g = copies[i % 2]
        nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A16, ws=ws[name])

    def step(i):
        for j in range(len(layers)):
            call(j, i)

    step_bytes = sum(decode_bytes(1, K, N) for _, K, N, *_ in layers)

    # eager warm-up (kernel attributes, cluster-size choice), then capture:
    # one graph per weight copy for the whole step, one per (shape, copy)
    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    step_graphs, shape_graphs = [], []
    with torch.cuda.stream(side):
        for i in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                step(i)
            step_graphs.append(g)
        # one linear alone: each graph launches it once per weight copy, with
        # enough copies that a replay streams > 3x the L2 (126 MB)
        for j, (name, K, N, copies, x, y) in enumerate(layers):
            nc = max(2, -(-3 * L2_BYTES // decode_bytes(1, K, N)))
            many = [copies[0]] + [tuple(t.clone() for t in copies[0]) for _ in range(nc - 1)]

            def chain(j=j, name=name, many=many, x=x, y=y):
                for c, s_, g_ in many:
                    nv.nvfp4_linear(x, c, s_, g_, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A16, ws=ws[name])

            chain()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                chain()
            shape_graphs.append((g, nc, many))
    stream.wait_stream(side)
    torch.cuda.synchronize()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        time.sleep(0.5)
        for i in range(args.warmup):
            step_graphs[i % 2].replay()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step_graphs[i % 2].replay()
        t1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    ms_per_step = ms / args.steps
    value = whole_job_gbs(world, step_bytes, ms_per_step)

    # per-shape device time: each linear alone, replayed from its graph
    reps = max(200, min(2000, args.steps))
    per_shape = {}
    for j, (name, K, N, *_) in enumerate(layers):
        g, nc, _ = shape_graphs[j]
        for i in range(4):
            g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps_j = max(20, reps // nc)
        a.record(stream)
        for i in range(reps_j):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        m = a.elapsed_time(b) / (reps_j * nc)
        per_shape[name] = {"us": round(m * 1e3, 2), "GB/s": round(decode_bytes(1, K, N) / (m * 1e-3) / 1e9, 1),
                           "weight_copies": nc}
    del shape_graphs

    # roofline of the dominant kernel: the W4A16 decode kernel is every launch of
    # the step, so bytes per launch / mean launch time = step bytes / step time
    peak, peak_kind = load_peaks()
    achieved = step_bytes / (ms_per_step * 1e-3) / 1e9
    traffic = kernel_traffic("gemv_tma.cu", "gemv_tma_decode")

    # end to end through the C ABI: every step copies the four inputs from one
    # pinned host buffer, calls nvfp4_linear four times (arguments marshalled
    # once, as a C caller holds them) and copies the four outputs back to one
    # pinned host buffer
    import ctypes
    ks, ns = [K for _, K, *_ in layers], [N for _, K, N, *_ in layers]
    xh = torch.empty(sum(ks), dtype=torch.bfloat16).pin_memory()
    xh.copy_(torch.cat([x.reshape(-1).cpu() for *_, x, y in layers]))
    yh = torch.empty(sum(ns), dtype=torch.float32).pin_memory()
    xd = torch.empty(sum(ks), dtype=torch.bfloat16, device=dev)
    yd = torch.empty(sum(ns), dtype=torch.float32, device=dev)
    h2d, d2h = xh.numel() * xh.element_size(), yh.numel() * yh.element_size()
    cstream = ctypes.c_void_p(stream.cuda_stream)
    abi_args = [[], []]
    xo, yo = 0, 0
    for (name, K, N, copies, x, y) in layers:
        wsp = ws[name]
        for i in range(2):
            c, s_, g_ = copies[i]
            abi_args[i].append((ctypes.c_void_p(xd[xo:].data_ptr()), nv.DTYPE_BF16, 1, K, ctypes.c_void_p(c.data_ptr()),
                                ctypes.c_void_p(s_.data_ptr()), nv.SF_TILED, ctypes.c_void_p(g_.data_ptr()), N,
                                ctypes.c_void_p(yd[yo:].data_ptr()), nv.DTYPE_F32, nv.MODE_W4A16,
                                None if wsp is None else ctypes.c_void_p(wsp.data_ptr()),
                                0 if wsp is None else wsp.numel(), cstream))
        xo, yo = xo + K, yo + N
    linear = nv.lib().nvfp4_linear

    def e2e_step(i):
        xd.copy_(xh, non_blocking=True)
        for a in abi_args[i % 2]:
            if linear(*a) != 0:
                raise RuntimeError("nvfp4_linear failed in the end-to-end step")
        yh.copy_(yd, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    e2e = whole_job_gbs(world, step_bytes, e_ms / args.steps)

    extra = {"decode_m1_per_shape": per_shape}
    if not args.quick:
        extra["decode_sweep"] = decode_sweep(nv, torch, dev, layers)
        extra["verify_widths"] = verify_section(nv, torch, dev, layers)
        extra["prefill"] = prefill_section(nv, torch, dev, layers, M=2048)
        extra["prefill_m512"] = prefill_section(nv, torch, dev, layers, M=512)
        extra["prefill_m8192"] = prefill_section(nv, torch, dev, layers, M=8192, reps=10)
        extra["quantize"] = quantize_section(nv, torch, dev)
        extra["moe_layer"] = moe_section(nv, torch, dev)
        try:
            extra["decode_stack"] = stack_section(nv, torch, dev, peak)
        except Exception as exc:  # reported in the line; the headline above stands
            extra["decode_stack"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 weights x bf16 activations, fp32 accumulate",
        "data": "synthetic: weights N(0,0.02) fp32 quantized on device, activations N(0,1) bf16",
        "config": workload_config(world),
        "timing": "CUDA-graph replay of the step (4 linears), events on the launching stream",
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                     "per": "decode step (4 launches, one per shape): algorithmic bytes / step time on this GPU",
                     "kernel": "gemv_tma_kernel (the only launch of each linear), CUDA events around the step graphs"},
        "e2e": {"value": round(e2e, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 4 * args.steps,
        "clocks": clk.summary(),
        **extra,
    }
    return line


def decode_sweep(nv, torch, dev, layers, reps=20):
    """Per-launch GB/s for each shape and M: a CUDA graph launches the linear once
    per weight copy, with enough copies that a replay streams > 3x the L2."""
    from bit_linear_moe_b200 import synth
    out = {}
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=dev)
    for name, K, N, copies, _, _ in layers:
        seed = dict((s[0], s[3]) for s in SHAPES)[name]
        nc = max(2, -(-3 * L2_BYTES // decode_bytes(1, K, N)))
        many = [copies[0]] + [tuple(t.clone() for t in copies[0]) for _ in range(nc - 1)]
        row = {}
        for M in synth.DECODE_M:
            x = torch.from_numpy(synth.decode_x(seed, M, K)).to(torch.bfloat16).to(dev)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            nbytes = int(nv.lib().nvfp4_linear_workspace(M, K, N, nv.MODE_W4A16))
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None

            def chain():
                for c, s, g in many:
                    nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A16, ws=ws)

            chain()
            torch.cuda.synchronize()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=side):
                    chain()
            stream.wait_stream(side)
            for i in range(3):
                gr.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(reps):
                gr.replay()
            b.record(stream)
            torch.cuda.synchronize()
            m = a.elapsed_time(b) / (reps * nc)
            row[str(M)] = round(decode_bytes(M, K, N) / (m * 1e-3) / 1e9, 1)
            del gr
        out[name] = row
        del many
    return out


def verify_section(nv, torch, dev, layers, reps=40):
    """Speculative-verify widths (one target-model pass over 1 + draft tokens):
    the decode step of the four linears at M in {8, 16, 64}, one CUDA graph
    per width (and per weight copy), W4A16; for 64 tokens also AUTO, which
    picks W4A4 above 32 tokens.  GB/s counts the step's algorithmic bytes."""
    from bit_linear_moe_b200 import synth
    out = {}
    seeds = dict((s[0], s[3]) for s in SHAPES)
    for M in synth.VERIFY_M:
        modes = [("W4A16", nv.MODE_W4A16)] + ([("AUTO", nv.MODE_AUTO)] if M > 32 else [])
        for mname, mode in modes:
            xs = [torch.from_numpy(synth.decode_x(seeds[name], M, K)).to(torch.bfloat16).to(dev)
                  for name, K, N, *_ in layers]
            ys = [torch.empty((M, N), dtype=torch.float32, device=dev) for _, K, N, *_ in layers]
            wss = [torch.empty(max(16, int(nv.lib().nvfp4_linear_workspace(M, K, N, mode))), dtype=torch.uint8,
                               device=dev) for _, K, N, *_ in layers]

            def step(i, xs=xs, ys=ys, wss=wss, mode=mode):
                for j, (name, K, N, copies, _, _) in enumerate(layers):
                    c, s_, g = copies[i % 2]
                    nv.nvfp4_linear(xs[j], c, s_, g, w_sf_layout=nv.SF_TILED, y=ys[j], mode=mode, ws=wss[j])

            t = _time_graphs(torch, _capture(torch, dev, step), reps)
            nbytes = sum(decode_bytes(M, K, N) for _, K, N, *_ in layers)
            out[f"M{M}_{mname}"] = {"us_per_step": round(t * 1e3, 2), "GB/s": round(nbytes / (t * 1e-3) / 1e9, 1),
                                    "tokens_per_s_per_layer_step": round(M / (t * 1e-3), 1)}
    return out


def _time_graphs(torch, graphs, reps):
    stream = torch.cuda.current_stream()
    for i in range(3):
        graphs[i % len(graphs)].replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(reps):
        graphs[i % len(graphs)].replay()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def _capture(torch, dev, fn_per_copy):
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=dev)
    for i in range(2):
        fn_per_copy(i)
    torch.cuda.synchronize()
    side.wait_stream(stream)
    graphs = []
    with torch.cuda.stream(side):
        for i in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                fn_per_copy(i)
            graphs.append(g)
    stream.wait_stream(side)
    return graphs


def prefill_section(nv, torch, dev, layers, M=2048, reps=30, library_ceiling=True):
    """W4A4 prefill at M tokens on the four shapes: TFLOP/s = 2 M N K / time of
      gemm        the GEMM alone (activations already NVFP4),
      with_quant  nvfp4_linear(W4A4): amax pass + quantize pass + GEMM,
      rms_*       a producer that renormalises the previous output first:
                  unfused  nvfp4_rms_norm -> nvfp4_linear(W4A4)
                  fused    nvfp4_rms_norm_quant -> nvfp4_linear_w4a4q,
      library     torch's scaled_mm on the same NVFP4 operands (cuBLASLt, block
                  scales 1x16 in the same swizzled layout): the measured FP4
                  ceiling of this GPU."""
    from bit_linear_moe_b200 import synth
    import torch.nn.functional as F
    seeds = dict((s[0], s[3]) for s in SHAPES)
    out = {"M": M, "shapes": {}}
    tot = {"flop": 0.0, "gemm": 0.0, "with_quant": 0.0, "rms_unfused": 0.0, "rms_fused": 0.0, "library": 0.0}
    for name, K, N, copies, _, _ in layers:
        x = torch.from_numpy(synth.prefill_x(seeds[name], M, K)[0]).to(torch.bfloat16).to(dev)
        xc, xs, xg = nv.nvfp4_quantize(x, sf_layout=nv.SF_TILED)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(int(nv.lib().nvfp4_linear_workspace(M, K, N, nv.MODE_W4A4)), dtype=torch.uint8, device=dev)
        xr = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        rq_ws = torch.empty(max(16, int(nv.lib().nvfp4_rms_norm_quant_workspace(M))), dtype=torch.uint8, device=dev)
        rc = torch.empty_like(xc)
        rs = torch.empty_like(xs)
        rg = torch.empty_like(xg)

        def gemm(i):
            c, s, g = copies[i]
            nv.nvfp4_linear_w4a4q(xc, xs, xg, c, s, g, y=y)

        def e2e(i):
            c, s, g = copies[i]
            nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A4, ws=ws)

        def rms_unfused(i):
            c, s, g = copies[i]
            nv.nvfp4_rms_norm(x, y=xr)
            nv.nvfp4_linear(xr, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A4, ws=ws)

        def rms_fused(i):
            c, s, g = copies[i]
            lib = nv.lib()
            nv._check(lib.nvfp4_rms_norm_quant(nv._ptr(x), nv.DTYPE_BF16, M, K, K, nv.SF_TILED, nv._ptr(rc),
                                               nv._ptr(rs), nv._ptr(rg), nv._ptr(rq_ws), rq_ws.numel(), nv._stream()),
                      "nvfp4_rms_norm_quant")
            nv.nvfp4_linear_w4a4q(rc, rs, rg, c, s, g, y=y)

        flop = 2.0 * M * N * K
        row = {}
        for key, fn in (("gemm", gemm), ("with_quant", e2e), ("rms_unfused", rms_unfused), ("rms_fused", rms_fused)):
            t = _time_graphs(torch, _capture(torch, dev, fn), reps)
            row[key + "_us"] = round(t * 1e3, 1)
            row[key + "_TFLOPs"] = round(flop / (t * 1e-3) / 1e12, 1)
            tot[key] += t
        if library_ceiling:
            try:
                a4, sa = xc.view(torch.float4_e2m1fn_x2), xs.view(torch.float8_e4m3fn)

                def lib_mm(i):
                    c, s, g = copies[i]
                    F.scaled_mm(a4, c.view(torch.float4_e2m1fn_x2).t(), [sa], [F.ScalingType.BlockWise1x16],
                                [s.view(torch.float8_e4m3fn)], [F.ScalingType.BlockWise1x16],
                                swizzle_a=[F.SwizzleType.SWIZZLE_32_4_4], swizzle_b=[F.SwizzleType.SWIZZLE_32_4_4],
                                output_dtype=torch.bfloat16)

                t = _time_graphs(torch, _capture(torch, dev, lib_mm), reps)
                row["library_us"] = round(t * 1e3, 1)
                row["library_TFLOPs"] = round(flop / (t * 1e-3) / 1e12, 1)
                tot["library"] += t
            except Exception as exc:  # reported, not fatal: the ceiling is context
                row["library"] = f"unavailable: {type(exc).__name__}: {str(exc)[:120]}"
                tot["library"] = float("nan")
        out["shapes"][name] = row
        tot["flop"] += flop
    for key in ("gemm", "with_quant", "rms_unfused", "rms_fused", "library"):
        if tot[key] == tot[key] and tot[key] > 0:
            out[key + "_TFLOPs"] = round(tot["flop"] / (tot[key] * 1e-3) / 1e12, 1)
    out["peak_nominal_dense_nvfp4_TFLOPs"] = 9000.0
    out["frac_of_nominal"] = round(out["gemm_TFLOPs"] / 9000.0, 4)
    if out.get("library_TFLOPs"):
        out["frac_of_library"] = round(out["gemm_TFLOPs"] / out["library_TFLOPs"], 4)
    return out


MOE_EXPERT_BYTES = 1024 * 2048 // 2 + 1024 * 2048 // 16 + 2048 * 512 // 2 + 2048 * 512 // 16  # 1,769,472


def moe_section(nv, torch, dev, reps=30):
    """One mixture-of-experts layer (512 experts, hidden 2048, expert width 512,
    top-10): route, gather + gate/up + SwiGLU, down + weighted combine.
    GB/s = (touched experts x 1,769,472 B + T x 2048 x (2 + 4) B for h in and
    y out) / time; W4A16 at T = 1, 32 and W4A4 at T = 4096, uniform routing
    and a Zipf(1.1) popularity bias.  Expert weights 0.02 N(0, 1) drawn on the
    device from a seeded generator and quantized per expert matrix."""
    from bit_linear_moe_b200 import synth
    E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_K
    gen = torch.Generator(device=dev)
    gen.manual_seed(10)

    def stack(n, kk):
        cs, ss, gs = [], [], []
        for _ in range(E):
            w = 0.02 * torch.randn((n, kk), generator=gen, device=dev)
            c, sc, g = nv.nvfp4_quantize(w, sf_layout=nv.SF_TILED)
            cs.append(c)
            ss.append(sc)
            gs.append(g)
        return torch.stack(cs), torch.stack(ss).reshape(-1), torch.cat(gs)

    gu = stack(2 * I, H)
    dn = stack(H, I)
    wr = (0.02 * torch.randn((E, H), generator=gen, device=dev)).to(torch.bfloat16)
    zipf = torch.from_numpy(synth.moe_zipf_bias()).to(dev)
    out = {"experts": E, "hidden": H, "expert_width": I, "top_k": k, "bytes_per_touched_expert": MOE_EXPERT_BYTES,
           "runs": {}}
    for T, mode, nbatch in ((1, nv.MODE_W4A16, 16), (32, nv.MODE_W4A16, 4), (4096, nv.MODE_W4A4, 2)):
        R = T * k
        ws1 = torch.empty(max(16, int(nv.lib().moe_grouped_linear_workspace(R, H, 2 * I, E, k, nv.EPI_SWIGLU, mode))),
                          dtype=torch.uint8, device=dev)
        ws2 = torch.empty(max(16, int(nv.lib().moe_grouped_linear_workspace(R, I, H, E, k, nv.EPI_COMBINE, mode))),
                          dtype=torch.uint8, device=dev)
        for bias_name, bias in (("uniform", None), ("zipf", zipf)):
            hs = [torch.randn((T, H), generator=gen, device=dev).to(torch.bfloat16) for _ in range(nbatch)]
            a = torch.empty((R, I), dtype=torch.bfloat16, device=dev)
            y = torch.empty((T, H), dtype=torch.float32, device=dev)
            touched = []

            def layer(i):
                r = nv.moe_route_topk(hs[i], wr, k, logit_bias=bias)
                nv.moe_grouped_linear(hs[i], r["expert_offsets"], gu[0], gu[1], gu[2], R, perm_tok=r["perm_tok"],
                                      gather=True, w_sf_layout=nv.SF_TILED, epilogue=nv.EPI_SWIGLU, y=a,
                                      mode=mode, ws=ws1)
                nv.moe_grouped_linear(a, r["expert_offsets"], dn[0], dn[1], dn[2], R, gather=False,
                                      w_sf_layout=nv.SF_TILED, epilogue=nv.EPI_COMBINE, topk_w=r["topk_w"],
                                      row_of=r["row_of"], k=k, y=y, mode=mode, ws=ws2)
                return r

            for i in range(nbatch):
                r = layer(i)
                touched.append(int((torch.diff(r["expert_offsets"]) > 0).sum().item()))
            torch.cuda.synchronize()
            stream = torch.cuda.current_stream()
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            graphs = []
            with torch.cuda.stream(side):
                for i in range(nbatch):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=side):
                        layer(i)
                    graphs.append(g)
            stream.wait_stream(side)
            t = _time_graphs(torch, graphs, max(reps, 2 * nbatch))
            nbytes = sum(touched) / nbatch * MOE_EXPERT_BYTES + T * H * 6
            flop = 2.0 * R * (H * 2 * I + I * H)
            key = f"T{T}_{bias_name}"
            out["runs"][key] = {"mode": "W4A16" if mode == nv.MODE_W4A16 else "W4A4", "us": round(t * 1e3, 2),
                                "touched_experts_mean": round(sum(touched) / nbatch, 1),
                                "GB/s": round(nbytes / (t * 1e-3) / 1e9, 1),
                                "TFLOPs": round(flop / (t * 1e-3) / 1e12, 2)}
    # the fused decode-time layer (router ... combine in one call) at T = 1, 32
    for T, nbatch in ((1, 16), (32, 4)):
        wsd = torch.empty(max(16, int(nv.lib().moe_layer_decode_workspace(T, H, I, E, k))), dtype=torch.uint8,
                          device=dev)
        for bias_name, bias in (("uniform", None), ("zipf", zipf)):
            hs = [torch.randn((T, H), generator=gen, device=dev).to(torch.bfloat16) for _ in range(nbatch)]
            y = torch.empty((T, H), dtype=torch.float32, device=dev)
            touched = []
            for i in range(nbatch):
                _, ex = nv.moe_layer_decode(hs[i], wr, k, gu, dn, logit_bias=bias, y=y, want_routing=True, ws=wsd)
                touched.append(int(torch.unique(ex["topk_idx"]).numel()))

            def layer(i, bias=bias, hs=hs, y=y):
                nv.moe_layer_decode(hs[i], wr, k, gu, dn, logit_bias=bias, y=y, ws=wsd)

            torch.cuda.synchronize()
            stream = torch.cuda.current_stream()
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            graphs = []
            with torch.cuda.stream(side):
                for i in range(nbatch):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=side):
                        layer(i)
                    graphs.append(g)
            stream.wait_stream(side)
            t = _time_graphs(torch, graphs, max(reps, 2 * nbatch))
            nbytes = sum(touched) / nbatch * MOE_EXPERT_BYTES + T * H * 6
            out["runs"][f"T{T}_{bias_name}_fused"] = {"mode": "W4A16 fused layer (moe_layer_decode)",
                                                     "us": round(t * 1e3, 2),
                                                     "touched_experts_mean": round(sum(touched) / nbatch, 1),
                                                     "GB/s": round(nbytes / (t * 1e-3) / 1e9, 1)}
    del gu, dn
    return out


def stack_section(nv, torch, dev, peak_gbs, reps=10):
    """The dense decode stack: 64 layers of the four 27B-shaped linears (12.46
    GB of NVFP4 weights resident), each layer chained through the library's
    glue kernels with attention left out:
        q = QKV(x); o = O(rms(q[:, :5120])); g = GU(rms(o));
        h = silu(g[:, :17408]) * g[:, 17408:]; x' = rms(Down(h))
    One step is the whole stack for M tokens, captured once as a CUDA graph and
    replayed; GB/s = (weight bytes + activation bytes read by the linears) /
    step time.  Weights 0.02 N(0, 1) drawn on the device (seed 1000 + 4 i + j)
    and quantized there; x0 N(0, 1) renormalised."""
    L = 64
    layers = []
    for i in range(L):
        mats = {}
        for j, (name, K, N, _) in enumerate(SHAPES):
            gen = torch.Generator(device=dev)
            gen.manual_seed(1000 + 4 * i + j)
            w = 0.02 * torch.randn((N, K), generator=gen, device=dev)
            mats[name] = nv.nvfp4_quantize(w, sf_layout=nv.SF_TILED)
            del w
        layers.append(mats)
    torch.cuda.synchronize()
    kq, nq = SHAPES[0][1], SHAPES[0][2]
    ng = SHAPES[2][2]
    out = {"layers": L, "weight_bytes": L * sum(N * K // 2 + N * K // 16 for _, K, N, _ in SHAPES),
           "timing": "CUDA-graph replay of the 64-layer step, events on the launching stream", "runs": {}}
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=dev)
    for M in (1, 8, 32):
        gx = torch.Generator(device=dev)
        gx.manual_seed(999)
        x = nv.nvfp4_rms_norm(torch.randn((M, kq), generator=gx, device=dev))
        bufs = {name: torch.empty((M, N), dtype=torch.float32, device=dev) for name, _, N, _ in SHAPES}
        ws = {name: torch.empty(max(16, int(nv.lib().nvfp4_linear_workspace(M, K, N, nv.MODE_W4A16))),
                                dtype=torch.uint8, device=dev) for name, K, N, _ in SHAPES}
        o_in = torch.empty((M, kq), dtype=torch.bfloat16, device=dev)
        gu_in = torch.empty((M, kq), dtype=torch.bfloat16, device=dev)
        h = torch.empty((M, ng // 2), dtype=torch.bfloat16, device=dev)
        x_next = torch.empty((M, kq), dtype=torch.bfloat16, device=dev)

        def lin(xin, li, name):
            c, s, g = layers[li][name]
            return nv.nvfp4_linear(xin, c, s, g, w_sf_layout=nv.SF_TILED, y=bufs[name], mode=nv.MODE_W4A16,
                                   ws=ws[name])

        def step():
            cur = x
            for li in range(L):
                q = lin(cur, li, "qkv")
                nv.nvfp4_rms_norm(q, cols=kq, y=o_in)
                o = lin(o_in, li, "o_proj")
                nv.nvfp4_rms_norm(o, y=gu_in)
                g = lin(gu_in, li, "gate_up")
                nv.nvfp4_silu_mul(g, h=h)
                d = lin(h, li, "down")
                nv.nvfp4_rms_norm(d, y=x_next)
                cur = x_next

        step()
        torch.cuda.synchronize()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=side):
                step()
        stream.wait_stream(side)
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            gr.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        nbytes = L * sum(decode_bytes(M, K, N) for _, K, N, _ in SHAPES)
        gbs = nbytes / (ms * 1e-3) / 1e9
        x_out = x_next.float()
        out["runs"][f"M{M}"] = {"ms_per_step": round(ms, 4), "us_per_layer": round(ms * 1e3 / L, 2),
                                "GB/s": round(gbs, 1), "frac_of_peak": round(gbs / peak_gbs, 4),
                                "final_rms": round(float(x_out.pow(2).mean().sqrt()), 4),
                                "finite": bool(torch.isfinite(x_out).all())}
        del gr
    return out


def quantize_section(nv, torch, dev, reps=30):
    """Activation quantize (two passes: amax, then scales and codes) of bf16
    [M, 5120]: GB/s = (2 M K + 2 M K + 0.5625 M K) / time."""
    out = {}
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    K = 5120
    for M in (2048, 8192):
        xs = [torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16) for _ in range(2)]
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(int(nv.nvfp4_scales_bytes(M, K, nv.SF_TILED)), dtype=torch.uint8, device=dev)
        gs = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(max(16, int(nv.lib().nvfp4_quantize_workspace(M, K))), dtype=torch.uint8, device=dev)

        def q(i):
            nv.nvfp4_quantize(xs[i], sf_layout=nv.SF_TILED, codes=codes, scales=scales, gs_out=gs, ws=ws)

        t = _time_graphs(torch, _capture(torch, dev, q), reps)
        out[f"M{M}_K{K}"] = {"us": round(t * 1e3, 2), "GB/s": round(4.5625 * M * K / (t * 1e-3) / 1e9, 1)}
    return out


# ------------------------------------------------------------ profile cases ----

CASES = ("decode_m1", "skinny_m4", "prefill_m2048", "quantize_m2048", "moe_t1", "moe_t32", "moe_t4096",
         "moe_fused_t1", "moe_fused_t32", "stack_glue_m1")


def profile_case(args):
    """One small workload, launched eagerly ``--steps`` times, for a profiler to
    capture a few launches of one kernel (a few GB on the device at most)."""
    import torch
    import bit_linear_moe_b200 as nv
    from bit_linear_moe_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    case = args.case
    shapes = {name: (K, N) for name, K, N, _ in SHAPES}

    def qw(K, N):
        return nv.nvfp4_quantize(0.02 * torch.randn((N, K), generator=gen, device=dev), sf_layout=nv.SF_TILED)

    if case in ("decode_m1", "skinny_m4", "stack_glue_m1"):
        M = 4 if case == "skinny_m4" else 1
        ws_ = {name: qw(K, N) for name, (K, N) in shapes.items()}
        xs = {name: torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16) for name, (K, N) in shapes.items()}

        def run():
            for name, (K, N) in shapes.items():
                c, s_, g = ws_[name]
                y = nv.nvfp4_linear(xs[name], c, s_, g, w_sf_layout=nv.SF_TILED, mode=nv.MODE_W4A16)
                if case == "stack_glue_m1":
                    if name == "gate_up":
                        nv.nvfp4_silu_mul(y)
                    else:
                        nv.nvfp4_rms_norm(y, cols=min(y.shape[1], 5120))
    elif case == "prefill_m2048":
        K, N = shapes["qkv"]
        c, s_, g = qw(K, N)
        x = torch.randn((2048, K), generator=gen, device=dev).to(torch.bfloat16)
        xc, xs_, xg = nv.nvfp4_quantize(x, sf_layout=nv.SF_TILED)

        def run():
            nv.nvfp4_linear_w4a4q(xc, xs_, xg, c, s_, g)
    elif case == "quantize_m2048":
        x = torch.randn((2048, 5120), generator=gen, device=dev).to(torch.bfloat16)

        def run():
            nv.nvfp4_quantize(x, sf_layout=nv.SF_TILED)
    else:
        E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_K
        T = int(case.rsplit("_t", 1)[1])
        mode = nv.MODE_W4A4 if T > 32 else nv.MODE_W4A16

        def stack(n, kk):
            sb = nv.nvfp4_scales_bytes(n, kk, nv.SF_TILED)
            codes = torch.empty((E, n, kk // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty(E * sb, dtype=torch.uint8, device=dev)
            gs = torch.empty(E, dtype=torch.float32, device=dev)
            for e in range(E):
                nv.nvfp4_quantize(0.02 * torch.randn((n, kk), generator=gen, device=dev), sf_layout=nv.SF_TILED,
                                  codes=codes[e], scales=scales[e * sb:(e + 1) * sb], gs_out=gs[e:e + 1])
            return codes, scales, gs

        gu, dn = stack(2 * I, H), stack(H, I)
        wr = (0.02 * torch.randn((E, H), generator=gen, device=dev)).to(torch.bfloat16)
        h = torch.randn((T, H), generator=gen, device=dev).to(torch.bfloat16)
        R = T * k

        def run_fused():
            nv.moe_layer_decode(h, wr, k, gu, dn)

        def run():
            if case.startswith("moe_fused"):
                return run_fused()
            r = nv.moe_route_topk(h, wr, k)
            a = nv.moe_grouped_linear(h, r["expert_offsets"], *gu, R, perm_tok=r["perm_tok"], gather=True,
                                      w_sf_layout=nv.SF_TILED, epilogue=nv.EPI_SWIGLU, y_dtype=torch.bfloat16,
                                      mode=mode)
            nv.moe_grouped_linear(a, r["expert_offsets"], *dn, R, gather=False, w_sf_layout=nv.SF_TILED,
                                  epilogue=nv.EPI_COMBINE, topk_w=r["topk_w"], row_of=r["row_of"], k=k,
                                  mode=mode)
    for _ in range(args.steps):
        run()
    torch.cuda.synchronize()
    assert nv.nvfp4_read_device_status() == nv.OK
    print(json.dumps({"case": case, "steps": args.steps, "ok": True}))


# --------------------------------------------------------------- reference ----

_ORACLE_W = {}


def oracle_weights(row_frac: int = 1):
    """The four linears' weights quantized by the oracle (every row_frac-th
    row), with their M = 1 inputs: [(K, N, (codes, scales, gs), x)]."""
    import oracle
    from bit_linear_moe_b200 import synth
    if row_frac not in _ORACLE_W:
        qs = []
        for name, K, N, seed in SHAPES:
            c, s_, g = oracle.quantize(synth.dense_weight(seed, K, N)[::row_frac])
            qs.append((K, c.shape[0], (c, s_, g), synth.decode_x(seed, 1, K)))
        _ORACLE_W[row_frac] = qs
    return _ORACLE_W[row_frac]


def _rate(fn, units: float, seconds: float):
    """(units per second, seconds, passes) of fn repeated for at least ``seconds``."""
    t = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t
        if dt >= seconds:
            return units * n / dt, dt, n


def oracle_decode_sample(min_seconds: float = 10.0, row_frac: int = 1):
    """Time the oracle's W4A16 linear on the same four shapes at M = 1 (weights
    quantized by the oracle outside the timed region), repeating the four
    linears until ``min_seconds`` have passed.  ``row_frac`` > 1 keeps every
    row_frac-th weight row (a bounded sample).  Returns (GB/s, seconds, passes, threads)."""
    import oracle
    qs = oracle_weights(row_frac)

    def step():
        for K, N, q, x in qs:
            oracle.linear_w4a16(x, *q)

    gbs, dt, passes = _rate(step, sum(decode_bytes(1, K, N) for K, N, _, _ in qs) / 1e9, min_seconds)
    return gbs, dt, passes, oracle.num_threads()


def oracle_single_thread(seconds: float = 4.0, row_frac: int = 16):
    """The headline sample on one host thread (a child process with
    OMP_NUM_THREADS=1): {value, unit, cores, sample}."""
    code = (f"import json, bench; g, dt, n, th = bench.oracle_decode_sample({seconds}, {row_frac}); "
            "print(json.dumps([g, dt, n, th]))")
    env = dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    if r.returncode != 0:
        return {"error": (r.stderr or r.stdout)[-300:]}
    g, dt, n, th = json.loads(r.stdout.strip().splitlines()[-1])
    return {"value": round(g, 3), "unit": "GB/s", "cores": th,
            "sample": f"the four linears at M=1 over every {row_frac}th weight row, {n} passes in {dt:.1f} s"}


def oracle_per_config(seconds: float = 2.0) -> dict:
    """The oracle, as it stands, on a bounded sample of each workload the
    parity suite covers (all host threads): {name: {value, unit, sample}}."""
    import oracle
    from oracle import moe as omoe
    from oracle import stack as ostack
    from bit_linear_moe_b200 import synth
    out = {}

    w, x = synth.single(0)
    q = oracle.quantize(w)
    g, dt, n = _rate(lambda: oracle.linear_w4a16(x, *q), decode_bytes(1, 2048, 2048) / 1e9, seconds)
    out["single_linear_m1_k2048_n2048"] = {"value": round(g, 3), "unit": "GB/s",
                                           "sample": f"the whole linear, {n} passes in {dt:.1f} s"}

    qs = oracle_weights(16)
    xs = [synth.decode_x(i + 1, 32, K) for i, (K, N, _, _) in enumerate(qs)]

    def dec32():
        for (K, N, qq, _), xx in zip(qs, xs):
            oracle.linear_w4a16(xx, *qq)

    g, dt, n = _rate(dec32, sum(decode_bytes(32, K, N) for K, N, _, _ in qs) / 1e9, seconds)
    out["dense27b_decode_m32"] = {"value": round(g, 3), "unit": "GB/s",
                                  "sample": f"M=32, every 16th weight row of the four linears, {n} passes in {dt:.1f} s"}

    # prefill: 8 of the 2048 rows (quantized with the whole batch's gs) x all weight rows
    pre = []
    for K, N, qq, _ in oracle_weights(1):
        seed = [sd for _, k_, n_, sd in SHAPES if k_ == K and n_ == N][0]
        xa, _ = synth.prefill_x(seed, 2048, K)
        xc, xsc, xg = oracle.quantize(xa)
        rows = np.arange(0, 2048, 256)
        pre.append((K, N, (np.ascontiguousarray(xc[rows]), np.ascontiguousarray(xsc[rows]), xg), qq))

    def prefill():
        for K, N, xq, qq in pre:
            oracle.linear_w4a4(xq, qq)

    g, dt, n = _rate(prefill, sum(2 * 8 * N * K for K, N, _, _ in pre) / 1e12, seconds)
    out["prefill_w4a4_m2048"] = {"value": round(g, 5), "unit": "TFLOP/s",
                                 "sample": f"8 of the 2048 rows x the four full weights, {n} passes in {dt:.1f} s"}

    # MoE layer, T = 1: router, top-10, the chosen experts' gate/up, SwiGLU, down, combine
    E, H, I, k = synth.MOE_E, synth.MOE_H, synth.MOE_I, synth.MOE_K
    wr = synth.moe_router()
    h = synth.moe_hidden(1)
    idx, _ = omoe.topk(omoe.router_logits(h, wr), k)
    chosen = [int(e) for e in idx[0]]
    gq, dq = [], []
    for e in chosen:
        wgu, wd = synth.moe_expert(e)
        gq.append(oracle.quantize(wgu))
        dq.append(oracle.quantize(wd))
    stk = lambda qq: (np.stack([a[0] for a in qq]), np.stack([a[1] for a in qq]),
                      np.array([a[2] for a in qq], np.float32))
    gu_w, dn_w = stk(gq), stk(dq)
    local = {e: j for j, e in enumerate(chosen)}

    def layer():
        logits = omoe.router_logits(h, wr)
        ix, wt = omoe.topk(logits, k)
        il = np.vectorize(local.get)(ix).astype(np.int32)
        offsets, perm_tok, perm_slot, row_of = omoe.permute(il, k)
        gu, _ = omoe.grouped_linear_w4a16(h, offsets, perm_tok, *gu_w, gather=True)
        a = ostack.bf16_round(omoe.swiglu(gu))
        d, _ = omoe.grouped_linear_w4a16(a, offsets, perm_tok, *dn_w, gather=False)
        omoe.combine(d, wt, row_of)

    touched = k * (2 * I * H + H * I) * 9 // 16
    g, dt, n = _rate(layer, touched / 1e9, seconds)
    out["moe_layer_t1"] = {"value": round(g, 3), "unit": "GB/s of touched expert weights",
                           "sample": f"one token, all {E} router rows, its {k} experts, {n} passes in {dt:.1f} s"}
    out["threads"] = oracle.num_threads()
    return out


def run_reference(args):
    """The oracle as the reference arm on the headline workload: each step is
    the four linears at M = 1.  Full weights when the whole run fits in about
    two minutes of host time; otherwise every n-th weight row, and the line's
    config says so."""
    import oracle
    qs = oracle_weights(1)

    def step(qq):
        for K, N, q, x in qq:
            oracle.linear_w4a16(x, *q)

    t = time.perf_counter()
    step(qs)
    t1 = time.perf_counter() - t
    row_frac = max(1, int(np.ceil(t1 * (args.steps + args.warmup) / 120.0)))
    if row_frac > 1:
        qs = oracle_weights(row_frac)
    step_bytes = sum(decode_bytes(1, K, N) for K, N, _, _ in qs)
    for _ in range(args.warmup):
        step(qs)
    t = time.perf_counter()
    for _ in range(args.steps):
        step(qs)
    dt = time.perf_counter() - t
    gbs = step_bytes * args.steps / dt / 1e9
    config = workload_config(args.gpus)
    if row_frac > 1:
        sample = f"each step: the four linears at M=1 over every {row_frac}th weight row"
        config["sample"] = sample
    else:
        sample = "each step: the whole workload (the four linears at M=1, all weight rows)"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 3), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp64 accumulate (CPU oracle)",
        "data": "synthetic, same generator as the native arm",
        "config": config,
        "timing": "host wall clock around the timed steps (CPU oracle)",
        "cpu_baseline": {"value": round(gbs, 3), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--quick", action="store_true", help="headline only (no sweeps, no CPU baseline)")
    ap.add_argument("--case", choices=CASES, default=None,
                    help="run one small workload eagerly --steps times (for profiler captures) and exit")
    args = ap.parse_args()
    if args.case:
        profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return

    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    line = run_native(args, rank, world, dist)
    if rank == 0 and world == 1 and not args.quick:
        gbs, dt, passes, threads = oracle_decode_sample(min_seconds=10.0)
        line["cpu_baseline"] = {"value": round(gbs, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"the four linears at M=1, full weights, {passes} passes in {dt:.1f} s",
                                "single_thread": oracle_single_thread(),
                                "per_config": oracle_per_config()}
    if rank == 0:
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
