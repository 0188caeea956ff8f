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
region): the decode sweep M in {1, 2, 4, 8, 16, 32} per shape, and whatever
other sections the library supports (prefill W4A4 TFLOP/s, MoE).

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


def decode_bytes(M, K, N):
    return N * K // 2 + N * K // 16 + M * K * 2 + 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic(kernel_src: str, name: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (matched by hash); else None."""
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
        return float(vals["dram_bytes_per_launch"])
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

    def step(i, events=None):
        for j, (name, K, N, copies, x, y) in enumerate(layers):
            c, s, g = copies[i % 2]
            if events is not None:
                events[j][0].record(stream)
            nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A16)
            if events is not None:
                events[j][1].record(stream)

    step_bytes = sum(decode_bytes(1, K, N) for _, K, N, *_ in layers)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    per_launch = [[] for _ in layers]
    ev_all = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in layers] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(i, ev_all[i])
        t1.record(stream)
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    for i in range(args.steps):
        for j in range(len(layers)):
            per_launch[j].append(ev_all[i][j][0].elapsed_time(ev_all[i][j][1]))
    if dist:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_per_step = ms / args.steps
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9

    # roofline of the dominant kernel (the W4A16 decode kernel: every launch)
    peak, peak_kind = load_peaks()
    launch_ms = sum(sum(v) for v in per_launch) / args.steps
    achieved = step_bytes / (launch_ms * 1e-3) / 1e9
    per_shape = {}
    for (name, K, N, *_), v in zip(layers, per_launch):
        m = statistics.median(v)
        per_shape[name] = {"us": round(m * 1e3, 2), "GB/s": round(decode_bytes(1, K, N) / (m * 1e-3) / 1e9, 1)}
    traffic = kernel_traffic("gemv.cu", "gemv_w4a16_decode")

    # end to end through the public API: pinned host x in, host y out, every step
    xh = [torch.empty((1, K), dtype=torch.bfloat16).pin_memory() for _, K, *_ in layers]
    for h_, (_, K, N, c, x, y) in zip(xh, layers):
        h_.copy_(x.cpu())
    yh = [torch.empty((1, N), dtype=torch.float32).pin_memory() for _, K, N, *_ in layers]
    h2d = sum(t.numel() * t.element_size() for t in xh)
    d2h = sum(t.numel() * t.element_size() for t in yh)

    def e2e_step(i):
        for j, (name, K, N, copies, x, y) in enumerate(layers):
            c, s, g = copies[i % 2]
            x.copy_(xh[j], non_blocking=True)
            nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A16)
            yh[j].copy_(y, non_blocking=True)

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
    e_ms = e0.elapsed_time(e1)
    if dist:
        t = torch.tensor([e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e_ms = float(t.item())
    e2e = world * step_bytes / (e_ms / args.steps * 1e-3) / 1e9

    extra = {"decode_m1_per_shape": per_shape}
    if not args.quick:
        extra["decode_sweep"] = decode_sweep(nv, torch, dev, layers)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 weights x bf16 activations, fp32 accumulate",
        "data": "synthetic: weights N(0,0.02) fp32 quantized on device, activations N(0,1) bf16",
        "config": {"workload": "dense27b decode linears (QKV 5120x10240, o_proj 5120x5120, gate_up 5120x34816, "
                               "down 17408x5120), W4A16, M=1",
                   "M": 1, "bytes_per_step": step_bytes,
                   "l2": "weights rotated over 2 copies (389 MB) > 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                     "kernel": "gemv_w4a16_kernel (4 launches per step, CUDA events per launch)"},
        "e2e": {"value": round(e2e, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 4 * args.steps,
        "clocks": clk.summary(),
        **extra,
    }
    return line


def decode_sweep(nv, torch, dev, layers, reps=20):
    """Median per-launch GB/s for each shape and M (weights rotated over 2 copies)."""
    from bit_linear_moe_b200 import synth
    out = {}
    stream = torch.cuda.current_stream()
    for name, K, N, copies, _, _ in layers:
        row = {}
        for M in synth.DECODE_M:
            x = torch.from_numpy(synth.decode_x(SHAPES[[s[0] for s in SHAPES].index(name)][3], M, K)).to(
                torch.bfloat16).to(dev)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            for i in range(3):
                c, s, g = copies[i % 2]
                nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A16)
            ts = []
            for i in range(reps):
                c, s, g = copies[i % 2]
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                nv.nvfp4_linear(x, c, s, g, w_sf_layout=nv.SF_TILED, y=y, mode=nv.MODE_W4A16)
                b.record(stream)
                ts.append((a, b))
            torch.cuda.synchronize()
            m = statistics.median(a.elapsed_time(b) for a, b in ts)
            row[str(M)] = round(decode_bytes(M, K, N) / (m * 1e-3) / 1e9, 1)
        out[name] = row
    return out


# --------------------------------------------------------------- reference ----

def oracle_decode_sample(reps: int = 1):
    """Time the oracle's W4A16 linear on the same four shapes at M = 1 (weights
    quantized by the oracle outside the timed region).  Returns (GB/s, seconds, threads)."""
    import oracle
    from bit_linear_moe_b200 import synth
    qs = []
    for name, K, N, seed in SHAPES:
        q = oracle.quantize(synth.dense_weight(seed, K, N))
        qs.append((K, N, q, synth.decode_x(seed, 1, K)))
    t = time.perf_counter()
    nbytes = 0
    for _ in range(reps):
        for K, N, q, x in qs:
            oracle.linear_w4a16(x, *q)
            nbytes += decode_bytes(1, K, N)
    dt = time.perf_counter() - t
    return nbytes / dt / 1e9, dt, oracle.num_threads()


def run_reference(args):
    gbs, dt, threads = oracle_decode_sample(reps=1)
    step_s = dt
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 3), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp64 accumulate (CPU oracle)",
        "data": "synthetic, same generator as the native arm",
        "config": {"workload": "dense27b decode linears (QKV 5120x10240, o_proj 5120x5120, gate_up 5120x34816, "
                               "down 17408x5120), W4A16, M=1", "M": 1},
        "cpu_baseline": {"value": round(gbs, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": "one step = the four linears at M=1, timed once after oracle quantization"},
        "e2e": {"value": round(gbs, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--quick", action="store_true", help="headline only (no sweeps, no CPU baseline)")
    args = ap.parse_args()
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
    if rank == 0 and not args.quick:
        gbs, dt, threads = oracle_decode_sample(reps=1)
        line["cpu_baseline"] = {"value": round(gbs, 3), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"the four linears at M=1 once ({dt:.1f} s)"}
    if rank == 0:
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
