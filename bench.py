#!/usr/bin/env python
"""Benchmark of the B200 dropless top-k MoE layer.

One step = one training pass of the whole layer (forward + backward: router,
dispatch metadata, permute, grouped SwiGLU GEMMs, combine and all backward
kernels) over one batch of synthetic tokens, through the C ABI.  Default
workload: the training-step configuration N=16384, H=4096, E=64, top_k=4,
F=2048, bf16 (the one workload that exercises every step of the layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica on its own batch: the layer has no exchange step of its own, so the
data path has no collective; the only collective is the max-over-ranks of
the timing.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s on 1 B200; grouped-GEMM % bf16 peak; meta/gather % HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="train_step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload forward timings of the other configurations")
    ap.add_argument("--train-mode", type=int, default=1, choices=[1, 2],
                    help="1: keep the SwiGLU gates for the backward; 2: recompute them (less memory)")
    ap.add_argument("--aux-alpha", type=float, default=0.0, help="load-balancing loss weight (0 = off)")
    ap.add_argument("--capacity-factor", type=float, default=0.0,
                    help="token-dropping variant: per-expert capacity ceil(N/E*cf) (0 = dropless)")
    ap.add_argument("--tokens", type=int, default=0, help="override N (small profiling cases)")
    ap.add_argument("--experts", type=int, default=0, help="override E (small profiling cases)")
    return ap.parse_args()


def workload(args):
    from gen import WORKLOADS
    s = WORKLOADS[args.workload]
    if args.tokens:
        s = s.with_(N=args.tokens, name=s.name + f"_N{args.tokens}")
    if args.experts:
        s = s.with_(E=args.experts, name=s.name + f"_E{args.experts}")
    return s


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- work model

def flops_by_kernel(s):
    """Algorithmic FLOPs per launch (padding rows and recompute not counted)."""
    NKHF = s.N * s.K * s.H * s.F
    return {"gemm1_swiglu": 4 * NKHF, "gemm2": 2 * NKHF, "dgrad_w2_swiglu_bwd": 2 * NKHF,
            "wgrad_w2": 2 * NKHF, "wgrad_w1_w3": 4 * NKHF, "dgrad_x": 4 * NKHF,
            "route_umma": 2 * s.N * s.H * s.E}


def bytes_by_kernel(s, padded_rows):
    """Algorithmic HBM bytes per launch of the bandwidth-bound kernels."""
    b = 2 if s.dtype == "bf16" else 4
    N, K, H, E = s.N, s.K, s.H, s.E
    return {"route_simt": N * H * b + H * E * b + N * K * 8,
            "permute": N * H * b + padded_rows * H * b + N * K * 4,
            "combine": N * K * H * b + N * K * 8 + N * H * b,
            "combine_bwd": N * H * b + N * K * H * b + padded_rows * H * b + N * K * 12,
            "unpermute_dx": N * K * H * b + N * H * b + N * K * 12,
            # x is needed once per token; the CUDA-core kernel (fp32 layers)
            # gathers it once per assignment (K times, the repeats mostly from L2)
            "router_wgrad_partial": N * H * b + N * K * 8 + (padded_rows // 128) * H * 4,
            # tensor-core x^T D: x once, the token's K dlogits and expert ids,
            # dW_r written
            "router_wgrad": N * H * b + N * K * 8 + H * E * b,
            "meta_count": N * K * 4, "meta_place": N * K * 4 * 3}


def kernel_rooflines(per, steps, timed_ms, fl, by, peaks):
    """Per-kernel figures over the timed region and stage totals.

    per: kernel -> (total ms, launches) from the CUDA events; timed_ms: the
    whole timed region (a kernel's share is of that); fl / by: the
    algorithmic FLOPs / HBM bytes per launch.  Each kernel with a work model
    gets its achieved rate and the fraction of the roof it meets first: the
    sustained bf16 tensor peak or the HBM copy bandwidth (both measured; a
    kernel with both models, the router, is rated by its arithmetic
    intensity against the ridge; the dispatch metadata, a few hundred KB,
    is latency-bound and gets no fraction).  Stage totals: the grouped GEMMs against
    the tensor peak, the bandwidth-bound row kernels against HBM, and the
    dispatch metadata (latency-bound) in microseconds per step."""
    tensor_peak, hbm_peak = peaks["bf16_tflops_sustained"], peaks["hbm_gbs"]
    ridge = tensor_peak * 1e12 / (hbm_peak * 1e9)          # FLOP per byte
    kernels = {}
    for name, (tot, n) in per.items():
        avg_s = tot / n * 1e-3
        k = {"launches": n, "ms_avg": round(tot / n, 4), "share": round(tot / timed_ms, 4)}
        if name in fl:
            k["tflops"] = round(fl[name] / avg_s / 1e12, 1)
        if name in by:
            k["gbs"] = round(by[name] / avg_s / 1e9, 1)
        if name.startswith("meta_"):
            k["bound"] = "latency"                        # a few hundred KB per launch
        elif name in fl and (name not in by or fl[name] / by[name] >= ridge):
            k["bound"], k["frac"] = "tensor", round(fl[name] / avg_s / 1e12 / tensor_peak, 4)
            if "bf16_tflops" in peaks:
                k["frac_burst"] = round(fl[name] / avg_s / 1e12 / peaks["bf16_tflops"], 4)
        elif name in by:
            k["bound"], k["frac"] = "hbm", round(by[name] / avg_s / 1e9 / hbm_peak, 4)
        kernels[name] = k

    def total(names, work):
        t = sum(per[n][0] for n in names) * 1e-3
        w = sum(work[n] * per[n][1] for n in names)
        return w / t if t > 0 else 0.0

    gemms = [n for n in per if n in fl and n not in by]
    rows = [n for n in per if n in by and n not in fl and not n.startswith("meta_")]
    meta = [n for n in per if n.startswith("meta_")]
    stages = {}
    if gemms:
        r = total(gemms, fl) / 1e12
        stages["grouped_gemms"] = {"kernels": sorted(gemms), "tflops": round(r, 1),
                                   "frac": round(r / tensor_peak, 4)}
        if "bf16_tflops" in peaks:
            stages["grouped_gemms"]["frac_burst"] = round(r / peaks["bf16_tflops"], 4)
    if rows:
        r = total(rows, by) / 1e9
        stages["bandwidth_kernels"] = {"kernels": sorted(rows), "gbs": round(r, 1),
                                       "frac": round(r / hbm_peak, 4)}
    if meta:
        stages["metadata_us_per_step"] = round(sum(per[n][0] for n in meta) / steps * 1e3, 2)
    return kernels, stages


def step_tokens(s):
    return s.N


def layer_flops(s):
    fwd = 6 * s.N * s.K * s.H * s.F + 2 * s.N * s.H * s.E
    return fwd * 3 if s.training else fwd


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- traffic

def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, only while the kernel's source is unchanged since the capture
    (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    src = os.path.join(ROOT, "dropless_top_moe_b200", "csrc")
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        if len(parts) < 5 or parts[0] != kernel or parts[1] != workload:
            continue
        bytes_, fname, sha = float(parts[2]), parts[3], parts[4]
        try:
            cur = hashlib.sha256(open(os.path.join(src, fname), "rb").read()).hexdigest()[:16]
        except OSError:
            return None
        return bytes_ if cur in sha.split(",") else None
    return None


def routing_stats(layer, shape):
    """Load of the last routed batch: per-expert assignment counts (from the
    layer's inclusive bins), maxvio = max count / mean count - 1, and the
    padded rows the grouped GEMMs computed."""
    import numpy as np
    bins = layer.bins.cpu().numpy().astype(np.int64)
    counts = np.diff(np.concatenate([[0], bins]))
    mean = counts.sum() / max(shape.E, 1)
    return {"min_count": int(counts.min()), "max_count": int(counts.max()),
            "maxvio": round(float(counts.max() / mean - 1.0), 3) if mean > 0 else None,
            "assignments": int(counts.sum()), "padded_rows": int(layer.padded_bins[-1].item())}


# ---------------------------------------------------------------- our arm

class Tracer:
    """CUDA events the library records just before and after each of its
    kernel launches (moe_trace_attach), with the launch names."""

    def __init__(self, cap: int):
        self.cap = 0
        self.evs = []
        self.count = ctypes.c_int32(0)
        self.grow(cap)

    def grow(self, cap: int):
        import torch
        if cap <= self.cap:
            return
        new = [torch.cuda.Event(enable_timing=True) for _ in range(2 * (cap - self.cap))]
        for e in new:           # torch creates the underlying cudaEvent on first record
            e.record()
        torch.cuda.synchronize()
        self.evs += new
        self.cap = cap
        self.arr = (ctypes.c_void_p * (2 * cap))(*[e.cuda_event for e in self.evs])
        self.labels = (ctypes.c_char_p * cap)()

    def attach(self):
        from dropless_top_moe_b200._lib import call
        self.count.value = 0
        call("moe_trace_attach", self.arr, self.cap, self.labels, ctypes.byref(self.count))

    def detach(self):
        from dropless_top_moe_b200._lib import call
        call("moe_trace_detach")

    def per_kernel(self):
        """kernel name -> (total ms, launches) over the launches recorded."""
        per = {}
        for i in range(min(self.count.value, self.cap)):
            name = self.labels[i].decode()
            d = self.evs[2 * i].elapsed_time(self.evs[2 * i + 1])
            tot, n = per.get(name, (0.0, 0))
            per[name] = (tot + d, n + 1)
        return fold_split_launches(per)


# GEMM1 and the SwiGLU-backward dgrad of a layer with many one-tile experts
# run as two launches each (CTA pairs, then the one-tile experts on single
# CTAs): second launch -> the kernel whose work model covers both.
SPLIT_LAUNCHES = (("gemm1_swiglu_single", "gemm1_swiglu"),
                  ("dgrad_w2_swiglu_bwd_single", "dgrad_w2_swiglu_bwd"))


def fold_split_launches(per):
    """Sum each second launch's time into its kernel, whose launch count
    (one per step) the work model divides by."""
    for part, whole in SPLIT_LAUNCHES:
        if part in per and whole in per:
            per[whole] = (per[whole][0] + per.pop(part)[0], per[whole][1])
    return per


def launches_per_step(step, tracer):
    import torch
    tracer.attach()
    step()
    torch.cuda.synchronize()
    tracer.detach()
    return tracer.count.value


def timed_steps(step, steps, tracer, gpu, flush=None):
    """Device time of `steps` calls of step() (CUDA events on the current
    stream, synchronised on both sides) with the per-launch trace attached
    and the SM clocks sampled meanwhile.  Without `flush` the steps run back
    to back between two events; with it, flush() (an L2-sized write) runs
    before every step, outside that step's own pair of events."""
    import torch
    clocks = ClockSampler(gpu)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    tracer.attach()
    if flush is None:
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(steps):
            step()
        s1.record()
        torch.cuda.synchronize()
        ms = s0.elapsed_time(s1)
    else:
        pairs = []
        for _ in range(steps):
            flush()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            step()
            s1.record()
            pairs.append((s0, s1))
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in pairs)
    tracer.detach()
    return ms / steps, clocks.stop()


def roofline_of(per, steps, ms, shape, layer, capacity, peaks, peak_src, traffic=None):
    """Per-kernel rooflines, stage totals and the dominant kernel's roofline
    object of one timed workload."""
    padded_rows = int(layer.padded_bins[-1].item()) if shape.N else 0
    # algorithmic work counts the assignments actually computed (all N*K when
    # dropless; the kept ones in the token-dropping variant)
    kept = int(layer.bins[-1].item()) if shape.N else 0
    work = shape.with_(K=1, N=kept) if capacity else shape
    fl = flops_by_kernel(work)
    fl["route_umma"] = 2 * shape.N * shape.H * shape.E
    by = bytes_by_kernel(shape, padded_rows)
    by["route_umma"] = by["route_simt"]
    kernels, stages = kernel_rooflines(per, steps, ms * steps, fl, by, peaks)
    dom = max(per, key=lambda n: per[n][0])
    dom_avg_s = per[dom][0] / per[dom][1] * 1e-3
    if dom in fl:
        peak, burst = peaks["bf16_tflops_sustained"], peaks["bf16_tflops"]
        achieved = fl[dom] / dom_avg_s / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} sustained bf16 (kernel timed inside a long step)",
                "peak_burst": burst, "frac_burst": round(achieved / burst, 4)}
    else:
        peak = peaks["hbm_gbs"]
        achieved = by.get(dom, 0) / dom_avg_s / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": f"{peak_src} copy bandwidth"}
    roof["traffic"] = traffic(dom) if traffic else None
    tfl = (layer_flops(work) - (2 * work.N * work.H * work.E) * (3 if shape.training else 1)
           + (2 * shape.N * shape.H * shape.E) * (3 if shape.training else 1))
    return roof, stages, kernels, round(tfl / (ms * 1e-3) / 1e12, 1)


def workload_desc(shape):
    return (f"{shape.name}: N={shape.N} H={shape.H} E={shape.E} top_k={shape.K} F={shape.F} SwiGLU, "
            f"{'forward+backward' if shape.training else 'forward'}")


L2_BYTES = 126 * 2 ** 20


def footprint_bytes(shape):
    """Bytes a step reads at least once: tokens, router and expert weights."""
    b = 2 if shape.dtype == "bf16" else 4
    return (shape.N * shape.H + shape.H * shape.E + 3 * shape.E * shape.H * shape.F) * b


def run_config(name, steps, dev, tracer, peaks, peak_src):
    """One forward workload of the layer, timed alone, for the per-config part
    of the JSON line."""
    import torch

    from gen import WORKLOADS, make_inputs
    import dropless_top_moe_b200 as moe
    shape = WORKLOADS[name]
    inp = make_inputs(shape, seed=0, device=dev)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=False, device=dev)

    def step():
        layer.forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"])

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    n_launch = launches_per_step(step, tracer)
    # enough steps for the clock samples (100 ms apart) to see the run
    t0 = time.perf_counter()
    step()
    torch.cuda.synchronize()
    est = max(time.perf_counter() - t0, 1e-5)
    n_steps = int(min(500, max(steps, 0.5 / est)))
    tracer.grow(n_launch * n_steps)
    flush = None
    l2 = "inputs larger than L2 (%.2f GB read per step)" % (footprint_bytes(shape) / 1e9)
    if footprint_bytes(shape) < 2 * L2_BYTES:
        buf = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
        flush = buf.zero_
        l2 = "L2 flushed before every step (256 MB write outside the step's events)"
    ms, clk = timed_steps(step, n_steps, tracer, dev.index or 0, flush)
    per = tracer.per_kernel()
    status = layer.status()
    roof, stages, kernels, tflops = roofline_of(per, n_steps, ms, shape, layer, 0, peaks, peak_src)
    out = {"workload": workload_desc(shape), "dtype": shape.dtype, "steps": n_steps, "warmup": 3,
           "ms_per_step": round(ms, 4), "value": round(shape.N / (ms * 1e-3), 1), "unit": "tokens/s",
           "tflops": tflops, "l2": l2, "routing": routing_stats(layer, shape), "roofline": roof,
           "stages": stages, "kernels": kernels, "gpu_launches": tracer.count.value,
           "launches_per_step": n_launch, "device_status": status, "clocks": clk}
    del layer, inp
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import math

    import torch
    import torch.distributed as dist

    from gen import WORKLOAD_ORDER, make_inputs, token_rows
    from gen.moe_inputs import _gen

    import dropless_top_moe_b200 as moe

    shape = workload(args)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = make_inputs(shape, seed=0, device=dev, with_dy=shape.training)
    if world > 1:   # each replica its own batch, same weights
        inp["x"] = token_rows(shape, shape.N, _gen(1000 + rank, dev), dev)
        if shape.training:
            inp["dy"] = torch.randn(shape.N, shape.H, generator=_gen(2000 + rank, dev), device=dev).to(shape.torch_dtype)
    # capacity per expert = ceil(N*K/E * cf): cf = 1 is the balanced load
    capacity = (int(math.ceil(shape.N * shape.K / shape.E * args.capacity_factor))
                if args.capacity_factor > 0 else 0)
    train_mode = args.train_mode if shape.training else 0
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=train_mode, device=dev, aux_alpha=args.aux_alpha, capacity=capacity)
    grads = layer.grad_buffers() if shape.training else None

    def step():
        layer.forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"])
        if shape.training:
            layer.backward(inp["dy"], inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], grads)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    tracer = Tracer(4096)
    per_step = launches_per_step(step, tracer)
    steps = args.steps
    tracer.grow(per_step * steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms, clk = timed_steps(step, steps, tracer, local_rank)
    if world > 1:
        dist.barrier()
    t = torch.tensor([ms], device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    status = layer.status()
    per = tracer.per_kernel()
    peaks, peak_src = load_peaks()
    default_variant = args.aux_alpha == 0 and args.capacity_factor == 0 and args.train_mode == 1
    # the capture is of the named workload's default variant only
    traffic = (lambda k: recorded_traffic(k, shape.name)) if default_variant else None
    roof, stages, kernels, tflops = roofline_of(per, steps, ms, shape, layer, capacity, peaks, peak_src, traffic)

    result = {
        "metric": METRIC, "value": None, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if shape.dtype == "bf16" else "f32",
        "data": "synthetic (seeded normal inputs and random-init weights of the stated shapes)",
        "config": {"workload": workload_desc(shape),
                   "tokens_per_step_per_gpu": shape.N, "parallelism": f"replicas x{world}",
                   "variant": {"train_mode": train_mode, "aux_alpha": args.aux_alpha,
                               "capacity": capacity or "dropless"},
                   "l2": "inputs larger than L2 (expert weights %.2f GB per step)" %
                         (3 * shape.E * shape.H * shape.F * 2 / 1e9)},
        "routing": routing_stats(layer, shape),
        "tflops": round(tflops * ms / ms_max, 1),
        "roofline": roof, "stages": stages, "kernels": kernels, "gpu_launches": tracer.count.value,
        "launches_per_step": per_step, "device_status": status, "clocks": clk,
    }
    result["value"] = round(shape.N * world / (ms_max * 1e-3), 1)

    # End to end through the same entry points with host buffers: every step
    # copies its x (and dy) from pinned host memory and reads y (and dx) back,
    # inside the timed region.  As a training loop's loader would, the next
    # step's inputs are copied while the current step computes (two device
    # buffer sets, one stream per copy direction).
    if not args.no_e2e:
        comp = torch.cuda.current_stream(dev)
        h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        xh = inp["x"].cpu().pin_memory()
        dyh = inp["dy"].cpu().pin_memory() if shape.training else None
        yh = torch.empty_like(xh).pin_memory()
        dxh = torch.empty_like(xh).pin_memory() if shape.training else None
        xd = [torch.empty_like(inp["x"]) for _ in range(2)]
        dyd = [torch.empty_like(inp["x"]) for _ in range(2)] if shape.training else None
        yd = [torch.empty_like(inp["x"]) for _ in range(2)]
        gb = None
        if shape.training:
            gb = [dict(grads), dict(grads)]
            gb[1]["dx"] = torch.empty_like(grads["dx"])
        ev = lambda: torch.cuda.Event()
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def h2d(b):
            with torch.cuda.stream(h2d_s):
                xd[b].copy_(xh, non_blocking=True)
                if shape.training:
                    dyd[b].copy_(dyh, non_blocking=True)
                h2d_done[b].record(h2d_s)

        def run(n):
            h2d(0)
            for i in range(n):
                b, nb = i % 2, 1 - i % 2
                if i + 1 < n:
                    if i >= 1:
                        h2d_s.wait_event(comp_done[nb])   # step i-1 is done with buffer nb
                    h2d(nb)
                comp.wait_event(h2d_done[b])
                if i >= 2:
                    comp.wait_event(d2h_done[b])          # step i-2's results read back
                y = layer.forward(xd[b], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], y=yd[b])
                if shape.training:
                    layer.backward(dyd[b], xd[b], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], gb[b])
                comp_done[b].record(comp)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(comp_done[b])
                    yh.copy_(y, non_blocking=True)
                    if shape.training:
                        dxh.copy_(gb[b]["dx"], non_blocking=True)
                    d2h_done[b].record(d2h_s)
            comp.wait_event(d2h_done[(n - 1) % 2])

        run(3)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        n_e2e = max(5, steps // 2)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(comp)
        h2d_s.wait_event(s0)
        run(n_e2e)
        s1.record(comp)
        torch.cuda.synchronize()
        ems = s0.elapsed_time(s1) / n_e2e
        te = torch.tensor([ems], device=dev)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        ems = float(te.item())
        eb = xh.element_size()
        result["e2e"] = {"value": round(shape.N * world / (ems * 1e-3), 1), "unit": "tokens/s",
                         "ms_per_step": round(ems, 4),
                         "h2d_bytes_per_step": xh.numel() * eb * (2 if shape.training else 1),
                         "d2h_bytes_per_step": xh.numel() * eb * (2 if shape.training else 1),
                         "note": "host copies of step i+1 / i overlap compute of step i"}

    # The other workloads of the layer (forward only), each timed alone on
    # this GPU after the headline workload, on rank 0 of a single-GPU run.
    if (world == 1 and not args.no_configs and args.workload == "train_step" and not args.tokens
            and not args.experts and default_variant):
        del layer, grads, inp
        torch.cuda.empty_cache()
        result["configs"] = {}
        for name in WORKLOAD_ORDER:
            if name != shape.name:
                result["configs"][name] = run_config(name, min(steps, 20), dev, tracer, peaks, peak_src)
        inp = None

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(shape, inp, target_s=10.0)
    return result


# ---------------------------------------------------------------- oracle legs

def _oracle_inputs(shape, inp=None):
    """float64 host copies of one workload's inputs (made once, outside timing)."""
    import torch
    from gen import make_inputs
    from oracle import moe_oracle as om
    if inp is None:
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        inp = make_inputs(shape, seed=0, device=dev, with_dy=True)
        if "dy" not in inp:
            inp["dy"] = torch.randn(shape.N, shape.H, device=dev).to(shape.torch_dtype)
    dy = inp.get("dy")
    if dy is None:
        dy = torch.zeros(shape.N, shape.H)
    return {k: om.f64(v) for k, v in (("x", inp["x"]), ("W_r", inp["W_r"]), ("W1", inp["W1"]),
                                      ("W3", inp["W3"]), ("W2", inp["W2"]), ("dy", dy))}


def _oracle_step(shape, o, tokens):
    from oracle import moe_oracle as om
    xs = o["x"][tokens]
    out = om.moe_forward(xs, o["W_r"], o["W1"], o["W3"], o["W2"], shape.K)
    if shape.training:
        om.moe_backward(xs, o["W_r"], o["W1"], o["W3"], o["W2"], shape.K, o["dy"][tokens],
                        routing=out["routing"])
    return out


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def _size_sample(shape, o, rng, target_s):
    """Token count of an oracle pass that takes about target_s seconds on
    this host, found by timing passes of growing seeded samples.

    A pass does not cost in proportion to its tokens while the sample is
    small: the backward zero-fills dense float64 weight gradients (E*H*F
    elements each, several GB at the training-step sizes) and every expert
    a sample touches streams its float64 weights.  So the sample grows from
    256 tokens, each next size extrapolated from the last two passes, until
    a pass takes at least half the target (or the sample is the whole
    batch).  Returns (tokens, seconds) of that last pass."""
    import numpy as np

    def timed(n):
        tok = np.sort(rng.choice(shape.N, n, replace=False))
        t0 = time.perf_counter()
        _oracle_step(shape, o, tok)
        return time.perf_counter() - t0

    n, prev = min(256, shape.N), None
    while True:
        dt = timed(n)
        if dt >= 0.5 * target_s or n >= shape.N:
            return n, dt
        guess = 4 * n
        if prev is not None and dt > prev[1] and n > prev[0]:
            guess = n + (target_s - dt) * (n - prev[0]) / (dt - prev[1])
        prev = (n, dt)
        n = int(min(shape.N, max(1.5 * n, min(guess, 8 * n))))


def cpu_baseline(shape, inp=None, target_s=10.0, o=None):
    """The oracle, as it stands, on one bounded token sample of the workload,
    grown until one pass takes about target_s seconds (its fixed per-call
    costs then weigh little in the tokens/s); the last pass is the number."""
    import numpy as np
    o = o if o is not None else _oracle_inputs(shape, inp)
    n, dt = _size_sample(shape, o, np.random.default_rng(0), target_s)
    return {"value": round(n / dt, 3), "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
            "sample": f"{n} of {shape.N} tokens of {shape.name} ({'fwd+bwd' if shape.training else 'fwd'}), "
                      f"float64 numpy oracle, {dt:.1f} s"}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on this workload's config, host cores.

    Each timed step is one oracle pass over a seeded token sample sized, like
    the in-line CPU baseline, to about 10 s (less when many steps would run
    past about 200 s of timed work), so that the oracle's fixed per-call
    costs do not dominate its tokens/s.  Warm-up steps use a small sample:
    they are untimed and only warm the host caches and allocator."""
    import numpy as np
    if rank != 0:
        return None
    shape = workload(args)
    o = _oracle_inputs(shape)
    rng = np.random.default_rng(1)
    target = min(10.0, 200.0 / max(args.steps, 1))
    n, _ = _size_sample(shape, o, rng, target)
    for _ in range(args.warmup):
        _oracle_step(shape, o, np.sort(rng.choice(shape.N, min(16, shape.N), replace=False)))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(shape, o, np.sort(rng.choice(shape.N, n, replace=False)))
    dt = time.perf_counter() - t0
    v = n * args.steps / dt
    ms = dt / args.steps * 1e3
    sample = f"{n} of {shape.N} tokens per step (seeded), float64 numpy oracle, {dt / args.steps:.1f} s per step"
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{shape.name}: N={shape.N} H={shape.H} E={shape.E} top_k={shape.K} "
                                   f"F={shape.F} SwiGLU, {'forward+backward' if shape.training else 'forward'}",
                       "tokens_per_step": n},
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import datetime
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if rank == 0:
        from dropless_top_moe_b200.build import build
        build()
    if world > 1:
        dist.barrier()
    res = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
