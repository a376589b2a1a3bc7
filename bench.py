#!/usr/bin/env python
"""Benchmark of the B200 weight-only quantized linear layer (int4 nested superscale).

Headline: int4 decode GEMV at M=1 in GB/s of algorithmic bytes (packed codes +
group metadata + step words + x + y) and its fraction of the measured HBM
peak; alongside it, the int4 prefill GEMM at M=2048 in TFLOP/s against the
measured dense bf16 peak.

One timed step = one decode token through two layers of the int4 decode
workload -- (K=5120, N=27648) then (K=27648, N=5120), M=1 -- each a single
qlinear_gemv launch.  Three packed copies of each layer are rotated so that a
weight copy is touched only once per 491 MB of traffic (> 3x the 126 MB L2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (replicas: the layer has no data-path exchange, so no collective runs);
time is the max over ranks; rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "int4 qmv GEMV GB/s & % HBM peak (M=1); qmm GEMM TFLOP/s at M=2048"
LAYERS = [(5120, 27648), (27648, 5120)]  # (K, N) of the two decode layers
GEMM_M, GEMM_K, GEMM_N = 2048, 5120, 27648
COPIES = 3
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per GEMV launch from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum),
# valid only while the GEMV source is unchanged (hash of csrc/gemv.cuh at capture time).
NCU_TRAFFIC = {"gemv_src_sha256": "e96a8dbc0350f04aaba0ef5fcaa3db81b517d0102074e935a68b0e258c1b5f39",
               "bytes_per_launch": 83039104}  # mean over the two decode layers


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--gemm-iters", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true")
    ap.add_argument("--load-window", type=float, default=1.5,
                    help="seconds of extra steps run after the timed region so the clock sampler sees load")
    ap.add_argument("--case", default=None,
                    help="profiling aid: pack one workload layer (synth.WORKLOADS name), run --case-calls "
                         "qlinear_gemv (or --case-gemm: qlinear_gemm) calls at --case-m tokens, print one line")
    ap.add_argument("--case-m", type=int, default=1)
    ap.add_argument("--case-calls", type=int, default=3)
    ap.add_argument("--case-gemm", action="store_true")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (also exercised by a 2-rank gloo test on CPU)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(backend: str):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def reduce_scalar(x: float, op: str, device=None) -> float:
    """max/sum of a float over ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(units_this_rank: float, seconds_this_rank: float, device=None):
    """Whole-job throughput: units summed over ranks / max time over ranks."""
    total = reduce_scalar(units_this_rank, "sum", device)
    tmax = reduce_scalar(seconds_this_rank, "max", device)
    return total, tmax, total / tmax


# ---------------------------------------------------------------------------
# clocks sampled while the GPU is under load
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t0: float, t1: float):
        self.windows.append((t0, t1))

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not any(a - 0.05 <= ts <= b + 0.05 for a, b in self.windows):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            n += 1
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": n}


DATA = "synthetic (seeded uniform codes/metadata per the workload recipe; x ~ N(0,1) in bf16)"


def workload_config(world: int) -> dict:
    return {"workload": "int4 nested-superscale decode GEMV, M=1, layers (K=5120,N=27648) and (K=27648,N=5120)",
            "M": 1, "layers": LAYERS,
            "parallelism": (f"{world} replicas: every rank runs the same two layers on its own GPU, no "
                            f"collective" if world > 1 else "single GPU"),
            "launch": "the K timed steps are one CUDA graph of 2K qlinear_gemv calls",
            "l2": f"{COPIES} rotating packed copies per layer "
                  f"({COPIES * sum(gemv_bytes(K, N) for K, N in LAYERS) / 1e6:.0f} MB per rotation > 3x 126 MB L2)"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def gemv_bytes(K: int, N: int, M: int = 1) -> int:
    """Algorithmic bytes of one int4 GEMV: packed codes + group words + step words + x + y."""
    return N * K // 2 + N * (K // 32) * 2 + N * (K // 256) * 4 + M * K * 2 + M * N * 2


def gemv_src_sha():
    """Hash of the GEMV source with its // comments removed: any code change invalidates the ncu
    traffic figure, a comment edit does not."""
    with open(os.path.join(ROOT, "int6_quantized_linear_b200", "csrc", "gemv.cuh")) as f:
        lines = (re.sub(r"//.*", "", line).rstrip() for line in f)
        code = "\n".join(line for line in lines if line)
    return hashlib.sha256(code.encode()).hexdigest()


# ---------------------------------------------------------------------------
# native (CUDA) arm
# ---------------------------------------------------------------------------

def build_layers(device, copies=COPIES):
    import torch

    import int6_quantized_linear_b200 as ql
    from int6_quantized_linear_b200 import synth

    layers = []
    for li, (K, N) in enumerate(LAYERS):
        d = ql.Desc("int4", N, K)
        w = synth.int4_weights(1, N, K)
        dev = lambda a: torch.from_numpy(a.view("int16") if a.itemsize == 2 else a).to(device)
        q, sc, zc, ss, zs = (dev(w[k]) for k in ("q", "sc", "zc", "ss", "zs"))
        c0, g0, s0 = ql.alloc_packed(d, device)
        ql.qlinear_pack(d, q, sc, zc, ss, zs, c0, g0, s0)
        del q, sc, zc, ss, zs
        reps = [(c0, g0, s0)] + [(c0.clone(), g0.clone(), s0.clone()) for _ in range(copies - 1)]
        x = torch.from_numpy(synth.activations(1, 1, K).view("int16")).to(device).view(torch.bfloat16)
        y = torch.empty((1, N), dtype=torch.bfloat16, device=device)
        ws = ql.alloc_gemv_workspace(d, 1, device)
        layers.append(dict(desc=d, reps=reps, x=x, y=y, K=K, N=N, ws=ws))
    torch.cuda.synchronize(device)
    return layers


def gemv_step(layers, i: int, ql):
    for L in layers:
        c, g, s = L["reps"][i % len(L["reps"])]
        ql.qlinear_gemv(L["desc"], c, g, s, L["x"], 1, L["y"], L["ws"])


def gemv_m1_launches(K: int, N: int, sms: int) -> int:
    """Kernels one qlinear_gemv call at int4, M=1 launches: the streaming kernel, plus the kernel that
    adds the parts when K is split (the launcher's rule: the 4-tile CTA groups fill 3 CTAs per SM, at
    most K/256 parts, and at least enough parts that each holds 22 super-blocks of x)."""
    NS, groups = K // 256, -(-(-(-N // 16)) // 4)
    P = max(1, min(NS, sms * 3 // groups))
    P = max(P, -(-NS // 22))
    return 1 + (P > 1)


def _ev():
    import torch
    return torch.cuda.Event(enable_timing=True)


def capture(fn, device):
    """Record fn()'s launches into a CUDA graph (replayed on the current stream) and upload it to the
    device: the first launch of an executable graph otherwise uploads it first, a one-time cost
    (measured about 120 us for the 20-step decode graph) that belongs to no step."""
    import torch
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        fn()
    torch.cuda.current_stream(device).wait_stream(side)
    import cuda.bindings.runtime as cudart
    err, = cudart.cudaGraphUpload(g.raw_cuda_graph_exec(), torch.cuda.current_stream(device).cuda_stream)
    if err != cudart.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphUpload: {err}")
    torch.cuda.synchronize(device)
    return g


def per_launch_us(layers, ql, device, calls=30, reps=5):
    """Device time of one qlinear_gemv call per layer: a graph of `calls` calls over the rotating
    copies, replayed `reps` times, each replay between CUDA events on the launching stream; the
    median replay's time per call."""
    import torch
    out = []
    for L in layers:
        def body(L=L):
            for i in range(calls):
                c, g, s = L["reps"][i % len(L["reps"])]
                ql.qlinear_gemv(L["desc"], c, g, s, L["x"], 1, L["y"], L["ws"])
        gr = capture(body, device)
        gr.replay()
        torch.cuda.synchronize(device)
        times = []
        for _ in range(reps):
            a, b = _ev(), _ev()
            a.record()
            gr.replay()
            b.record()
            torch.cuda.synchronize(device)
            times.append(a.elapsed_time(b) * 1e3 / calls)
        out.append(sorted(times)[reps // 2])
        del gr
    return out


def run_native(args):
    import torch

    import int6_quantized_linear_b200 as ql

    rank, world = dist_init("nccl")
    _, _, local_rank = dist_env()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    peaks = load_peaks()
    sampler = ClockSampler(local_rank)
    sampler.start()

    layers = build_layers(device)
    step_bytes = sum(gemv_bytes(L["K"], L["N"]) for L in layers)

    # the timed steps are one CUDA graph (as a decode loop runs its layers), so each call's weight
    # stream can start while the previous call drains; warm-up is a graph of its own
    for i in range(COPIES):  # eager calls first: set-up work stays out of the captures
        gemv_step(layers, i, ql)
    torch.cuda.synchronize(device)

    def steps_graph(n):
        return capture(lambda: [gemv_step(layers, i, ql) for i in range(n)], device)

    g_warm, g_timed = steps_graph(args.warmup), steps_graph(args.steps)

    # warm-up, then exactly K timed steps between barrier + synchronize
    g_warm.replay()
    torch.cuda.synchronize(device)
    barrier(device)
    t_wall0 = time.time()
    ev0, ev1 = _ev(), _ev()
    ev0.record()
    g_timed.replay()
    ev1.record()
    torch.cuda.synchronize(device)
    t_wall1 = time.time()
    barrier(device)
    sampler.mark(t_wall0, t_wall1)
    assert ql.qlinear_sync_status() == ql.QL_OK
    elapsed_s = ev0.elapsed_time(ev1) / 1e3

    # keep the same load running for ~1.5 s so the clock sampler sees it
    t_a = time.time()
    while time.time() - t_a < args.load_window:
        g_timed.replay()
        torch.cuda.synchronize(device)
    sampler.mark(t_a, time.time())
    del g_warm, g_timed

    total_bytes, tmax, value_bps = aggregate(step_bytes * args.steps, elapsed_s, device)
    ms_per_step = tmax / args.steps * 1e3

    # roofline of the dominant kernel (the GEMV): algorithmic bytes per call / mean call time
    launch_us = per_launch_us(layers, ql, device)
    bytes_per_call = [gemv_bytes(L["K"], L["N"]) for L in layers]
    achieved_gbs = sum(bytes_per_call) / sum(launch_us) / 1e3
    traffic = (NCU_TRAFFIC["bytes_per_launch"]
               if NCU_TRAFFIC["gemv_src_sha256"] == gemv_src_sha() else None)

    gemm = run_gemm(args, device, peaks, sampler)
    e2e = run_e2e(args, layers, device, step_bytes)
    others = None if args.no_other_configs else run_other_configs(device, peaks)
    for L in layers:
        L["reps"].clear()
    clocks = sampler.stop()

    if rank != 0:
        return None
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    line = {
        "metric": METRIC,
        "value": round(value_bps / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int4 weights, bf16 activations, fp32 accumulate",
        "data": DATA,
        "config": workload_config(world),
        "pct_hbm_peak": round(100 * value_bps / 1e9 / peaks["hbm_gbs"], 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved_gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "peak_source": f"{peaks['source']} (copy bandwidth)", "kernel": "qlinear_gemv (int4, M=1)",
                     "bytes_per_call": bytes_per_call, "mean_call_us": [round(u, 3) for u in launch_us]},
        "gemm_m2048": gemm,
        "other_configs": others,
        "e2e": e2e,
        "gpu_launches": args.steps * sum(gemv_m1_launches(L["K"], L["N"], sms) for L in layers),
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "clock_samples": clocks["samples"],
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    return line


def run_gemm(args, device, peaks, sampler):
    """qlinear_gemm on the int4 prefill workload at M=2048 (K=5120, N=27648)."""
    import torch

    import int6_quantized_linear_b200 as ql
    from int6_quantized_linear_b200 import synth

    d = ql.Desc("int4", GEMM_N, GEMM_K)
    w = synth.int4_weights(3, GEMM_N, GEMM_K)
    t16 = lambda a: torch.from_numpy(a.view("int16") if a.itemsize == 2 else a).to(device)
    c, g, s = ql.alloc_packed(d, device)
    ql.qlinear_pack(d, t16(w["q"]), t16(w["sc"]), t16(w["zc"]), t16(w["ss"]), t16(w["zs"]), c, g, s)
    x = t16(synth.activations(3, GEMM_M, GEMM_K)).view(torch.bfloat16)
    y = torch.empty((GEMM_M, GEMM_N), dtype=torch.bfloat16, device=device)
    ws = ql.alloc_gemm_workspace(d, GEMM_M, device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    for _ in range(3):
        ql.qlinear_gemm(d, c, g, s, x, GEMM_M, y, ws)
    torch.cuda.synchronize(device)
    times = []
    t0 = time.time()
    for _ in range(args.gemm_iters):
        flush.fill_(1)  # write > L2 between timed calls
        a, b = _ev(), _ev()
        a.record()
        ql.qlinear_gemm(d, c, g, s, x, GEMM_M, y, ws)
        b.record()
        torch.cuda.synchronize(device)
        times.append(a.elapsed_time(b) / 1e3)
    sampler.mark(t0, time.time())
    assert ql.qlinear_sync_status() == ql.QL_OK
    flops = 2.0 * GEMM_M * GEMM_N * GEMM_K
    tmed = statistics.median(times)
    tmax = reduce_scalar(tmed, "max", device)
    tflops = flops / tmax / 1e12
    del flush, x, y, c, g, s, ws
    return {"value": round(tflops, 1), "unit": "TFLOP/s", "ms": round(tmax * 1e3, 4), "M": GEMM_M,
            "K": GEMM_K, "N": GEMM_N, "iters": args.gemm_iters,
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tflops / peaks["bf16_tflops"], 4),
                         "peak_source": f"{peaks['source']} dense bf16 (burst)"},
            "l2": "256 MiB buffer written between timed calls",
            "launches_per_call": 3, "note": "each call = x->fp16 pass + weight-scale pass + tcgen05 GEMM"}


def packed_layer(wl, device):
    """Pack one synthetic workload layer on the device; returns (desc, (codes, gmeta, steps), bytes)."""
    import numpy as np
    import torch

    import int6_quantized_linear_b200 as ql

    d = ql.Desc(wl.fmt, wl.N, wl.K, wl.bits, wl.group)
    w = wl.weights()
    t16 = lambda a: torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(device)
    if wl.fmt == "int4":
        u = (w["q"], w["sc"], w["zc"], w["ss"], w["zs"])
    elif wl.fmt in ("int6", "int6p"):
        u = (w["q"], w["sc"], None, w["st"], None)
    else:
        u = (w["q"], w["s"], w["b"], None, None)
    packed = ql.alloc_packed(d, device)
    ql.qlinear_pack(d, *[t16(a) if a is not None else None for a in u], *packed)
    return d, packed, sum(ql.qlinear_packed_bytes(d))


def run_other_configs(device, peaks):
    """The remaining workload configurations, each at its batch sizes: GB/s of algorithmic bytes for
    the GEMVs (CUDA-graph replays of at least 30 calls over enough rotating weight copies to move 3x
    the L2 per pass), TFLOP/s for the GEMM (CUDA events around single calls, 256 MiB written between
    calls)."""
    import torch

    import int6_quantized_linear_b200 as ql
    from int6_quantized_linear_b200 import synth

    out = {}
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    for name in ("int4_gemv_2048x2048", "int4_gemv_k5120_n27648", "int4_gemv_k27648_n5120",
                 "int6_gemv_k5120_n5120", "int6_gemv_k5120_n27648", "int6p_gemv_k5120_n5120",
                 "int6p_gemv_k5120_n27648", "affine2_k4096_n14336", "affine4_k4096_n14336",
                 "affine8_k4096_n14336"):
        wl = synth.WORKLOADS[name]
        d, p0, wbytes = packed_layer(wl, device)
        # enough rotating copies that one pass over them moves over 3x the L2 (every call reads HBM)
        copies = max(3, -(-3 * l2 // wbytes))
        reps = [p0] + [tuple(t.clone() for t in p0) for _ in range(copies - 1)]
        xb = torch.from_numpy(wl.x(max(wl.Ms)).view("int16")).to(device).view(torch.bfloat16)
        res = {}
        for M in wl.Ms:
            if name.startswith("int4") and name != "int4_gemv_2048x2048" and M == 1:
                continue  # the headline line above
            x = xb[:M].contiguous()
            y = torch.empty((M, wl.N), dtype=torch.bfloat16, device=device)
            ws = ql.alloc_gemv_workspace(d, M, device)
            for i in range(3):
                ql.qlinear_gemv(d, *reps[i], x, M, y, ws)
            calls = max(30, copies)
            g = capture(lambda: [ql.qlinear_gemv(d, *reps[i % copies], x, M, y, ws) for i in range(calls)], device)
            g.replay()
            torch.cuda.synchronize(device)
            a, b = _ev(), _ev()
            a.record()
            g.replay()
            g.replay()
            b.record()
            torch.cuda.synchronize(device)
            us = a.elapsed_time(b) * 1e3 / (2 * calls)
            nbytes = wbytes + M * wl.K * 2 + M * wl.N * 2
            res[f"M{M}"] = {"us": round(us, 3), "GB/s": round(nbytes / us / 1e3, 1),
                            "frac_hbm": round(nbytes / us / 1e3 / peaks["hbm_gbs"], 4), "copies": copies}
            if nbytes < 16e6:
                res[f"M{M}"]["note"] = (f"{nbytes / 1e6:.1f} MB per call: launch- and latency-dominated "
                                        f"(the weights alone take {nbytes / peaks['hbm_gbs'] / 1e3:.2f} us at peak)")
            del g
        out[name] = res
        del reps
    # the int4 decode GEMV with a bias epilogue (M=1, first decode layer)
    wl = synth.WORKLOADS["int4_gemv_k5120_n27648"]
    d, p0, wbytes = packed_layer(wl, device)
    reps = [p0] + [tuple(t.clone() for t in p0) for _ in range(2)]
    x = torch.from_numpy(wl.x(1).view("int16")).to(device).view(torch.bfloat16)
    y = torch.empty((1, wl.N), dtype=torch.bfloat16, device=device)
    bias = torch.zeros(wl.N, dtype=torch.bfloat16, device=device)
    ws = ql.alloc_gemv_workspace(d, 1, device)
    for i in range(3):
        ql.qlinear_gemv_bias(d, *reps[i], x, 1, bias, y, ws)
    calls = 30
    g = capture(lambda: [ql.qlinear_gemv_bias(d, *reps[i % 3], x, 1, bias, y, ws) for i in range(calls)], device)
    g.replay()
    torch.cuda.synchronize(device)
    a, b = _ev(), _ev()
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize(device)
    us = a.elapsed_time(b) * 1e3 / calls
    nbytes = wbytes + wl.K * 2 + wl.N * 4
    out["int4_gemv_bias_k5120_n27648"] = {"M1": {"us": round(us, 3), "GB/s": round(nbytes / us / 1e3, 1),
                                                 "frac_hbm": round(nbytes / us / 1e3 / peaks["hbm_gbs"], 4)}}
    del g, reps
    # metadata encoder on the int4 decode layer's metadata: float scale and zero per group -> codes + steps
    wl = synth.WORKLOADS["int4_gemv_k5120_n27648"]
    G = wl.K // 32
    gen = torch.Generator(device=device).manual_seed(wl.seed)
    scale = torch.rand((wl.N, G), generator=gen, device=device) * 1e-2 + 1e-4
    zero = torch.rand((wl.N, G), generator=gen, device=device) * 15
    sc, zc = (torch.empty((wl.N, G), dtype=torch.uint8, device=device) for _ in range(2))
    ss, zs = (torch.empty((wl.N, G // 8), dtype=torch.int16, device=device) for _ in range(2))
    de = ql.Desc("int4", wl.N, wl.K)
    calls = 20
    g = capture(lambda: [ql.qlinear_quantize_meta(de, scale, zero, sc, zc, ss, zs) for _ in range(calls)], device)
    g.replay()
    torch.cuda.synchronize(device)
    a, b = _ev(), _ev()
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize(device)
    us = a.elapsed_time(b) * 1e3 / calls
    nbytes = 2 * wl.N * G * 4 + 2 * wl.N * G + 2 * wl.N * (G // 8) * 2
    out["metadata_encoder_int4_k5120_n27648"] = {"us": round(us, 3), "GB/s": round(nbytes / us / 1e3, 1),
                                                 "frac_hbm": round(nbytes / us / 1e3 / peaks["hbm_gbs"], 4)}
    del g, scale, zero, sc, zc, ss, zs
    wl = synth.WORKLOADS["int4_gemm_k5120_n27648"]
    d, (c, g_, s), _ = packed_layer(wl, device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    res = {}
    for M in (512, 8192):
        x = torch.from_numpy(wl.x(M).view("int16")).to(device).view(torch.bfloat16)
        y = torch.empty((M, wl.N), dtype=torch.bfloat16, device=device)
        ws = ql.alloc_gemm_workspace(d, M, device)
        for _ in range(2):
            ql.qlinear_gemm(d, c, g_, s, x, M, y, ws)
        times = []
        for _ in range(5):
            flush.fill_(1)
            a, b = _ev(), _ev()
            a.record()
            ql.qlinear_gemm(d, c, g_, s, x, M, y, ws)
            b.record()
            torch.cuda.synchronize(device)
            times.append(a.elapsed_time(b) / 1e3)
        t = statistics.median(times)
        tf = 2.0 * M * wl.N * wl.K / t / 1e12
        res[f"M{M}"] = {"ms": round(t * 1e3, 4), "TFLOP/s": round(tf, 1),
                        "frac_bf16_peak": round(tf / peaks["bf16_tflops"], 4)}
        del x, y, ws
    out["int4_gemm_k5120_n27648"] = res
    # the tcgen05 GEMM on the other formats at M=2048: int6 (dense and planar) on the int6 layer's
    # shape, affine on the affine layer's shape
    for name in ("int6_gemv_k5120_n27648", "int6p_gemv_k5120_n27648", "affine2_k4096_n14336",
                 "affine4_k4096_n14336", "affine8_k4096_n14336"):
        wl = synth.WORKLOADS[name]
        d, (c, g_, s), _ = packed_layer(wl, device)
        M = 2048
        x = torch.from_numpy(wl.x(M).view("int16")).to(device).view(torch.bfloat16)
        y = torch.empty((M, wl.N), dtype=torch.bfloat16, device=device)
        ws = ql.alloc_gemm_workspace(d, M, device)
        for _ in range(2):
            ql.qlinear_gemm(d, c, g_, s, x, M, y, ws)
        times = []
        for _ in range(5):
            flush.fill_(1)
            a, b = _ev(), _ev()
            a.record()
            ql.qlinear_gemm(d, c, g_, s, x, M, y, ws)
            b.record()
            torch.cuda.synchronize(device)
            times.append(a.elapsed_time(b) / 1e3)
        t = statistics.median(times)
        tf = 2.0 * M * wl.N * wl.K / t / 1e12
        out["gemm_M2048_" + name.split("_")[0] + f"_k{wl.K}_n{wl.N}"] = {
            "ms": round(t * 1e3, 4), "TFLOP/s": round(tf, 1), "frac_bf16_peak": round(tf / peaks["bf16_tflops"], 4)}
        del x, y, ws, c, g_, s
    assert ql.qlinear_sync_status() == ql.QL_OK
    return out


def run_e2e(args, layers, device, step_bytes):
    """Same metric through the public API with host buffers: every step copies x from pinned host
    memory to the device and reads y back, inside the timed region."""
    import torch

    import int6_quantized_linear_b200 as ql

    # the step's inputs (both layers' x) in one pinned host buffer and one device buffer, its results
    # likewise: one copy each way per step; every layer's slice starts on a 16-byte boundary
    xs, ys = [L["x"].reshape(-1) for L in layers], [L["y"].reshape(-1) for L in layers]
    assert all(t.numel() % 8 == 0 for t in xs + ys)
    xh = torch.cat([t.cpu() for t in xs]).pin_memory()
    yh = torch.empty(sum(t.numel() for t in ys), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty(xh.numel(), dtype=torch.bfloat16, device=device)
    yd = torch.empty(yh.numel(), dtype=torch.bfloat16, device=device)
    xv = list(torch.split(xd, [t.numel() for t in xs]))
    yv = list(torch.split(yd, [t.numel() for t in ys]))
    h2d = xh.numel() * 2
    d2h = yh.numel() * 2

    stream = torch.cuda.current_stream(device)

    def step(i):  # the step's inputs in, its layers back to back (chained on the stream), its results out
        xd.copy_(xh, non_blocking=True)
        for L, x, y in zip(layers, xv, yv):
            c, g, s = L["reps"][i % len(L["reps"])]
            ql.qlinear_gemv(L["desc"], c, g, s, x, 1, y, L["ws"], stream)
        yh.copy_(yd, non_blocking=True)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(device)
    barrier(device)
    a, b = _ev(), _ev()
    a.record()
    for i in range(args.steps):
        step(i)
    b.record()
    torch.cuda.synchronize(device)
    barrier(device)
    _, tmax, v = aggregate(step_bytes * args.steps, a.elapsed_time(b) / 1e3, device)
    return {"value": round(v / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(tmax / args.steps * 1e3, 5)}


# ---------------------------------------------------------------------------
# CPU oracle: the baseline leg and the reference arm
# ---------------------------------------------------------------------------

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_layers(rows=None):
    """Both decode layers packed by the C oracle (the first `rows` rows of each when given), with
    their activation row: the same seeded inputs as the CUDA arm."""
    from int6_quantized_linear_b200 import synth
    from oracle import oracle_c as OC

    out = []
    for (K, N) in LAYERS:
        n = N if rows is None else min(N, rows)
        w = synth.int4_weights(1, N, K)  # the full layer's draw (a leading block of rows of it)
        packed = OC.int4_pack(w["q"][:n], w["sc"][:n], w["zc"][:n], w["ss"][:n], w["zs"][:n])
        del w
        out.append(dict(K=K, N=n, packed=packed, x=synth.activations(1, 1, K)))
    return out


def oracle_step(layers, block_weights: int = 1 << 24):
    """One pass of the C oracle over the given layers (fp32 dequant + fp64 matmul), in blocks of rows
    of about `block_weights` weights so host memory stays bounded.  Returns (algorithmic bytes, s)."""
    from oracle import oracle_c as OC

    total_b, total_s = 0, 0.0
    for L in layers:
        codes, gmeta, steps = L["packed"]
        rb = max(1, block_weights // L["K"])
        for r0 in range(0, L["N"], rb):
            sl = slice(r0, min(L["N"], r0 + rb))
            t0 = time.perf_counter()
            wf = OC.int4_dequant(codes[sl], gmeta[sl], steps[sl])
            OC.matmul_f64(L["x"], wf)
            total_s += time.perf_counter() - t0
        total_b += gemv_bytes(L["K"], L["N"])
    return total_b, total_s


def cpu_baseline(min_seconds: float = 10.0, one_core_rows: int = 1024) -> dict:
    """The C oracle on this host: whole decode steps (both layers, every row) on all cores, repeated
    until about `min_seconds` of CPU work; then one core on the first rows of each layer."""
    from oracle import oracle_c as OC

    cores = OC.num_threads()
    layers = oracle_layers()
    b_all, s_all, steps = 0, 0.0, 0
    while s_all < min_seconds:
        b, s = oracle_step(layers)
        b_all, s_all, steps = b_all + b, s_all + s, steps + 1
    del layers
    small = oracle_layers(one_core_rows)
    OC.set_num_threads(1)
    try:
        b1, s1 = oracle_step(small)
    finally:
        OC.set_num_threads(cores)
    return {"value": round(b_all / s_all / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{steps} whole decode steps (both layers, all rows, M=1): C oracle fp32 dequant + fp64 "
                      f"matmul, {b_all / 1e6:.0f} MB of algorithmic bytes in {s_all:.1f} s on {cores} threads",
            "one_core": {"value": round(b1 / s1 / 1e9, 5), "unit": "GB/s", "cores": 1,
                         "sample": f"first {one_core_rows} rows of each decode layer ({b1 / 1e6:.1f} MB in "
                                   f"{s1:.2f} s)"}}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:  # the oracle runs once, on rank 0's host cores
        return None
    from oracle import oracle_c as OC
    layers = oracle_layers()
    for _ in range(args.warmup):
        oracle_step(layers)
    tot_b, tot_s = 0, 0.0
    for _ in range(args.steps):
        b, s = oracle_step(layers)
        tot_b += b
        tot_s += s
    v = tot_b / tot_s / 1e9
    cores = OC.num_threads()
    sample = (f"whole decode steps: both layers, every row, M=1 (C oracle fp32 dequant + fp64 matmul on "
              f"{cores} threads of {cpu_model()})")
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_s / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights, bf16 activations, fp64 accumulate", "data": DATA, "config": workload_config(world),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_case(args):
    """A few eager calls of one workload layer, for a profiler's launch list or capture (the
    commands in profiles/): no timing, no JSON contract line."""
    import torch

    import int6_quantized_linear_b200 as ql
    from int6_quantized_linear_b200 import synth

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wl = synth.WORKLOADS[args.case]
    d, packed, _ = packed_layer(wl, device)
    M = args.case_m
    x = torch.from_numpy(wl.x(M).view("int16")).to(device).view(torch.bfloat16)
    y = torch.empty((M, wl.N), dtype=torch.bfloat16, device=device)
    if args.case_gemm:
        ws = ql.alloc_gemm_workspace(d, M, device)
        for _ in range(args.case_calls):
            ql.qlinear_gemm(d, *packed, x, M, y, ws)
    else:
        ws = ql.alloc_gemv_workspace(d, M, device)
        for _ in range(args.case_calls):
            ql.qlinear_gemv(d, *packed, x, M, y, ws)
    status = ql.qlinear_sync_status()
    print(f"case {args.case} M={M} calls={args.case_calls} status={ql.status_string(status)}")
    return None


def main(argv=None):
    args = parse_args(argv)
    if args.case:
        run_case(args)
        return
    line = run_reference(args) if args.impl == "reference" else run_native(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    try:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
