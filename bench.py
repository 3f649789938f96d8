#!/usr/bin/env python3
"""Benchmark of the FP6 x FP16 weight-only linear layer on B200.

Workload (one "step"): the Llama-70B-shaped attention output projection,
N = K = 8192, at decode batch sizes M = 1, 2, 4, 8, 16 -- one fp6_linear
launch per M, each reading a different copy of the packed weights (copies
rotate so the weights streamed per launch are never L2-resident).  Metric:
effective weight GB/s = 0.75 * N * K bytes per launch / time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp6|reference]

Under torchrun (N > 1) every rank runs the same independent workload on its
own GPU (weak scaling, no data-path collective); the step time is the max over
ranks.  `--impl reference` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
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

WORKLOAD_NAME = "llama70b_o_proj_decode"
N_DIM, K_DIM = 8192, 8192
MS = [1, 2, 4, 8, 16]
METRIC = "FP6xFP16 linear: weight GB/s (M<=16) & TFLOP/s (M>=256), % of roofline"
UNIT = "GB/s"


# bytes per weight of each packed format
FORMAT_BYTES = {"e3m2": 0.75, "e2m3": 0.75, "e2m1": 0.5, "e2m2": 0.625, "s24": 0.375}
FORMAT_CODE = {"e3m2": None, "e2m3": 1, "e2m1": 2, "e2m2": 3, "s24": 4}


def wbytes(N, K, per_weight=0.75):
    return per_weight * N * K


def algo_bytes(M, N, K, per_weight=0.75):
    """Algorithmic bytes of one launch: packed weights + fp16 scales + fp16 activations."""
    return per_weight * N * K + 2 * N + 2 * M * K


PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "fp6_linear_decode_kernel_llama70b_o_proj_decode.md")


# The device sources the decode kernel (the bench's kernel) is compiled from:
# its own header and the headers it includes.  Its launch configuration
# (grid = SM count, block and shared memory from DecodeShape, T = kTMax) is
# fixed by them too.
DECODE_KERNEL_SOURCES = ["fp6_format.cuh", "fp6_linear.cuh", "fp6_linear_decode.cuh", "ptx.cuh"]


def kernel_source_hash() -> str:
    """First 16 hex digits of the SHA-256 over the decode kernel's device
    sources, in sorted name order."""
    import hashlib
    csrc = os.path.join(ROOT, "weight_only_quantized_fp6_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(DECODE_KERNEL_SOURCES):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes (read + write) of one launch from the committed ncu summary, or
    None when that capture was taken of a different kernel source."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    fields = {}
    for line in open(PROFILE_SUMMARY):
        m = re.match(r"^(kernel_source_sha256|dram_bytes_per_launch|captured_launch_M):\s*(\S+)", line)
        if m:
            fields[m.group(1)] = m.group(2)
    if fields.get("kernel_source_sha256") != kernel_source_hash() or "dram_bytes_per_launch" not in fields:
        return None
    return {"bytes": int(fields["dram_bytes_per_launch"]), "M": int(fields.get("captured_launch_M", 0))}


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---- clocks sampled during the timed region ---------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def mark(self) -> int:
        """Number of samples so far; stop(since=mark()) keeps only later ones."""
        return len(self.lines)

    def stop(self, since: int = 0):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[since:]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---- distributed plumbing --------------------------------------------------------

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- the oracle (CPU baseline / reference arm) ------------------------------------

def oracle_workload(rows: int):
    """Codes/scales of the first `rows` weight rows and the activations, from the oracle."""
    import oracle
    from weight_only_quantized_fp6_b200 import inputs
    wseed = inputs.weight_seed("llama70b_o_decode", 0)
    W = inputs.weights(wseed, N_DIM, K_DIM, rows=range(rows))
    codes, scales = oracle.quantize(W)
    xs = {M: inputs.activations(inputs.activation_seed(wseed, M), M, K_DIM) for M in MS}
    return codes, scales, xs


def time_oracle(rows: int, threads: int, reps: int = 1, workload=None):
    import oracle
    codes, scales, xs = workload if workload is not None else oracle_workload(rows)
    t0 = time.perf_counter()
    for _ in range(reps):
        for M in MS:
            oracle.linear(xs[M], codes, scales, nthreads=threads)
    dt = time.perf_counter() - t0
    gbs = reps * len(MS) * wbytes(rows, K_DIM) / dt / 1e9
    return gbs, dt


def cpu_baseline(target_s: float = 15.0):
    """The oracle on all host cores, on whole steps of the workload, repeated
    until about `target_s` seconds of CPU work have been timed."""
    threads = os.cpu_count() or 1
    rows = N_DIM  # the whole layer
    work = oracle_workload(rows)
    _, dt1 = time_oracle(rows, threads, workload=work)
    reps = max(1, int(math.ceil(target_s / max(dt1, 1e-3))))
    gbs, dt = time_oracle(rows, threads, reps=reps, workload=work)
    return {"value": round(gbs, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{reps} full steps (N={N_DIM}, K={K_DIM}, M={MS}) on {threads} threads, {dt:.2f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    threads = os.cpu_count() or 1
    rows = 2048  # a quarter of the layer per step keeps --steps 10 within a few minutes
    import oracle
    codes, scales, xs = oracle_workload(rows)
    for _ in range(args.warmup):
        for M in MS:
            oracle.linear(xs[M], codes, scales, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for M in MS:
            oracle.linear(xs[M], codes, scales, nthreads=threads)
    dt = time.perf_counter() - t0
    value = args.steps * len(MS) * wbytes(rows, K_DIM) / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": f"{WORKLOAD_NAME} N={N_DIM} K={K_DIM} M={MS}",
                                        "rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"first {rows} of {N_DIM} weight rows, all M, per step"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- context measurements outside the timed region ---------------------------------

PREFILL_SHAPES = [(28672, 8192), (8192, 28672)]   # Llama-70B-shaped gate/up and down halves
PREFILL_MS = [256, 1024, 4096]


def _graph_us(fn, stream, launches, reps=5):
    """Per-call device time of fn(i): `launches` calls captured in one CUDA
    graph (i = 0 .. launches-1, so fn can rotate over buffers), one untimed
    replay, then the median over `reps` timed replays."""
    import torch
    with torch.cuda.stream(stream):
        fn(0)                                 # eager call first: kernel attributes, cuBLAS handles
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(launches):
                fn(i)
        graph.replay()
        ts = []
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3 / launches)
    torch.cuda.synchronize()
    del graph
    return statistics.median(ts)


def measure_prefill_and_ablation(dev, stream, peaks, packs, scales, xs):
    """Compute-bound prefill sizes (TFLOP/s against the measured dense bf16/fp16
    peak) and the two-kernel comparison of the pages (separate dequant kernel,
    then a cuBLAS fp16 GEMM) next to the fused kernel and a plain fp16 GEMM
    (cuBLAS W16A16).  cuBLAS appears only here, as context.  Every figure is a
    CUDA-graph replay of several calls (median of 5 replays); outputs are
    allocated once, outside the graphs; the weights (176 MB per prefill
    layer, more than L2) are read from HBM by every call."""
    import torch

    import weight_only_quantized_fp6_b200 as fp6
    gen = torch.Generator(device=dev)
    gen.manual_seed(5000)
    prefill, ablation = [], []
    ws = fp6.Workspace(dev)
    for (N, K) in PREFILL_SHAPES:
        W = torch.randn(N, K, device=dev, generator=gen) * 0.02
        layer = fp6.FP6Linear.from_float(W)
        del W
        W16 = fp6.dequant(layer.packed, layer.scales, N, K)
        W16b = torch.empty_like(W16)
        for M in PREFILL_MS:
            x = torch.randn(M, K, device=dev, generator=gen).half()
            y = torch.empty((M, N), dtype=torch.float16, device=dev)
            ws.get(fp6.workspace_bytes(M, N, K))
            n_launch = 8 if M <= 1024 else 4
            t = _graph_us(lambda i: fp6.linear(x, layer.packed, layer.scales, N, K, out=y, workspace=ws),
                          stream, n_launch)
            t16 = _graph_us(lambda i: torch.matmul(x, W16.t(), out=y), stream, n_launch)
            t2 = _graph_us(lambda i: torch.matmul(x, fp6.dequant(layer.packed, layer.scales, N, K, out=W16b).t(),
                                                  out=y), stream, n_launch)
            fl = 2.0 * M * N * K
            prefill.append({"N": N, "K": K, "M": M, "us": round(t, 2), "tflops": round(fl / t / 1e6, 1),
                            "frac_of_peak": round(fl / t / 1e6 / peaks["bf16_tflops"], 4)})
            ablation.append({"N": N, "K": K, "M": M, "fused_us": round(t, 2), "dequant_then_gemm_us": round(t2, 2),
                             "cublas_w16a16_us": round(t16, 2)})
        # the dequant kernel alone: 0.75 B read + 2 B written per weight
        td = _graph_us(lambda i: fp6.dequant(layer.packed, layer.scales, N, K, out=W16b), stream, 8)
        dq_bytes = 0.75 * N * K + 2 * N + 2.0 * N * K
        ablation.append({"N": N, "K": K, "dequant_us": round(td, 2),
                         "dequant_gbs": round(dq_bytes / td / 1e3, 1),
                         "dequant_frac_of_hbm": round(dq_bytes / td / 1e3 / peaks["hbm_gbs"], 4)})
        del layer, W16, W16b
    # decode shape: rotate the packed copies (and two fp16 copies, 134 MB each) past L2
    N, K = N_DIM, K_DIM
    W16s = [fp6.dequant(packs[i], scales, N, K) for i in range(2)]
    W16b = torch.empty_like(W16s[0])
    for M in (1, 16):
        x = xs[M]
        y16 = torch.empty((M, N), dtype=torch.float16, device=dev)
        nl = 2 * len(packs)
        fused = _graph_us(lambda i: fp6.linear(x, packs[i % len(packs)], scales, N, K, out=y16, workspace=ws),
                          stream, nl)
        two = _graph_us(lambda i: torch.matmul(x, fp6.dequant(packs[i % len(packs)], scales, N, K, out=W16b).t(),
                                               out=y16), stream, nl)
        w16 = _graph_us(lambda i: torch.matmul(x, W16s[i % 2].t(), out=y16), stream, nl)
        ablation.append({"N": N, "K": K, "M": M, "fused_us": round(fused, 2),
                         "dequant_then_gemm_us": round(two, 2), "cublas_w16a16_us": round(w16, 2)})
    del W16s, W16b
    return prefill, ablation


# ---- the GPU arm -------------------------------------------------------------------

def run_fp6(args, world, rank, local):
    import torch

    import weight_only_quantized_fp6_b200 as fp6
    from weight_only_quantized_fp6_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024)

    # weights: seeded N(0, 0.02), quantized and packed by the library
    wseed = inputs.weight_seed("llama70b_o_decode", rank)
    W = inputs.weights_parallel(wseed, N_DIM, K_DIM)
    layer = fp6.FP6Linear.from_float(torch.from_numpy(W).to(dev))
    del W
    copies = max(2, math.ceil(4 * l2 / wbytes(N_DIM, K_DIM)))
    packs = [layer.packed] + [layer.packed.clone() for _ in range(copies - 1)]
    scales = layer.scales
    xs = {M: torch.from_numpy(inputs.activations(inputs.activation_seed(wseed, M), M, K_DIM).view(np.int16))
          .to(dev).view(torch.float16) for M in MS}
    ys = {M: torch.empty((M, N_DIM), dtype=torch.float16, device=dev) for M in MS}
    ws = fp6.Workspace(dev)
    ws.get(max(fp6.workspace_bytes(M, N_DIM, K_DIM) for M in MS))

    stream = torch.cuda.Stream(device=dev)
    # The timed steps are captured in one CUDA graph, as a serving engine runs
    # a decode step: each step's 5 launches back to back, every launch on the
    # next packed copy (kernel nodes only, so consecutive launches keep their
    # programmatic dependent-launch overlap, across step boundaries too).
    # Replaying it once runs exactly args.steps steps; a second graph of
    # args.warmup steps is the warm-up.
    def capture(n_steps):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for s in range(n_steps):
                for i, M in enumerate(MS):
                    fp6.linear(xs[M], packs[(s * len(MS) + i) % copies], scales, N_DIM, K_DIM,
                               out=ys[M], workspace=ws)
        return graph

    with torch.cuda.stream(stream):
        for M in MS:  # eager warm-up (sets kernel attributes before capture)
            fp6.linear(xs[M], packs[0], scales, N_DIM, K_DIM, out=ys[M], workspace=ws)
        stream.synchronize()
        timed_graph = capture(args.steps)
        warm_graph = capture(args.warmup)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        warm_graph.replay()
        timed_graph.replay()                 # first replay of the timed graph itself, untimed
    torch.cuda.synchronize()
    barrier(world)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.5)                          # nvidia-smi start-up
    since = sampler.mark()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t_start.record()
        timed_graph.replay()                 # exactly args.steps steps
        t_end.record()
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t_start.elapsed_time(t_end)
    # The timed region lasts milliseconds, less than the sampling period: keep
    # replaying the same step (untimed) for 0.5 s so the clock record covers
    # this load.
    t_soak = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_soak < 0.5:
            warm_graph.replay()
            stream.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop(since)
    clocks["window"] = "timed region + 0.5 s of the same graph replays right after it"

    elapsed_max = max_over_ranks(elapsed_ms, world)
    launches = args.steps * len(MS)
    total_bytes = world * launches * wbytes(N_DIM, K_DIM)
    value = total_bytes / (elapsed_max / 1e3) / 1e9
    # Roofline of the dominant (only) kernel: algorithmic bytes of the launches
    # in the timed region / their average duration back to back.
    algo = np.array([algo_bytes(M, N_DIM, K_DIM) for M in MS])
    avg_launch_ms = elapsed_ms / launches
    achieved = float(algo.mean() / (avg_launch_ms / 1e3) / 1e9)
    peaks = read_peaks()
    prof = profiled_traffic()

    # Per-M breakdown (outside the timed region): a graph of 2*copies launches
    # of one M, timed as a whole.
    per_m = []
    with torch.cuda.stream(stream):
        for M in MS:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for i in range(2 * copies):
                    fp6.linear(xs[M], packs[i % copies], scales, N_DIM, K_DIM, out=ys[M], workspace=ws)
            graph.replay()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(3):
                graph.replay()
            e1.record()
            torch.cuda.synchronize()
            per_m.append(e0.elapsed_time(e1) / (3 * 2 * copies))
            del graph
    per_m = np.array(per_m)

    # End to end through the public API with host buffers: every step copies
    # its five activation matrices host -> device from one pinned staging
    # buffer, runs the five layer calls (FP6Linear.__call__) and copies their
    # five outputs device -> host into a pinned buffer.  As a serving loop
    # would, consecutive steps overlap: two sets of device buffers, the input
    # copies on one copy stream and the output copies on another, so step
    # s + 1's inputs travel while step s computes and step s's outputs while
    # step s + 1 computes.  Every step's copies are inside the timed region.
    rows = sum(MS)
    x_host = torch.empty((rows, K_DIM), dtype=torch.float16).pin_memory()
    y_host = [torch.empty((rows, N_DIM), dtype=torch.float16).pin_memory() for _ in range(2)]
    off = np.cumsum([0] + MS)
    for M, o in zip(MS, off):
        x_host[o:o + M].copy_(xs[M].cpu())
    x_dev = [torch.empty((rows, K_DIM), dtype=torch.float16, device=dev) for _ in range(2)]
    y_dev = [torch.empty((rows, N_DIM), dtype=torch.float16, device=dev) for _ in range(2)]
    x_views = [[xd[o:o + M] for M, o in zip(MS, off)] for xd in x_dev]
    y_views = [[yd[o:o + M] for M, o in zip(MS, off)] for yd in y_dev]
    layers = [fp6.FP6Linear(p_, scales, N_DIM, K_DIM) for p_ in packs]
    h2d = x_host.numel() * 2
    d2h = y_host[0].numel() * 2
    e2e_steps = max(1, args.steps)
    h2d_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b on the device
    ev_comp = [torch.cuda.Event() for _ in range(2)]   # the step using buffer b has computed
    ev_out = [torch.cuda.Event() for _ in range(2)]    # buffer b's outputs are on the host

    def e2e_step(s):
        b = s % 2
        h2d_stream.wait_event(ev_comp[b])            # step s - 2 no longer reads x_dev[b]
        with torch.cuda.stream(h2d_stream):
            x_dev[b].copy_(x_host, non_blocking=True)
        ev_in[b].record(h2d_stream)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])                 # step s - 2's outputs have left y_dev[b]
        for i in range(len(MS)):
            layers[(s * len(MS) + i) % copies](x_views[b][i], out=y_views[b][i])
        ev_comp[b].record(stream)
        d2h_stream.wait_event(ev_comp[b])
        with torch.cuda.stream(d2h_stream):
            y_host[b].copy_(y_dev[b], non_blocking=True)
        ev_out[b].record(d2h_stream)

    def drain():
        for b in range(2):
            stream.wait_event(ev_out[b])

    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            e2e_step(s)
        drain()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        h2d_stream.wait_event(e0)
        d2h_stream.wait_event(e0)
        for s in range(e2e_steps):
            e2e_step(s)
        drain()                                       # every output copy is inside the region
        e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = world * e2e_steps * len(MS) * wbytes(N_DIM, K_DIM) / (e2e_ms / 1e3) / 1e9

    prefill = ablation = prefill_clocks = None
    if rank == 0 and not args.no_extra:
        psampler = ClockSampler(local)
        psampler.start()
        time.sleep(0.3)
        pmark = psampler.mark()
        prefill, ablation = measure_prefill_and_ablation(dev, stream, peaks, packs, scales, xs)
        prefill_clocks = psampler.stop(pmark)

    ok = fp6.device_status(dev)
    if ok != 0:
        raise SystemExit(f"device error word set: {ok}")

    if rank == 0:
        cpu = cpu_baseline() if world == 1 else None
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed_max / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16 x e3m2 -> f32 accumulate", "data": "synthetic (seeded N(0,0.02) weights, N(0,1) fp16 x)",
            "config": {
                "workload": f"{WORKLOAD_NAME} N={N_DIM} K={K_DIM} M={MS}",
                "launches_per_step": len(MS),
                "l2": f"{copies} rotating packed-weight copies ({copies * wbytes(N_DIM, K_DIM) / 1e6:.0f} MB > 4x L2 "
                      f"{l2 / 1e6:.0f} MB); CUDA-graph replay",
                "per_M_us": {str(M): round(float(t) * 1e3, 3) for M, t in zip(MS, per_m)},
                "avg_launch_us": round(avg_launch_ms * 1e3, 3),
                "per_M_roofline_frac": {str(M): round(algo_bytes(M, N_DIM, K_DIM) / (float(t) / 1e3) / 1e9
                                                      / peaks["hbm_gbs"], 4) for M, t in zip(MS, per_m)},
                "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
            },
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "traffic": prof["bytes"] if prof else None,
                         "traffic_note": (f"ncu dram read+write of one M={prof['M']} launch "
                                          f"(algorithmic {algo_bytes(prof['M'], N_DIM, K_DIM):.0f} B)")
                         if prof else "no ncu capture of this kernel source",
                         "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)",
                         "kernel": "fp6_linear_decode_kernel<16, Fmt::E3M2>"},
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        if prefill is not None:
            line["prefill"] = {"metric": "TFLOP/s, fused kernel, M >= 256 (tensor-bound sizes)",
                               "method": "CUDA-graph replay of 4-8 calls, median of 5 replays",
                               "clocks": prefill_clocks,
                               "peak_tflops": peaks["bf16_tflops"],
                               "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json bf16_tflops; fp16 runs at "
                                              f"the bf16 rate)", "runs": prefill}
            line["ablation"] = {"note": "separate dequant kernel + cuBLAS fp16 GEMM, and cuBLAS fp16 GEMM on "
                                        "the dequantized weights (W16A16), against the fused kernel; "
                                        "per launch, microseconds", "runs": ablation}
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """Every layer shape and M of the Llama-70B, OPT-30B and prefill configs:
    per-launch time (a CUDA graph of launches rotating over enough packed-weight
    copies that no launch finds its weights in L2), weight GB/s, TFLOP/s and the
    fraction of the roofline max(2MNK / P_tensor, (bNK + 2N + 2MK) / BW_hbm),
    b = 0.75 bytes per weight (FP6), 0.625 (FP5, --fmt e2m2) or 0.5 (FP4, --fmt e2m1).
    Weights and activations come from torch's seeded CUDA generator: the
    times do not depend on the values (parity is the tests' job)."""
    import torch

    import weight_only_quantized_fp6_b200 as fp6
    from weight_only_quantized_fp6_b200 import inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 1024 * 1024)
    peaks = read_peaks()
    gen = torch.Generator(device=dev)
    gen.manual_seed(6000)
    stream = torch.cuda.Stream(device=dev)
    ws = fp6.Workspace(dev)
    fmt, bpw = FORMAT_CODE[args.fmt], FORMAT_BYTES[args.fmt]
    rows = []
    for wname in ("llama70b_o_decode", "llama70b_all", "opt30b", "prefill"):
        spec = inputs.WORKLOADS[wname]
        for lname, (N, K) in spec["layers"].items():
            W = torch.randn(N, K, device=dev, generator=gen) * 0.02
            layer = fp6.FP6Linear.from_float(W, fmt=fmt)
            del W
            copies = max(1, min(8, math.ceil(4 * l2 / wbytes(N, K, bpw))))
            packs = [layer.packed] + [layer.packed.clone() for _ in range(copies - 1)]
            for M in spec["M"]:
                x = torch.randn(M, K, device=dev, generator=gen).half()
                y = torch.empty((M, N), dtype=torch.float16, device=dev)
                ws.get(fp6.workspace_bytes(M, N, K))
                n_launch = max(2 * copies, 8)
                with torch.cuda.stream(stream):
                    fp6.linear(x, packs[0], layer.scales, N, K, out=y, workspace=ws, fmt=fmt)
                    stream.synchronize()
                    graph = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(graph, stream=stream):
                        for i in range(n_launch):
                            fp6.linear(x, packs[i % copies], layer.scales, N, K, out=y, workspace=ws, fmt=fmt)
                    graph.replay()
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    for _ in range(3):
                        graph.replay()
                    e1.record()
                torch.cuda.synchronize()
                t = e0.elapsed_time(e1) * 1e-3 / (3 * n_launch)
                del graph
                t_tc = 2.0 * M * N * K / (peaks["bf16_tflops"] * 1e12)
                t_hbm = algo_bytes(M, N, K, bpw) / (peaks["hbm_gbs"] * 1e9)
                rows.append({"config": wname, "format": args.fmt, "layer": lname, "N": N, "K": K, "M": M,
                             "us": round(t * 1e6, 2), "weight_gbs": round(wbytes(N, K, bpw) / t / 1e9, 1),
                             "tflops": round(2.0 * M * N * K / t / 1e12, 1),
                             "bound": "tensor" if t_tc > t_hbm else "hbm",
                             "roofline_frac": round(max(t_tc, t_hbm) / t, 4)})
                print(json.dumps(rows[-1]), file=sys.stderr, flush=True)
            del layer, packs
    if fp6.device_status(dev) != 0:
        raise SystemExit("device error word set")
    print(json.dumps({"sweep": rows, "peaks": peaks, "l2_bytes": l2}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["fp6", "reference"], default="fp6")
    ap.add_argument("--sweep", action="store_true",
                    help="time every layer shape and M of the Llama-70B, OPT-30B and prefill configs (1 GPU)")
    ap.add_argument("--fmt", choices=sorted(FORMAT_BYTES), default="e3m2",
                    help="weight format of the --sweep (e3m2 = the FP6 layer the bench line times)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the prefill and two-kernel context measurements (outside the timed region)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.sweep:
        return run_sweep(args)
    if args.impl == "reference":
        # The reference arm runs on the host cores of rank 0 alone and uses no
        # collective: under torchrun the other ranks exit without work, and no
        # process group (nor CUDA) is set up for it.
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
    world, rank, local = dist_setup(args)
    try:
        rc = run_fp6(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
