#!/usr/bin/env python
"""Benchmark of the H-BitLinear forward on B200: one JSON line on rank 0.

A step is one pass of the whole forward over one batch of synthetic input: absmean
ternarisation + packing of the latent weights (2 kernels), the fused Hadamard + absmax INT8
quantisation of the tokens (1 kernel) and the ternary x int8 tensor-core product with the bf16
rescale (1 kernel).  Default workload: the 7B-scale down projection, the largest layer of the
pages' workloads that one GPU holds (M = 16384 tokens, K = 16384, N = 4096, H-BitLinear, INT4
activations).

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier and
cuda.synchronize on both sides, timed with CUDA events on the launching stream, max over ranks.
Inputs are rotated over several copies whose total exceeds twice the L2 cache, so no step finds
its inputs in L2.  Each copy's step is one CUDA graph, so host launch overhead does not starve
the GPU: the weight ternarisation and the activation quantisation run side by side on two
streams (they are independent), then the tensor-core product.  The last few timed steps replay
a copy of their graph in which two timing events bracket the product; those events give the
product's live duration for the roofline figure.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
Under torchrun (N > 1) every rank runs its own batch (weak scaling, no collective on the data
path); rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_activation_linear_b200 import synth  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
PROFILES = os.path.join(ROOT, "profiles")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense ratio on B200: 4.5 POPS int8 vs 2.25 PFLOP/s bf16
# the product's kernel by the library's plan query (bitnet_product_path), for M > 8
PRODUCT_KERNEL = {1: "ternary_gemv", 2: "ternary_gemm_tc", 3: "ternary_gemm_skinny",
                  4: "ternary_gemm_pair_ts"}
# the activation quantiser's kernel, by the library's own plan query (bitnet_quant_path)
QUANT_KERNEL = {1: "act_quant_plain", 2: "fwht_quant", 3: "hadamard_tc_quant"}
METRIC = "H-BitLinear tokens/s and effective int8 TOPS (% of roofline) on 1 B200"


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------------------
# algorithmic work per kernel (bytes at the stored widths, ops of the product)
# ----------------------------------------------------------------------------------------

def weight_bytes(N: int, K: int, base3: bool) -> int:
    """Bytes of stored ternary weights: 2 bits a weight, or rows of ceil(K/20) 32-bit words of
    five base-3 weights a byte."""
    return N * 4 * ((K + 19) // 20) if base3 else N * K // 4


def kernel_work(wl, base3: bool = False, rotate: bool = False):
    M, K, N = wl.M, wl.K, wl.N
    code_bytes = M * K if wl.act_bits == 8 else M * K // 2
    wb = weight_bytes(N, K, base3)
    return {
        # read W (bf16) once; with the weight rotation: the transform (bf16 in, fp32 out), then
        # the sum over the fp32 rows
        "absmean_partials": {"bytes": (2 + 4 + 4) * N * K if rotate else 2 * N * K},
        # read W (bf16) once, write the stored weights
        "ternarize_pack": {"bytes": (4 if rotate else 2) * N * K + wb},
        # read X (bf16), write codes + scale + code sum per token
        "fwht_quant": {"bytes": 2 * M * K + code_bytes + 8 * M},
        # product: 2 M N K integer ops; bytes = codes + 2-bit weights + bf16 Y
        "ternary_gemm_tc": {"ops": 2 * M * N * K,
                            "bytes": code_bytes + wb + 2 * M * N + 8 * M},
    }


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (read + write) from the committed ncu capture of this workload
    (profiles/ncu_traffic_<workload>.json), or None when there is none or the kernel's source
    changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(PROFILES, f"ncu_traffic_{workload}.json")) as f:
            cap = json.load(f)
    except (OSError, ValueError):
        return None
    k = cap.get("kernels", {}).get(kernel)
    if k is None or not cap.get("workload", "").startswith(workload + " "):
        return None
    with open(os.path.join(ROOT, k["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != k["source_sha256_16"]:
            return None
    return k["dram_read_bytes"] + k["dram_write_bytes"]


# ----------------------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        # the raw samples go to $BITNET_BENCH_OUT (default: the system temporary directory); the
        # JSON line carries their summary
        out_dir = os.environ.get("BITNET_BENCH_OUT", tempfile.gettempdir())
        os.makedirs(out_dir, exist_ok=True)
        self.path = os.path.join(out_dir, f"bench_clocks_rank{self.idx}.csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append({"sm": float(parts[1]), "max": float(parts[2]),
                                 "power": float(parts[3]), "active": parts[4],
                                 "hw": parts[5], "hw_thermal": parts[6],
                                 "sw_thermal": parts[7], "sw_power": parts[8]})
                except ValueError:
                    continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples under load: the SM clock is the one the GPU ran the steps at
        loaded = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in loaded),
                "power_w_max": max(r["power"] for r in loaded),
                "samples": len(loaded), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------------------
# the oracle as a CPU baseline (test infrastructure, timed as it stands)
# ----------------------------------------------------------------------------------------

def oracle_sample(wl, rows: int, seed: int = 0, int4_absmax: bool = False):
    """Time the oracle's forward on `rows` tokens (full weight preparation included once)."""
    import oracle
    X = wl.activations(seed=seed, rows=rows)
    W = wl.weights(seed=seed)
    t0 = time.perf_counter()
    oracle.bitlinear_forward(X, W, wl.hadamard, wl.act_bits, int4_absmax=int4_absmax)
    return time.perf_counter() - t0


def oracle_baseline(wl, target_s: float = 12.0, int4_absmax: bool = False):
    """tokens/s of the oracle, measured on a bounded sample and scaled to one full step:
    t_step = t_prep + (M / r) * t_rows(r), tokens/s = M / t_step."""
    import oracle
    W = wl.weights()
    t0 = time.perf_counter()
    g = oracle.absmean_gamma(W)
    oracle.pack_ternary(oracle.ternarize(W, g))
    t_prep = time.perf_counter() - t0
    probe_rows = 16
    t_probe = oracle_sample(wl, probe_rows, int4_absmax=int4_absmax) - t_prep
    per_row = max(t_probe, 1e-6) / probe_rows
    rows = int(max(probe_rows, min(wl.M, (target_s - t_prep) / per_row)))
    t_rows = oracle_sample(wl, rows, int4_absmax=int4_absmax) - t_prep
    t_step = t_prep + (wl.M / rows) * max(t_rows, 1e-9)
    return {"value": wl.M / t_step, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"{rows} of {wl.M} token rows of {wl.name} through the C oracle "
                       f"(plain loops, fp64 FWHT, int64 GEMM, OpenMP over rows) plus one full "
                       f"weight ternarisation ({t_prep:.2f} s); per-step time scaled to all "
                       f"{wl.M} tokens: t_prep + (M/rows) * t_rows"),
            "t_prep_s": t_prep, "t_rows_s": t_rows, "rows": rows}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    import oracle
    int4_absmax = bool(getattr(args, "absmax4", False))
    budget_s = 150.0
    W = wl.weights()
    t0 = time.perf_counter()
    g = oracle.absmean_gamma(W)
    oracle.pack_ternary(oracle.ternarize(W, g))
    t_prep = time.perf_counter() - t0
    t_probe = oracle_sample(wl, 8, int4_absmax=int4_absmax) - t_prep
    per_row = max(t_probe, 1e-6) / 8
    steps_total = args.steps + args.warmup
    rows = int(max(1, min(wl.M, (budget_s / steps_total - t_prep) / per_row)))
    times = []
    for i in range(steps_total):
        X = wl.activations(seed=i, rows=rows)
        t0 = time.perf_counter()
        oracle.bitlinear_forward(X, W, wl.hadamard, wl.act_bits, int4_absmax=int4_absmax)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    t_rows = statistics.mean(times) - t_prep
    t_step = t_prep + (wl.M / rows) * max(t_rows, 1e-9)
    value = wl.M / t_step
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N,
                   "hadamard": wl.hadamard, "act_bits": wl.act_bits},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": (f"each step: {rows} token rows of {wl.name} through the C "
                                    f"oracle; weight ternarisation of the full W included once "
                                    f"per step; time scaled to all {wl.M} tokens")},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------------------

def aggregate_max(value: float, device) -> float:
    """Maximum of a per-rank float over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes its own tokens_per_rank
    tokens per step, and ms_per_step is the slowest rank's time (already max-reduced)."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def weight_ws_bytes(B, args, N: int, K: int) -> int:
    if args.rotate_weights:
        return B.bitnet_weight_workspace_bytes_rotated(N, K)
    return B.bitnet_weight_workspace_bytes(N, K)


def run_gpu(args, wl, rank, world, device):
    from bit_activation_linear_b200 import binding as B
    B.load_library()
    stream = torch.cuda.Stream(device)
    torch.cuda.set_stream(stream)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    M, K, N = wl.M, wl.K, wl.N
    code_bytes = M * K if wl.act_bits == 8 else M * K // 2
    per_copy = 2 * M * K + 2 * N * K + weight_bytes(N, K, args.base3) + code_bytes + 2 * M * N
    copies = max(2, math.ceil(2 * l2 / per_copy) + 1)

    # inputs: one batch per rank (seed = rank), rotated copies of X and W
    X0 = synth.to_torch_bf16(wl.activations(seed=rank))
    W0 = synth.to_torch_bf16(wl.weights(seed=rank))
    bufs = []
    for i in range(copies):
        X = X0.to(device, non_blocking=False).clone()
        W = W0.to(device).clone()
        Wp = torch.empty((N, weight_bytes(N, K, args.base3) // N), dtype=torch.uint8,
                         device=device)
        gamma = torch.empty(1, dtype=torch.float32, device=device)
        wws = torch.empty(max(weight_ws_bytes(B, args, N, K), 256), dtype=torch.uint8,
                          device=device)
        codes = torch.empty((M, K if wl.act_bits == 8 else K // 2), dtype=torch.uint8,
                            device=device)
        scales = torch.empty(M, dtype=torch.float32, device=device)
        rowsum = torch.empty(M, dtype=torch.int32, device=device)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        bufs.append(dict(X=X, W=W, Wp=Wp, gamma=gamma, wws=wws, codes=codes, scales=scales,
                         rowsum=rowsum, Y=Y))

    def weights(b):
        if args.rotate_weights:  # the weight half of the weight + activation rotation
            B.bitnet_quantize_pack_weights_rotated(b["W"], b["Wp"], b["gamma"], b["wws"])
            return
        if args.base3:
            B.bitnet_quantize_pack_weights_base3(b["W"], b["Wp"], b["gamma"], b["wws"])
            return
        B.bitnet_quantize_pack_weights(b["W"], b["Wp"], b["gamma"], b["wws"])

    # with --rmsnorm the token rows are RMS-normalised inside the quantiser (gain of ones
    # perturbed per feature, eps 1e-5)
    gain = None
    if args.rmsnorm:
        g = np.random.default_rng(7).uniform(0.5, 1.5, K).astype(np.float32)
        gain = synth.to_torch_bf16(synth.f32_to_bf16_bits(g)).to(device)

    def quant(b):
        if args.absmax4:  # the variant INT4 quantiser (absmax scale)
            B.bitnet_act_quant_absmax4(b["X"], wl.hadamard, b["codes"], b["scales"], b["rowsum"])
            return
        if gain is not None:
            B.bitnet_act_quant_norm(b["X"], gain, 1e-5, wl.hadamard, wl.act_bits, b["codes"],
                                    b["scales"], b["rowsum"])
            return
        B.bitnet_act_quant(b["X"], wl.hadamard, wl.act_bits, b["codes"], b["scales"],
                           b["rowsum"])

    act = {"none": 0, "relu2": B.ACT_RELU2, "swiglu": B.ACT_SWIGLU}[args.activation]

    def gemm(b):
        if args.base3:  # decode product on base-3 weights (Y's first M x N' elements)
            B.bitnet_ternary_gemv_base3(b["codes"], b["scales"], b["rowsum"], K, b["Wp"],
                                        b["gamma"], act, Y=b["Y"])
            return
        if act:  # the activation in the product's epilogue (Y's first M x N' elements)
            B.bitnet_ternary_gemm_act(b["codes"], b["scales"], b["rowsum"], K, b["Wp"],
                                      b["gamma"], wl.act_bits, act, Y=b["Y"])
            return
        B.bitnet_ternary_gemm(b["codes"], b["scales"], b["rowsum"], K, b["Wp"], b["gamma"],
                              wl.act_bits, want_acc=False, want_y=True, Y=b["Y"])

    phases = (("weights", weights), ("act_quant", quant), ("ternary_gemm", gemm))
    wstream = torch.cuda.Stream(device)

    def prep(b):
        # weight ternarisation and activation quantisation are independent: run them side by
        # side on two streams, join before the product
        wstream.wait_stream(stream)
        with torch.cuda.stream(wstream):
            weights(b)
        quant(b)
        stream.wait_stream(wstream)

    launches_before = B.bitnet_launch_count()
    for b in bufs:  # eager run once (sets kernel attributes, checks status)
        for _, fn in phases:
            fn(b)
    B.bitnet_sync_status(stream)
    launches_per_step = (B.bitnet_launch_count() - launches_before) // copies

    # One CUDA graph per input copy holds the whole step.  Timing-event nodes inside a graph
    # cost ~5 us per step on B200, so the timed loop replays event-free graphs, except for its
    # last n_timed (at most SAMPLES) steps: each of those replays its own copy of the step graph
    # whose product is bracketed by two timing events.  Those events give the product's live
    # duration inside the timed region, at a fixed cost of a few microseconds per run.
    SAMPLES = 4
    graphs = []
    for b in bufs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            prep(b)
            gemm(b)
        graphs.append(g)
    n_timed = min(args.steps, SAMPLES)
    first_timed = args.steps - n_timed
    timed = {}  # step index -> (graph, (start event, end event))
    for i in range(first_timed, args.steps):
        b = bufs[i % copies]
        gt = torch.cuda.CUDAGraph()
        ev = (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True))
        with torch.cuda.graph(gt, stream=stream):
            prep(b)
            ev[0].record(stream)
            gemm(b)
            ev[1].record(stream)
        timed[i] = (gt, ev)
    torch.cuda.synchronize(device)

    def step(i, sampled=False):
        if sampled:
            timed[i][0].replay()
        else:
            graphs[i % copies].replay()

    for i in range(args.warmup):
        step(i)
    for gt, _ in timed.values():  # first replays upload the sampled graphs outside the timed region
        gt.replay()
    torch.cuda.synchronize(device)
    B.bitnet_sync_status(stream)

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)

    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    barrier()
    torch.cuda.synchronize(device)
    # a short device sleep lets the host queue the first replays before the clock starts
    torch.cuda._sleep(int(2e7))
    t_start.record(stream)
    for i in range(args.steps):
        step(i, sampled=i >= first_timed)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    clocks = sampler.stop()
    B.bitnet_sync_status(stream)

    elapsed_ms = t_start.elapsed_time(t_end)
    # the product's duration in each sampled step (all inside the timed region)
    samples = [ev[0].elapsed_time(ev[1]) for _, ev in timed.values()]
    gemm_ms = statistics.mean(samples)
    elapsed_ms = aggregate_max(elapsed_ms, device)
    gemm_ms = aggregate_max(gemm_ms, device)
    # the two preparation phases run side by side inside the step; their own durations are
    # timed here, one phase at a time, on the same rotated inputs: one graph of many launches
    # (so the host's launch cost stays out of the figure), timed as a whole
    phase_ms = []
    for _, fn in phases[:2]:
        n_iso = copies * max(1, math.ceil(32 / copies))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_iso):
                fn(bufs[i % copies])
        g.replay()
        torch.cuda.synchronize(device)
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b2.record(stream)
        torch.cuda.synchronize(device)
        phase_ms.append(aggregate_max(a.elapsed_time(b2) / (reps * n_iso), device))
        del g
    phase_ms.append(gemm_ms)
    ms_per_step = elapsed_ms / args.steps

    # end to end through the public API: pinned host X and W in, Y out, every step
    e2e = None if args.no_e2e else run_e2e(args, wl, B, stream, device, X0, W0)

    if rank == 0:
        peaks, peak_kind = load_peaks()
        work = kernel_work(wl, args.base3, args.rotate_weights)
        int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16
        achieved = work["ternary_gemm_tc"]["ops"] / (gemm_ms * 1e-3) / 1e12
        hbm = peaks["hbm_gbs"]
        w_bytes = work["absmean_partials"]["bytes"] + work["ternarize_pack"]["bytes"]
        q_bytes = work["fwht_quant"]["bytes"]
        per_kernel = {
            "weights (absmean_partials + ternarize_pack; alone, outside the timed steps)": {
                "us": 1e3 * phase_ms[0], "bound": "hbm", "bytes": w_bytes,
                "achieved_gbs": w_bytes / (phase_ms[0] * 1e-3) / 1e9,
                "frac": w_bytes / (phase_ms[0] * 1e-3) / 1e9 / hbm},
            QUANT_KERNEL[B.bitnet_act_quant_plan(K, wl.hadamard, bool(args.rmsnorm))]
            + ("+rmsnorm" if args.rmsnorm else "") + ("+absmax4" if args.absmax4 else "")
            + " (alone, outside the timed steps)": {
                "us": 1e3 * phase_ms[1], "bound": "hbm", "bytes": q_bytes,
                "achieved_gbs": q_bytes / (phase_ms[1] * 1e-3) / 1e9,
                "frac": q_bytes / (phase_ms[1] * 1e-3) / 1e9 / hbm},
        }
        prod_bytes = work["ternary_gemm_tc"]["bytes"]
        prod_gbs = prod_bytes / (gemm_ms * 1e-3) / 1e9
        # the product kernel the library's plan query names for this shape
        path = B.bitnet_product_plan(M, K, N, wl.act_bits)[0]
        if path in (B.PATH_TC, B.PATH_TC_TMEM):
            tc_name = PRODUCT_KERNEL[path]
            per_kernel[tc_name] = {
                "us": 1e3 * gemm_ms, "bound": "tensor", "ops": work["ternary_gemm_tc"]["ops"],
                "achieved_tops": achieved, "frac": achieved / int8_peak}
            roofline = {"kernel": tc_name, "bound": "tensor",
                        "achieved": achieved, "peak": int8_peak, "unit": "TOPS",
                        "frac": achieved / int8_peak,
                        "traffic": ncu_traffic(tc_name + "_kernel", wl.name),
                        "ms_per_launch": gemm_ms,
                        "peak_source": f"{peak_kind} bf16 {peaks['bf16_tflops']} TFLOP/s x "
                                       f"{INT8_PER_BF16} (nominal int8:bf16 dense ratio)"}
        else:
            # a few tokens: the product streams the stored weights once (bytes = weights +
            # codes + bf16 Y), so HBM bounds it
            gemv = ("ternary_gemv_base3" if args.base3 else
                    PRODUCT_KERNEL.get(path, "ternary_gemv"))
            per_kernel[gemv] = {
                "us": 1e3 * gemm_ms, "bound": "hbm", "bytes": prod_bytes,
                "achieved_gbs": prod_gbs, "frac": prod_gbs / hbm,
                "ops": work["ternary_gemm_tc"]["ops"], "achieved_tops": achieved}
            roofline = {"kernel": gemv, "bound": "hbm", "achieved": prod_gbs, "peak": hbm,
                        "unit": "GB/s", "frac": prod_gbs / hbm,
                        "traffic": ncu_traffic(gemv + "_kernel", wl.name),
                        "ms_per_launch": gemm_ms,
                        "peak_source": f"{peak_kind} HBM copy bandwidth"}
        tokens_per_s = job_tokens_per_s(world, M, ms_per_step)
        line = {
            "metric": METRIC,
            "value": tokens_per_s,
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            # the activation code width; the tensor cores contract int8 operands (INT4 codes are
            # widened on chip) into int32 accumulators
            "dtype": f"int{wl.act_bits}",
            "data": "synthetic",
            "effective_tops": world * wl.ops / (ms_per_step * 1e-3) / 1e12,
            "config": {"workload": wl.name, "M": M, "K": K, "N": N, "hadamard": wl.hadamard,
                       "act_bits": wl.act_bits,
                       "contraction": "ternary weights x int8 operands (tcgen05 kind::i8), "
                                      "int32 accumulate, bf16 out",
                       "rmsnorm": bool(args.rmsnorm),
                       "activation": args.activation,
                       "weights": "base3" if args.base3 else "2bit",
                       "act_scale": ("absmean" if wl.act_bits == 4 and not args.absmax4
                                     else "absmax"),
                       "weight_rotation": bool(args.rotate_weights),
                       "tokens_per_rank": M,
                       "parallelism": f"replicas{world}",
                       "l2": f"inputs rotated over {copies} copies "
                             f"({copies * per_copy / 2**20:.0f} MiB > 2 x L2)"},
            "roofline": roofline,
            "kernels": per_kernel,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = oracle_baseline(wl, args.cpu_seconds, args.absmax4)
        elif not args.no_cpu_baseline:
            line["cpu_baseline"] = None
        print(json.dumps(line), flush=True)


def run_e2e(args, wl, B, stream, device, X0, W0):
    """The same step through the public API from pinned host memory: every step copies its X and
    W in, ternarises W, runs the forward and copies Y out.  Three buffer sets on a copy-in, a
    compute and a copy-out stream let step i+1's input copy and step i-1's output copy run while
    step i computes (the copies of every step stay inside the timed region)."""
    M, K, N = wl.M, wl.K, wl.N
    NB = 3
    act = {"none": 0, "relu2": B.ACT_RELU2, "swiglu": B.ACT_SWIGLU}[args.activation]
    n_out = N // 2 if act == B.ACT_SWIGLU else N
    Xh = X0.pin_memory()
    Wh = W0.pin_memory()
    sets = []
    for _ in range(NB):
        sets.append(dict(
            Yh=torch.empty((M, n_out), dtype=torch.bfloat16).pin_memory(),
            Xd=torch.empty_like(Xh, device=device), Wd=torch.empty_like(Wh, device=device),
            Yd=torch.empty((M, n_out), dtype=torch.bfloat16, device=device),
            Wp=torch.empty((N, weight_bytes(N, K, args.base3) // N), dtype=torch.uint8,
                           device=device),
            gamma=torch.empty(1, dtype=torch.float32, device=device),
            wws=torch.empty(max(weight_ws_bytes(B, args, N, K), 256), dtype=torch.uint8,
                            device=device),
            ws=torch.empty(max(B.bitnet_workspace_bytes(M, K, N, wl.act_bits), 256),
                           dtype=torch.uint8, device=device)))
    gain = None
    if args.rmsnorm:  # the same gain as the timed steps
        g = np.random.default_rng(7).uniform(0.5, 1.5, K).astype(np.float32)
        gain = synth.to_torch_bf16(synth.f32_to_bf16_bits(g)).to(device)

    def fwd(b):
        if args.absmax4:
            B.bitnet_bitlinear_forward_absmax4(b["Xd"], b["Wp"], b["gamma"], wl.hadamard,
                                               Y=b["Yd"], ws=b["ws"])
        elif args.base3:
            B.bitnet_bitlinear_forward_base3(b["Xd"], b["Wp"], b["gamma"], wl.hadamard, act,
                                             Y=b["Yd"], ws=b["ws"])
        elif gain is not None:
            B.bitnet_norm_bitlinear_forward(b["Xd"], gain, 1e-5, wl.hadamard, b["Wp"], b["gamma"],
                                            wl.act_bits, Y=b["Yd"], ws=b["ws"])
        elif act:
            B.bitnet_bitlinear_forward_act(b["Xd"], b["Wp"], b["gamma"], wl.act_bits, wl.hadamard,
                                           act, Y=b["Yd"], ws=b["ws"])
        elif wl.hadamard:
            B.bitnet_hbitlinear_forward(b["Xd"], b["Wp"], b["gamma"], wl.act_bits, Y=b["Yd"],
                                        ws=b["ws"])
        else:
            B.bitnet_bitlinear_forward(b["Xd"], b["Wp"], b["gamma"], wl.act_bits, Y=b["Yd"],
                                       ws=b["ws"])

    s_in, s_c, s_out = torch.cuda.Stream(device), stream, torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(NB)]
    ev_c = [torch.cuda.Event() for _ in range(NB)]
    ev_free = [torch.cuda.Event() for _ in range(NB)]
    used = [False] * NB

    def step(i):
        k = i % NB
        b = sets[k]
        with torch.cuda.stream(s_in):
            if used[k]:  # the previous step on these buffers has copied its Y out
                s_in.wait_event(ev_free[k])
            b["Xd"].copy_(Xh, non_blocking=True)
            b["Wd"].copy_(Wh, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_c):
            s_c.wait_event(ev_in[k])
            pack = (B.bitnet_quantize_pack_weights_base3 if args.base3
                    else B.bitnet_quantize_pack_weights_rotated if args.rotate_weights
                    else B.bitnet_quantize_pack_weights)
            pack(b["Wd"], b["Wp"], b["gamma"], b["wws"])
            fwd(b)
            ev_c[k].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[k])
            b["Yh"].copy_(b["Yd"], non_blocking=True)
            ev_free[k].record(s_out)
        used[k] = True

    n = max(3, min(args.steps, 100))
    for i in range(NB):
        step(i)
    torch.cuda.synchronize(device)
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(n):
        step(i)
    t1.record(s_out)
    torch.cuda.synchronize(device)
    barrier()
    ms = aggregate_max(t0.elapsed_time(t1) / n, device)
    world = dist.get_world_size() if dist.is_initialized() else 1
    return {"value": world * M / (ms * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": Xh.numel() * 2 + Wh.numel() * 2,
            "d2h_bytes_per_step": sets[0]["Yh"].numel() * 2, "ms_per_step": ms, "steps": n,
            "pipelined": f"{NB} buffer sets; copy-in, compute and copy-out streams"}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="down_7b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--activation", default="none", choices=["none", "relu2", "swiglu"],
                    help="activation in the product's epilogue (squared ReLU, SwiGLU)")
    ap.add_argument("--rmsnorm", action="store_true",
                    help="RMS-normalise the token rows inside the quantiser (fused prologue)")
    ap.add_argument("--base3", action="store_true",
                    help="store the weights five to a byte (base 3) for the decode product "
                         "(at most 8 tokens, INT8 activations)")
    ap.add_argument("--absmax4", action="store_true",
                    help="variant INT4 activation quantiser with a per-token absmax scale "
                         "(INT4 workloads)")
    ap.add_argument("--rotate-weights", action="store_true",
                    help="weight + activation Hadamard rotation: ternarise the rotated weight "
                         "rows (H-BitLinear workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (e.g. to keep a profiler capture small)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.WORKLOADS[args.workload]
    if args.absmax4 and (wl.act_bits != 4 or args.rmsnorm or args.base3 or
                         args.activation != "none"):
        ap.error("--absmax4 serves INT4 workloads, without --rmsnorm, --base3 or --activation")
    if args.rotate_weights and (not wl.hadamard or args.base3):
        ap.error("--rotate-weights serves H-BitLinear workloads with the 2-bit weights")
    if args.base3 and (wl.M > 8 or wl.act_bits != 8 or args.rmsnorm):
        ap.error("--base3 serves workloads of at most 8 tokens with INT8 activations, "
                 "without --rmsnorm")

    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=device)
    try:
        run_gpu(args, wl, rank, world, device)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
