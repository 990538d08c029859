#!/usr/bin/env python
"""Benchmark of the BitLinear W1.58A8 forward on B200.

Headline (one JSON line on rank 0): decode GEMV throughput in GB/s of packed
weight bytes. One step is a decode pass over a 2B-shaped model's BitLinear
projections: 30 layers x the four decode shapes (K=2560 -> N in {2560, 640,
6912}, K=6912 -> N=2560), one token (M=1), each layer with its own weight copy
(327 MB of packed weights per step, so every step streams its weights from HBM;
no L2 flush is needed). Each call quantises the token per absmax, runs the
ternary GEMV and dequantises to bf16. The step is captured once in a CUDA graph
and replayed.

Extras on the same line: batched decode (M = 4, 8, 16) and the 100B-class
shapes at M = 1 and 16, each rotating ceil(3 x L2 / matrix bytes) weight copies
so every call reads its weights from DRAM; prefill int8 TOPS (M = 512, 2048,
4096 at the 2B shapes, M = 2048 at the 100B-class shapes) against the int8 peak
measured here with torch._int_mm; the 30-layer FFN chain; every BitLinear of 30
decoder layers at one token (Q/K/V with the pre-norm, the output projection with
its subln, the FFN) beside the pages' whole-model CPU figure; the roofline of the
dominant kernel; the end-to-end number through the public API with host buffers;
the CPU oracle on all host cores and on one thread; and the SM clocks.

Multi-GPU: one process per GPU (torchrun); every rank runs the same independent
decode step on its own weights (weak scaling, no data-path collective); the
time is the max over ranks.

--impl reference times the CPU oracle (plain C) on a bounded sample of the same
workload on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W1.58A8 BitLinear: decode GEMV HBM GB/s (% peak); prefill int8 TOPS (% peak)"
DECODE_SHAPES = [(2560, 2560), (2560, 640), (2560, 6912), (6912, 2560)]  # (K, N)
LAYERS = 30
# the headline workload and its inputs, named the same way by both arms
WORKLOAD = ("decode_2b: M=1, (K,N) in {(2560,2560),(2560,640),(2560,6912),(6912,2560)}, "
            "30 layer copies each, 120 BitLinear calls per step")
DATA = "synthetic (seeded N(0,0.02^2) weights, N(0,1) activations with 1% x20 outlier channels)"
# DRAM bytes (read + write) per launch of the decode GEMV, averaged over the
# step's four shapes: ncu captures of one launch per shape read 1,664,512 +
# 435,712 + 4,449,792 + 4,460,288 bytes (0 written) for 2,723,840 packed bytes
# per launch on average (x 1.0106). Set to None whenever the kernel changes until
# a new capture is taken.
GEMV_TRAFFIC_PER_LAUNCH = 2752576
# The pages' only latency figure, quoted beside the whole-decoder-layer number as
# context (not a target): whole-model CPU decode, ms per output token.
PAGES_CPU_MS_PER_TOKEN = 29.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense int8 (= fp8) rate over dense bf16 on B200


def measure_int8_peak(torch, dev, sustained_s: float = 3.0):
    """Dense int8 tensor throughput of this GPU as cuBLASLt gives it: torch._int_mm
    at 8192^3 (2 N^3 ops), best of 10 single calls (burst) and back to back for
    `sustained_s` seconds (sustained). None if the call is unavailable."""
    n = 8192
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t().contiguous().t()
        torch._int_mm(a, b)
        torch.cuda.synchronize()
    except (RuntimeError, AttributeError) as e:
        return {"available": False, "why": str(e).splitlines()[0][:200]}
    ops = 2.0 * n ** 3
    best = float("inf")
    for _ in range(10):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    reps = max(1, int(sustained_s / (best * 1e-3)))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        torch._int_mm(a, b)
    e1.record()
    torch.cuda.synchronize()
    sust_ms = e0.elapsed_time(e1) / reps
    del a, b
    torch.cuda.empty_cache()
    return {"available": True, "burst_tops": round(ops / (best * 1e-3) / 1e12, 1),
            "sustained_tops": round(ops / (sust_ms * 1e-3) / 1e12, 1), "n": n, "reps_sustained": reps,
            "how": "torch._int_mm int8 x int8 -> int32, 8192^3: best of 10 (burst); back to back (sustained)"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_ops(torch, dist, world: int, device):
    """Barrier and max-over-ranks of a float, the two collectives the timing
    uses (NCCL on the GPUs; the same code runs under gloo on the CPU in tests)."""
    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return barrier, max_over_ranks


def whole_job_gbs(world: int, step_bytes: int, steps: int, ms_total: float) -> float:
    """Aggregate throughput: every rank streams step_bytes per step (weak
    scaling); the time is the slowest rank's."""
    return world * step_bytes * steps / (ms_total * 1e-3) / 1e9


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [ln.strip().split(",") for ln in self.file.read().splitlines() if ln.strip()]
        self.file.close()
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- ours

def run_ours(args):
    import torch
    import torch.distributed as dist

    import bitlinear_w1_a8_02_b200 as bl
    from bitlinear_w1_a8_02_b200 import synth

    rank, world, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks, peak_kind = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    int8_from_bf16 = float(peaks["bf16_tflops"]) * INT8_PER_BF16
    int8_from_bf16_sust = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * INT8_PER_BF16
    int8_meas = measure_int8_peak(torch, dev) if (rank == 0 and not args.no_extras) else {"available": False,
                                                                                           "why": "not measured"}
    if int8_meas.get("available"):
        int8_peak, int8_peak_sust = int8_meas["burst_tops"], int8_meas["sustained_tops"]
        int8_kind = "measured on this GPU (torch._int_mm, 8192^3)"
    else:
        int8_peak, int8_peak_sust = int8_from_bf16, int8_from_bf16_sust
        int8_kind = peak_kind + " bf16 x 2 (the nominal dense int8 / bf16 ratio)"

    barrier, max_over_ranks = rank_ops(torch, dist, world, dev)

    # ---- decode weights: 30 copies of each of the four shapes, packed on device
    weights = []  # weights[layer][shape] = (Wp, gamma)
    for layer in range(LAYERS):
        row = []
        for si, (K, N) in enumerate(DECODE_SHAPES):
            W = synth.weights(N, K, synth.SIGMA_2B, synth.weight_seed(si, layer) + 7919 * rank,
                              device=dev)
            row.append(bl.pack_weights(W))
            del W
        weights.append(row)
    xs = [synth.activations(1, K, seed=1, outliers=True, device=dev) for K, _ in DECODE_SHAPES]
    ys = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for _, N in DECODE_SHAPES]
    ws = torch.empty(max(bl.workspace_bytes(bl.BL_OP_FORWARD, 16, N, K) for K, N in DECODE_SHAPES),
                     dtype=torch.uint8, device=dev)
    step_bytes = LAYERS * sum(K * N // 4 for K, N in DECODE_SHAPES)
    kernels_per_call = 1  # M = 1: the GEMV quantises x itself

    def step():
        for layer in range(LAYERS):
            for si in range(len(DECODE_SHAPES)):
                Wp, g = weights[layer][si]
                bl.forward(Wp, g, xs[si], out=ys[si], ws=ws)

    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        step()  # warm the code paths before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    ev0.record(cur)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(cur)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1))
    ms_step = ms_total / args.steps
    value = whole_job_gbs(world, step_bytes, args.steps, ms_total)

    # ---- dominant kernel: the decode GEMV. At M = 1 each forward call is one
    # kernel (quantisation fused); consecutive calls overlap through programmatic
    # dependent launch, so the average launch duration is the timed region's
    # device time over the launches in it (CUDA events on the launching stream).
    calls = args.steps * LAYERS * len(DECODE_SHAPES)
    per_launch_s = (ev0.elapsed_time(ev1) * 1e-3) / calls
    achieved = (step_bytes / (LAYERS * len(DECODE_SHAPES))) / per_launch_s / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "traffic": GEMV_TRAFFIC_PER_LAUNCH,
                "kernel": "gemv_mma_kernel<1,SRC_X,0,dp4a,0,BIG=1|2> (register quantiser + ternary GEMV + dequant, "
                          "one launch per call)",
                "us_per_launch": round(per_launch_s * 1e6, 3),
                "bytes_per_launch": step_bytes // (LAYERS * len(DECODE_SHAPES)),
                "peak_kind": peak_kind}

    # the tensor-parallel FFN runs on every rank (its collectives need them all)
    tp_extra = run_tp_extra(bl, synth, dev, rank, world, barrier, max_over_ranks) if world > 1 else None
    extras = {}
    if rank == 0 and not args.no_extras:
        extras = run_extras(args, bl, synth, dev, hbm_peak, int8_peak)
    if tp_extra is not None:
        extras["ffn_tp"] = tp_extra

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, bl, dev, graph, xs, ys, step_bytes, world, barrier, max_over_ranks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(weights, xs, bl, budget_s=args.cpu_seconds)

    del graph
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": DATA,
        "config": {"workload": WORKLOAD,
                   "M": 1, "layers": LAYERS, "calls_per_step": LAYERS * len(DECODE_SHAPES),
                   "packed_bytes_per_step": step_bytes,
                   "l2": "inputs larger than L2: 327 MB of packed weights per step vs 126 MB L2",
                   "launch": "cuda_graph replay of the 120 calls", "parallelism": f"replicas x{world}"},
        "hbm_frac": round(value / world / hbm_peak, 4),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * LAYERS * len(DECODE_SHAPES) * kernels_per_call,
        "clocks": clk,
        "peaks": {"hbm_gbs": hbm_peak, "hbm_kind": peak_kind, "int8_tops_burst": int8_peak,
                  "int8_tops_sustained": int8_peak_sust, "int8_kind": int8_kind, "int8_measured": int8_meas,
                  "int8_cross_check_bf16x2": {"burst": round(int8_from_bf16, 1),
                                              "sustained": round(int8_from_bf16_sust, 1)}},
        "extras": extras,
    }
    print(json.dumps(line), flush=True)


def time_graph(torch, fn, reps: int, warm: int = 3):
    """Capture fn in a CUDA graph; return mean ms per replay (events)."""
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    del g
    return ms


def cold_copies(l2_bytes: int, matrix_bytes: int) -> int:
    """Weight copies to rotate so that every call reads its weights from DRAM:
    ceil(3 x L2 / bytes of one copy), at least 2."""
    return max(2, -(-3 * l2_bytes // matrix_bytes))


def run_extras(args, bl, synth, dev, hbm_peak, int8_peak):
    import torch

    out = {}
    l2 = int(torch.cuda.get_device_properties(dev).L2_cache_size)
    out["l2_bytes"] = l2
    # Batched decode at the 2B FFN shapes: ceil(3 L2 / 4.42 MB) rotating weight
    # copies per shape (about 90 on a 126 MB L2), so every call streams its
    # weights from DRAM; the codes of x and the outputs stay in L2.
    shapes = [(2560, 6912), (6912, 2560)]
    batched = {}
    for si, (K, N) in enumerate(shapes):
        ncp = cold_copies(l2, K * N // 4)
        cps = [bl.pack_weights(synth.weights(N, K, synth.SIGMA_2B, 50 + 1000 * si + c, device=dev))
               for c in range(ncp)]
        for M in (4, 8, 16):
            x = synth.activations(M, K, seed=M, device=dev)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bl.workspace_bytes(bl.BL_OP_FORWARD, M, N, K), dtype=torch.uint8, device=dev)

            def fn():
                for Wp, g in cps:
                    bl.forward(Wp, g, x, out=y, ws=ws)
            ms = time_graph(torch, fn, reps=10) / len(cps)
            gbs = K * N / 4 / (ms * 1e-3) / 1e9
            batched.setdefault(f"M{M}", {})[f"{K}x{N}"] = {
                "us_per_call": round(ms * 1e3, 2), "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm_peak, 4),
                "copies": len(cps), "rotated_mb": round(len(cps) * K * N / 4 / 1e6, 1)}
        del cps
    out["batched_decode_2b"] = batched

    packs = {(K, N): bl.pack_weights(synth.weights(N, K, synth.SIGMA_2B, 50 + 1000 * si, device=dev))
             for si, (K, N) in enumerate(shapes)}
    prefill = {}
    for M in (512, 2048, 4096):
        per = {}
        for K, N in shapes:
            x = synth.activations(M, K, seed=M, device=dev)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bl.workspace_bytes(bl.BL_OP_FORWARD, M, N, K), dtype=torch.uint8, device=dev)
            Wp, g = packs[(K, N)]

            def fn():
                bl.forward(Wp, g, x, out=y, ws=ws)
            ms = time_graph(torch, fn, reps=10)
            tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
            per[f"{K}x{N}"] = {"ms": round(ms, 4), "tops": round(tops, 1),
                               "frac_int8_peak": round(tops / int8_peak, 4)}
        prefill[f"M{M}"] = per
    out["prefill_2b"] = prefill
    del packs

    # 100B-class shapes: M = 1 and 16 rotate ceil(3 L2 / 58.7 MB) copies (7 on a
    # 126 MB L2: 411 MB per shape) so every call reads its weights from DRAM;
    # M = 2048 is the tensor-core GEMM on one copy.
    big = {}
    for K, N in ((8192, 28672), (28672, 8192)):
        ncp = cold_copies(l2, K * N // 4)
        cps = [bl.pack_weights(synth.weights(N, K, synth.SIGMA_100B, 90 + c, device=dev)) for c in range(ncp)]
        torch.cuda.empty_cache()
        for M in (1, 16):
            x = synth.activations(M, K, seed=M, device=dev)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bl.workspace_bytes(bl.BL_OP_FORWARD, M, N, K), dtype=torch.uint8, device=dev)

            def fn():
                for Wp, g in cps:
                    bl.forward(Wp, g, x, out=y, ws=ws)
            ms = time_graph(torch, fn, reps=10) / len(cps)
            gbs = K * N / 4 / (ms * 1e-3) / 1e9
            big[f"{K}x{N}_M{M}"] = {"us_per_call": round(ms * 1e3, 2), "gbs": round(gbs, 1),
                                    "hbm_frac": round(gbs / hbm_peak, 4), "copies": len(cps),
                                    "rotated_mb": round(len(cps) * K * N / 4 / 1e6, 1)}
        M = 2048
        x = synth.activations(M, K, seed=M, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(bl.workspace_bytes(bl.BL_OP_FORWARD, M, N, K), dtype=torch.uint8, device=dev)
        Wp, g = cps[0]

        def fn():
            bl.forward(Wp, g, x, out=y, ws=ws)
        ms = time_graph(torch, fn, reps=5)
        tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        big[f"{K}x{N}_M{M}"] = {"ms": round(ms, 4), "tops": round(tops, 1),
                                "frac_int8_peak": round(tops / int8_peak, 4)}
        del cps, x, y, ws
        torch.cuda.empty_cache()
    out["stress_100b"] = big

    # The three M <= 16 kernels side by side (bitlinear_set_gemv_kernel): the
    # streamed dp4a / mma.sync GEMV (the automatic choice), the tensor-core GEMV
    # with the weights in TMEM, and the lookup-table GEMV after the bitnet.cpp
    # CPU kernels; cold weights as above.
    kinds = (("stream", bl.BL_GEMV_STREAM), ("tensor", bl.BL_GEMV_TENSOR), ("lut", bl.BL_GEMV_LUT))
    compared = {}
    for K, N, sigma in ((2560, 6912, synth.SIGMA_2B), (8192, 28672, synth.SIGMA_100B)):
        ncp = cold_copies(l2, K * N // 4)
        cps = [bl.pack_weights(synth.weights(N, K, sigma, 70 + c, device=dev)) for c in range(ncp)]
        for M in (1, 4, 16):
            x = synth.activations(M, K, seed=M, device=dev)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(bl.workspace_bytes(bl.BL_OP_FORWARD, M, N, K), dtype=torch.uint8, device=dev)
            row = {}
            for name, kind in kinds:
                with bl.gemv_kernel(kind):
                    def fn():
                        for Wp, g in cps:
                            bl.forward(Wp, g, x, out=y, ws=ws)
                    ms = time_graph(torch, fn, reps=3) / len(cps)
                gbs = K * N / 4 / (ms * 1e-3) / 1e9
                row[name] = {"us_per_call": round(ms * 1e3, 2), "hbm_frac": round(gbs / hbm_peak, 4)}
            compared[f"{K}x{N}_M{M}"] = row
        del cps
        torch.cuda.empty_cache()
    out["gemv_kernels_compared"] = compared

    # FFN chain: 30 layers, d=2560, f=6912, residual add
    d, f = 2560, 6912
    layers = []
    for layer in range(LAYERS):
        sg, su, sd = synth.ffn_layer_seeds(layer)
        layers.append([bl.pack_weights(synth.weights(N, K, synth.SIGMA_2B, seed, device=dev))
                       for N, K, seed in ((f, d, sg), (f, d, su), (d, f, sd))])
    ffn = {}
    for M in (1, 512):
        h0 = synth.activations(M, d, seed=1, outliers=False, device=dev)
        bufs = [torch.empty_like(h0), torch.empty_like(h0)]
        ws = torch.empty(bl.workspace_bytes(bl.BL_OP_FFN, M, f, d), dtype=torch.uint8, device=dev)

        def fn():
            h = h0
            for li, (g_, u_, d_) in enumerate(layers):
                o = bufs[li % 2]
                bl.ffn(g_[0], g_[1], u_[0], u_[1], d_[0], d_[1], h, residual=h, out=o, ws=ws)
                h = o
        ms = time_graph(torch, fn, reps=5)
        wbytes = LAYERS * 3 * d * f / 4
        ent = {"ms_30_layers": round(ms, 4), "packed_gbs": round(wbytes / (ms * 1e-3) / 1e9, 1)}
        if M > 1:
            tops = 2.0 * M * 3 * d * f * LAYERS / (ms * 1e-3) / 1e12
            ent["tops"] = round(tops, 1)
            ent["frac_int8_peak"] = round(tops / int8_peak, 4)
        ffn[f"M{M}"] = ent
    out["ffn_2b_30_layers"] = ffn

    # Every BitLinear of a 2B-shaped decoder layer, 30 layers, one token per step:
    # Q/K/V in one call with the block's pre-norm, the output projection with its
    # subln and the residual, then the FFN. The attention itself (RoPE, softmax,
    # the KV cache) is not part of this library: the output projection reads a
    # fixed synthetic attention output.
    qkv_rows = [2560, 640, 640]
    dec = []
    for layer in range(LAYERS):
        qkv = [bl.pack_weights(synth.weights(n, d, synth.SIGMA_2B, 5000 + 10 * layer + i, device=dev))
               for i, n in enumerate(qkv_rows)]
        o_w = bl.pack_weights(synth.weights(d, d, synth.SIGMA_2B, 5000 + 10 * layer + 3, device=dev))
        dec.append((torch.cat([w for w, _ in qkv]), torch.cat([g_.reshape(1) for _, g_ in qkv]),
                    o_w[0], o_w[1].reshape(1)))
    linears = {}
    for M in (1,):
        h0 = synth.activations(M, d, seed=3, outliers=False, device=dev)
        attn = synth.activations(M, d, seed=4, outliers=False, device=dev)
        yqkv = torch.empty((M, sum(qkv_rows)), dtype=torch.bfloat16, device=dev)
        hbuf = [torch.empty_like(h0) for _ in range(3)]
        ws_f = torch.empty(bl.workspace_bytes(bl.BL_OP_FFN, M, f, d), dtype=torch.uint8, device=dev)
        ws_q = torch.empty(bl.workspace_bytes(bl.BL_OP_FORWARD, M, sum(qkv_rows), d), dtype=torch.uint8,
                           device=dev)

        def fn():
            h = h0
            for li in range(LAYERS):
                wq, gq, wo, go = dec[li]
                g_, u_, d_ = layers[li]
                bl.forward_ex(wq, gq, qkv_rows, h, rmsnorm=True, out=yqkv, ws=ws_q)
                h1 = hbuf[(2 * li) % 3]
                bl.forward_ex(wo, go, [d], attn, rmsnorm=True, residual=h, out=h1, ws=ws_q)
                h2 = hbuf[(2 * li + 1) % 3]
                bl.ffn(g_[0], g_[1], u_[0], u_[1], d_[0], d_[1], h1, residual=h1, out=h2, ws=ws_f)
                h = h2
        ms = time_graph(torch, fn, reps=5)
        wbytes = LAYERS * (sum(qkv_rows) * d + d * d + 3 * d * f) / 4
        linears[f"M{M}"] = {"ms_30_layers": round(ms, 4), "us_per_layer": round(ms * 1e3 / LAYERS, 2),
                            "launches_per_layer": 4, "packed_gbs": round(wbytes / (ms * 1e-3) / 1e9, 1),
                            "pages_context": {
                                "ms_per_token": PAGES_CPU_MS_PER_TOKEN,
                                "what": "whole 2B model per output token on a laptop CPU (i7-13800H, 8 threads, "
                                        "bitnet.cpp); includes attention, embeddings and the LM head, which "
                                        "this number does not",
                                "source": "paper card 'BitNet b1.58 2B4T Technical Report', Evidence, Table 1"}}
    out["decoder_linears_2b_30_layers"] = linears
    del layers, dec
    torch.cuda.empty_cache()
    return out


def run_tp_extra(bl, synth, dev, rank, world, barrier, max_over_ranks, layers: int = 4):
    """The FFN sub-layer split over the ranks (bitlinear_w1_a8_02_b200.tp): d = 2560,
    f = 6912, each rank owning its shard of the hidden width, NCCL exchanges of the
    subln statistics and the int32 accumulators; `layers` layers chained, at
    M = 1 and 512. Device time on each rank, the max over ranks reported."""
    import torch

    from bitlinear_w1_a8_02_b200 import tp

    d, f = 2560, 6912
    c0, c1 = tp.shard_range(f, world, rank)
    shards = []
    for layer in range(layers):
        sg, su, sd = synth.ffn_layer_seeds(layer)
        Wg = synth.weights(f, d, synth.SIGMA_2B, sg, device=dev)
        Wu = synth.weights(f, d, synth.SIGMA_2B, su, device=dev)
        Wd = synth.weights(d, f, synth.SIGMA_2B, sd, device=dev)
        shards.append(tp.pack_ffn_shard(Wg[c0:c1].contiguous(), Wu[c0:c1].contiguous(), Wd[:, c0:c1].contiguous(),
                                        f, c0, c1))
        del Wg, Wu, Wd
    out = {"world": world, "shard_columns": [c0, c1], "layers": layers}
    for M in (1, 512):
        h0 = synth.activations(M, d, seed=1, outliers=False, device=dev)

        def run():
            h = h0
            for sh in shards:
                h = tp.ffn_tp(sh, h, residual=h)
            return h
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        barrier()
        reps = 10
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            run()
        b.record()
        torch.cuda.synchronize()
        ms = max_over_ranks(a.elapsed_time(b) / reps)
        out[f"M{M}"] = {"ms_per_step": round(ms, 4), "us_per_layer": round(ms * 1e3 / layers, 2)}
    torch.cuda.synchronize()
    barrier()
    return out


def run_e2e(args, bl, dev, graph, xs, ys, step_bytes, world, barrier, max_over_ranks):
    """Each step: pinned host -> device copy of the step's activations, the
    captured public-API calls, device -> host copy of the step's outputs."""
    import torch

    h_in = [x.detach().cpu().pin_memory() for x in xs]
    h_out = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in ys]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    cur = torch.cuda.current_stream(dev)

    def one():
        for hx, dx in zip(h_in, xs):
            dx.copy_(hx, non_blocking=True)
        graph.replay()
        for hy, dy in zip(h_out, ys):
            hy.copy_(dy, non_blocking=True)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(cur)
    for _ in range(args.steps):
        one()
    b.record(cur)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(a.elapsed_time(b))
    value = world * step_bytes * args.steps / (ms * 1e-3) / 1e9
    return {"value": round(value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms / args.steps, 5)}


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(weights, xs, bl, budget_s: float):
    """The oracle (as it stands) on a bounded sample of the decode step: whole
    layers of the four shapes, one after another, until the budget is spent;
    once on every host core (the reported value) and once on one thread."""
    import numpy as np

    import oracle

    bits = [x.cpu().view(__import__("torch").int16).numpy().view(np.uint16) for x in xs]
    host = [[(Wp.cpu().numpy(), float(g.cpu().item())) for Wp, g in row] for row in weights]

    def run(threads: int, seconds: float):
        used = oracle.set_threads(threads)
        done_bytes, n_layers = 0, 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            row = host[n_layers % LAYERS]
            for (Wp, g), xb in zip(row, bits):
                oracle.forward(Wp, g, xb)
                done_bytes += Wp.size
            n_layers += 1
        dt = time.perf_counter() - t0
        return used, done_bytes, n_layers, dt

    all_cores = os.cpu_count() or 1
    used, nbytes, nl, dt = run(all_cores, budget_s)
    used1, nbytes1, nl1, dt1 = run(1, budget_s / 2)
    oracle.set_threads(all_cores)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
            "sample": f"{nl} layers of the decode step, cycling over its 30 layers "
                      f"(4 shapes each, M=1): {nbytes} packed bytes in {dt:.2f} s",
            "cpu_model": cpu_model(),
            "single_thread": {"value": round(nbytes1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": used1,
                              "sample": f"{nl1} layers, {nbytes1} packed bytes in {dt1:.2f} s"}}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The CPU oracle on the same workload: each step is a bounded sample (one
    layer of the four decode shapes, M=1); value in packed GB/s."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    from bitlinear_w1_a8_02_b200 import synth

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    packed = []
    for si, (K, N) in enumerate(DECODE_SHAPES):
        W = synth.weights(N, K, synth.SIGMA_2B, synth.weight_seed(si, 0))
        packed.append(oracle.pack_weights(bits(W)))
    xs = [bits(synth.activations(1, K, seed=1, outliers=True)) for K, _ in DECODE_SHAPES]
    step_bytes = sum(Wp.size for Wp, _ in packed)

    def step():
        for (Wp, g), x in zip(packed, xs):
            oracle.forward(Wp, g, x)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = step_bytes * args.steps / dt / 1e9
    cores = oracle.set_threads(0)
    sample = f"one layer of the four decode shapes per step (M=1), of the 30-layer step; {cpu_model()}"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": DATA,
        "config": {"workload": WORKLOAD, "M": 1, "layers": LAYERS,
                   "calls_per_step": LAYERS * len(DECODE_SHAPES), "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


PROFILE_CASES = {
    # name: (K, N, M) of one forward call; used for ncu captures of one kernel
    "gemv_2b": (2560, 6912, 1),
    "gemv_2b_2560": (2560, 2560, 1),
    "gemv_2b_640": (2560, 640, 1),
    "gemv_2b_down": (6912, 2560, 1),
    "gemv_2b_m16": (2560, 6912, 16),
    "gemv_100b": (8192, 28672, 1),
    "gemv_100b_m16": (8192, 28672, 16),
    "gemv_100b_down_m16": (28672, 8192, 16),
    "gemm_2b": (2560, 6912, 4096),
    "gemm_2b_down": (6912, 2560, 4096),
}


def run_profile_case(name: str, reps: int, gemv_kernel: int = 0):
    """Run one forward call `reps` times (after packing); for ncu -k/-s/-c.
    gemv_kernel selects the M <= 16 kernel (bitlinear_set_gemv_kernel)."""
    import torch

    import bitlinear_w1_a8_02_b200 as bl
    from bitlinear_w1_a8_02_b200 import synth

    K, N, M = PROFILE_CASES[name]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sigma = synth.SIGMA_100B if K * N > 10 ** 8 else synth.SIGMA_2B
    Wp, g = bl.pack_weights(synth.weights(N, K, sigma, seed=1, device=dev))
    x = synth.activations(M, K, seed=2, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(bl.workspace_bytes(bl.BL_OP_FORWARD, M, N, K), dtype=torch.uint8, device=dev)
    with bl.gemv_kernel(gemv_kernel):
        for _ in range(reps):
            bl.forward(Wp, g, x, out=y, ws=ws)
    torch.cuda.synchronize()
    assert bl.get_device_error() == 0
    print(f"profile case {name}: K={K} N={N} M={M}, {reps} calls, GEMV kernel {gemv_kernel}", flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="run one forward call repeatedly for an ncu capture, then exit")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--gemv-kernel", type=int, default=0,
                    help="M <= 16 kernel for --profile-case: 0 auto, 1 streamed, 2 tensor-core")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case, args.reps, args.gemv_kernel)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
