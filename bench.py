#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear hot path on B200.

One step = NF4 quantisation of the frozen weight (absmax per 64, FP8 double
quantisation per 256) + forward (U = X A^T; Y = X W'^T + s U B^T with W'
dequantised inside the GEMM) + backward (dU, dB, dX, dA), all through the
library's C ABI, on the LLaMA-7B-shaped attention projection: W 4096x4096,
4 x 1024 tokens, LoRA r=64, alpha=16, synthetic seeded inputs.

value = algorithmic fwd+bwd FLOPs (4MNK + 6MKr + 6MNr) / device time per
step, summed over all ranks (each rank runs its own batch: weak scaling; the
adapter gradients dA, dB are summed across ranks with NCCL, the one exchange
of data-parallel training).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s (% bf16 peak); NF4 quant/dequant HBM GB/s"
WORKLOAD = "c2"
WORKLOAD_NAME = "LLaMA-7B attention projection: W 4096x4096 NF4/64 + FP8/256, 4x1024 tokens, r=64, alpha=16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# Per-launch DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the
# tensor-core kernels of this workload, from one ncu capture of the CTA-pair
# kernels on this workload (c2 forward and dX); emptied whenever those kernels change.
NCU_TRAFFIC_BYTES = {"fused_fwd": 43.871232e6 + 3.50336e6, "fused_dx": 43.949312e6 + 2.96576e6}


def flops_fwd_bwd(M, N, K, r):
    return 4 * M * N * K + 6 * M * K * r + 6 * M * N * r


def kernel_flops(name, M, N, K, r):
    """Algorithmic FLOPs of one launch of the tensor-core kernels."""
    return {"fused_fwd": 2 * M * N * K + 2 * M * N * r, "fused_dx": 2 * M * N * K + 2 * M * K * r,
            "lora_down": 2 * M * K * r, "lora_du": 2 * M * N * r, "lora_db": 2 * M * N * r,
            "lora_da": 2 * M * K * r}.get(name)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
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
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        loaded = [v for v in sm if v > 0.5 * smax] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ CPU baseline

def cpu_oracle_sample(reps=1, m_s=512, n_s=2048, seed=0):
    """Time the oracle on a bounded sample of the workload.

    Sample: the first n_s output features of the 4096x4096 weight and m_s
    tokens: NF4-quantise + dequantise those weight rows, then the fp64
    forward and backward on (m_s tokens, n_s features, K=4096, r=64).
    Returns (TFLOP/s on the sample's fwd+bwd FLOPs, seconds, description).
    """
    import synth
    from oracle import linear as ol
    from oracle import nf4
    wl = synth.WORKLOADS[WORKLOAD]
    lin = wl.linears[0]
    d = synth.linear_inputs(synth.Linear("sample", n_s, lin.k_in), m_s, wl.r, seed)
    b = {k: synth.bf16_bits(v) for k, v in d.items()}
    t0 = time.perf_counter()
    for _ in range(reps):
        codes, c8, s2 = nf4.quantize(b["W"].reshape(-1))
        wd = nf4.dequantize(codes, c8, s2, b["W"].size).reshape(b["W"].shape)
        ol.linear_fwd(b["X"], wd, b["A"], b["B"], wl.s)
        ol.linear_bwd(b["dY"], b["X"], wd, b["A"], b["B"], wl.s)
    dt = time.perf_counter() - t0
    fl = flops_fwd_bwd(m_s, n_s, lin.k_in, wl.r) * reps
    desc = (f"{reps} x (quantize+dequantize {n_s}x{lin.k_in} weight rows, fp64 fwd+bwd on {m_s} tokens x "
            f"{n_s} features x K={lin.k_in}, r={wl.r})")
    return fl / dt / 1e12, dt, desc


def cpu_cores():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"), default=n)
    except Exception:
        blas = n
    return n, blas


# ------------------------------------------------------------------ arms

def c5_forward_sweep(lib, synth, torch, dev, flush, peaks, reps=5):
    """Forward of the 65B-shaped 8192<->22016 linears over M in {1,16,128,2048,16384}.

    Per case: algorithmic bytes 0.5159 N K + 2 M K + 2 M N + 2 r (K + N) and
    FLOPs 2 M N K + 2 M K r + 2 M N r, over the mean device time of the
    forward call (L2 flushed before each run).
    """
    out = {}
    r, s = 64, 0.25
    for lin in synth.C5_SHAPES:
        N, K = lin.n_out, lin.k_in
        w = synth.weight_bf16(N, K, seed=650 + N, device=dev)
        W = lib.quantize_weight(w)
        del w
        A = synth.normal_bf16((r, K), 1.0 / K, seed=651, device=dev)
        B = synth.normal_bf16((N, r), synth.B_STD, seed=652, device=dev)
        for M in synth.C5_M:
            X = synth.normal_bf16((M, K), 1.0, seed=653 + M, device=dev)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            U = torch.empty((M, r), dtype=torch.float32, device=dev)
            ws = torch.empty(max(lib.qlora_fwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)
            for _ in range(2):
                lib.qlora_linear_fwd(X, W, A, B, s, Y=Y, U=U, ws=ws)
            ts = []
            for _ in range(reps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                lib.qlora_linear_fwd(X, W, A, B, s, Y=Y, U=U, ws=ws)
                e1.record()
                e1.synchronize()
                ts.append(e0.elapsed_time(e1))
            ms = float(np.mean(ts))
            # one more call with per-kernel event brackets (not part of ms)
            flush.zero_()
            lib.profile_enable(True)
            lib.qlora_linear_fwd(X, W, A, B, s, Y=Y, U=U, ws=ws)
            torch.cuda.synchronize()
            lib.profile_enable(False)
            kern = {}
            for name, kms in lib.profile_collect():
                kern[name] = round(kern.get(name, 0.0) + kms, 5)
            byts = 0.51587 * N * K + 2 * M * K + 2 * M * N + 2 * r * (K + N)
            fl = 2 * M * N * K + 2 * M * K * r + 2 * M * N * r
            out[f"{lin.name}_{N}x{K}_M{M}"] = {
                "ms": round(ms, 5), "tflops": round(fl / ms / 1e9, 2), "gbs": round(byts / ms / 1e6, 1),
                "hbm_frac": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4),
                "tensor_frac": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4), "kernels_ms": kern}
            del X, Y, U, ws
        del W, A, B
    return out


def c1_graph_timing(lib, synth, torch, dev, reps=200):
    """c1 step (quantize + fwd + bwd, 512x512, 64 tokens, r=16) eager vs one CUDA graph.

    The step is launch-bound at this size; the graph holds the library's
    kernels (programmatic launches and the side-stream fork/join included).
    Outputs of a replay are compared bit for bit with an eager step.
    """
    wl = synth.WORKLOADS["c1"]
    lin = wl.linears[0]
    M, N, K, r, s = wl.m_tokens, lin.n_out, lin.k_in, wl.r, wl.s
    g = {k: v.to(dev) for k, v in synth.linear_inputs(lin, M, r, 0).items()}
    nc, nb, ns = lib.nf4_sizes(N * K)
    codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    c8 = torch.empty(nb, dtype=torch.uint8, device=dev)
    s2 = torch.empty(ns, dtype=torch.float32, device=dev)
    W = lib.NF4Weight(codes, c8, s2, N, K)
    out = {"Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
           "U": torch.empty((M, r), dtype=torch.float32, device=dev),
           "dX": torch.empty((M, K), dtype=torch.bfloat16, device=dev),
           "dA": torch.empty((r, K), dtype=torch.float32, device=dev),
           "dB": torch.empty((N, r), dtype=torch.float32, device=dev)}
    ws_f = torch.empty(max(lib.qlora_fwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(max(lib.qlora_bwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)

    def step():
        lib.nf4_quantize(g["W"].reshape(-1), codes, c8, s2)
        lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], s, Y=out["Y"], U=out["U"], ws=ws_f)
        lib.qlora_linear_bwd(g["dY"], g["X"], out["U"], W, g["A"], g["B"], s, dX=out["dX"], dA=out["dA"],
                             dB=out["dB"], ws=ws_b)

    cs = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(cs):
        for _ in range(3):
            step()
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in out.items()}
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs):
        step()
    for v in out.values():
        v.zero_()
    graph.replay()
    torch.cuda.synchronize()
    equal = all(torch.equal(out[k].view(torch.int16) if out[k].dtype == torch.bfloat16 else out[k].view(torch.int32),
                            ref[k].view(torch.int16) if ref[k].dtype == torch.bfloat16 else ref[k].view(torch.int32))
                for k in out)

    def timed(fn):
        with torch.cuda.stream(cs):
            for _ in range(10):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(cs)
            for _ in range(reps):
                fn()
            e1.record(cs)
        e1.synchronize()
        return 1000.0 * e0.elapsed_time(e1) / reps

    eager_us = timed(step)
    graph_us = timed(graph.replay)
    del graph
    return {"eager_us_per_step": round(eager_us, 2), "graph_us_per_step": round(graph_us, 2),
            "replay_bit_equal": bool(equal), "steps": reps,
            "workload": "512x512 NF4, 64 tokens, r=16: quantize + fwd + bwd back to back (L2-resident)"}


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    cores, blas = cpu_cores()
    times, vals = [], []
    for i in range(args.warmup + args.steps):
        v, dt, desc = cpu_oracle_sample(reps=1, m_s=256, n_s=1024, seed=i)
        if i >= args.warmup:
            times.append(dt)
            vals.append(v)
    value = float(np.mean(vals))
    ms = 1e3 * float(np.mean(times))
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD_NAME, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist

    import bit_nf4_quantized_26_b200 as lib
    import synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[WORKLOAD]
    lin = wl.linears[0]
    M, N, K, r, s = wl.m_tokens, lin.n_out, lin.k_in, wl.r, wl.s
    d = synth.dp_shard_inputs(lin, M, r, rank)
    g = {k: v.to(dev) for k, v in d.items()}
    W_bf16 = g["W"]
    nc, nb, ns = lib.nf4_sizes(N * K)
    codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    c8 = torch.empty(nb, dtype=torch.uint8, device=dev)
    s2 = torch.empty(ns, dtype=torch.float32, device=dev)
    W = lib.NF4Weight(codes, c8, s2, N, K)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    U = torch.empty((M, r), dtype=torch.float32, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    dB = torch.empty((N, r), dtype=torch.float32, device=dev)
    ws_f = torch.empty(lib.qlora_fwd_workspace_size(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(lib.qlora_bwd_workspace_size(M, N, K, r), dtype=torch.uint8, device=dev)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        lib.nf4_quantize(W_bf16.reshape(-1), codes, c8, s2, status=status)
        lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], s, Y=Y, U=U, ws=ws_f, status=status)
        lib.qlora_linear_bwd(g["dY"], g["X"], U, W, g["A"], g["B"], s, dX=dX, dA=dA, dB=dB, ws=ws_b,
                             status=status)
        if world > 1:
            dist.all_reduce(dA)
            dist.all_reduce(dB)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # ---------------------------------------------------------- timed region
    # Phase A (the reported value): K steps, one event pair per step, nothing
    # else in the stream between the step's kernels (they chain through
    # programmatic dependent launch).  Phase B: the same K steps again with
    # every library kernel bracketed by events, for the per-kernel table and
    # the roofline of the dominant kernel.
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)

    def timed_steps():
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            step()
            e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return [a.elapsed_time(b) for a, b in evs]

    step_ms = timed_steps()
    lib.profile_enable(True)
    step_ms_profiled = timed_steps()
    lib.profile_enable(False)
    clocks = sampler.stop()
    records = lib.profile_collect()
    ms = float(sum(step_ms) / len(step_ms))
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    assert int(status[0].item()) == 0, f"device status {int(status[0].item())}"

    # per-kernel statistics from the library's event brackets
    kern = {}
    for name, t in records:
        k = kern.setdefault(name, {"launches": 0, "ms_total": 0.0})
        k["launches"] += 1
        k["ms_total"] += t
    tot = sum(k["ms_total"] for k in kern.values()) or 1.0
    for k in kern.values():
        k["share"] = k["ms_total"] / tot
        k["ms_avg"] = k["ms_total"] / k["launches"]
    peaks = load_peaks()
    tc = {n: k for n, k in kern.items() if n in ("fused_fwd", "fused_dx")}
    dom = max(tc, key=lambda n: tc[n]["ms_total"]) if tc else None
    roofline = None
    if dom:
        fl = kernel_flops(dom, M, N, K, r)
        ach = fl / (kern[dom]["ms_avg"] * 1e-3) / 1e12
        roofline = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"], "traffic": NCU_TRAFFIC_BYTES.get(dom),
                    "peak_source": f"{peaks['source']} bf16 burst"}
        for n in tc:
            kf = kernel_flops(n, M, N, K, r)
            kern[n]["tflops"] = kf / (kern[n]["ms_avg"] * 1e-3) / 1e12

    if args.kernels_only:
        if rank == 0:
            print(json.dumps({"kernels_only": True, "ms_per_step": ms,
                              "ms_per_step_profiled": float(np.mean(step_ms_profiled)), "kernels": kern}), flush=True)
        return

    # ------------------------------------------------ NF4 stream bandwidth
    # Separate launches on a weight larger than L2 (22016x8192, 65B-shaped).
    big = synth.weight_bf16(22016, 8192, seed=99, device=dev)
    bcodes, bc8, bs2 = lib.nf4_quantize(big.reshape(-1))
    bout = torch.empty(big.numel(), dtype=torch.bfloat16, device=dev)
    lib.profile_enable(True)
    for _ in range(5):
        flush.zero_()
        lib.nf4_quantize(big.reshape(-1), bcodes, bc8, bs2)
        flush.zero_()
        lib.nf4_dequantize(bcodes, bc8, bs2, big.numel(), out=bout)
    torch.cuda.synchronize()
    lib.profile_enable(False)
    qrec = lib.profile_collect()
    bytes_nf4 = big.numel() * (2 + 0.5 + 1 / 64 + 4 / 16384)
    qt = [t for n, t in qrec if n == "nf4_quantize"]
    dqt = [t for n, t in qrec if n == "nf4_dequantize"]
    quant_gbs = bytes_nf4 / (statistics.median(qt) * 1e-3) / 1e9
    dequant_gbs = bytes_nf4 / (statistics.median(dqt) * 1e-3) / 1e9
    del big, bcodes, bc8, bs2, bout

    # ------------------------------------------- adapter optimizer step
    adamw = adamw8_timing(lib, synth, torch, dev, flush, peaks) if (rank == 0 and not args.no_sweep) else None
    drop = dropout_timing(lib, synth, torch, dev, flush) if (rank == 0 and not args.no_sweep) else None

    # ------------------------------------------- 65B-shaped forward sweep
    c5 = c5_forward_sweep(lib, synth, torch, dev, flush, peaks) if (rank == 0 and not args.no_sweep) else None
    c1g = c1_graph_timing(lib, synth, torch, dev) if (rank == 0 and not args.no_sweep) else None

    # ------------------------------------------------------------- e2e
    host = {k: torch.empty_like(g[k], device="cpu").pin_memory() for k in ("W", "X", "dY")}
    for k in host:
        host[k].copy_(d[k])
    hout = {"Y": torch.empty_like(Y, device="cpu").pin_memory(), "dX": torch.empty_like(dX, device="cpu").pin_memory(),
            "dA": torch.empty_like(dA, device="cpu").pin_memory(), "dB": torch.empty_like(dB, device="cpu").pin_memory()}
    outs = {"Y": Y, "dX": dX, "dA": dA, "dB": dB}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in hout.values())
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for k in host:
            g[k].copy_(host[k], non_blocking=True)
        step()
        for k in hout:
            hout[k].copy_(outs[k], non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e = float(np.mean(e2e_ms))
    if world > 1:
        t = torch.tensor([e2e], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e = float(t.item())

    fl = flops_fwd_bwd(M, N, K, r)
    value = world * fl / (ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cores, blas = cpu_cores()
        v, dt, desc = cpu_oracle_sample(reps=4)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": blas, "kind": "oracle", "sample": desc,
               "seconds": dt}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAME, "M": M, "N": N, "K": K, "r": r, "alpha": wl.alpha,
                       "parallelism": f"dp{world}", "global_batch": M * world,
                       "step": "nf4_quantize + qlora_linear_fwd + qlora_linear_bwd (+ dA/dB all-reduce if N>1)",
                       "l2": "flushed before every step (512 MB memset outside the step's events)",
                       "pdl": os.environ.get("QLORA_PDL", "1") != "0"},
            "pct_bf16_peak": value / world / peaks["bf16_tflops"],
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": world * fl / (e2e * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": len(records),
            "timing": {"value_from": "phase A: K steps, step-level events only",
                       "kernels_from": "phase B: the same K steps with per-kernel event brackets",
                       "ms_per_step_phase_b": float(np.mean(step_ms_profiled))},
            "clocks": clocks,
            "kernels": {n: {kk: round(vv, 5) if isinstance(vv, float) else vv for kk, vv in k.items()}
                        for n, k in sorted(kern.items(), key=lambda x: -x[1]["ms_total"])},
            "nf4_quantize_gbs": quant_gbs, "nf4_dequantize_gbs": dequant_gbs,
            "c5_forward": c5,
            "c1_graph": c1g,
            "adamw8": adamw,
            "lora_dropout": drop,
            "nf4_hbm_frac": {"quantize": quant_gbs / peaks["hbm_gbs"], "dequantize": dequant_gbs / peaks["hbm_gbs"],
                             "peak_gbs": peaks["hbm_gbs"], "peak_source": peaks["source"]},
        }
        print(json.dumps(line), flush=True)


def dropout_timing(lib, synth, torch, dev, flush, p=0.05, reps=10):
    """The c2 forward + backward with LoRA dropout (p = 0.05, the tutorial's
    lora_dropout) against the same step without it; L2 flushed before each."""
    import statistics
    M = N = K = 4096
    r, s = 64, 0.25
    d = {k: v.to(dev) for k, v in synth.linear_inputs(synth.Linear("c2", N, K), M, r, 0).items()}
    W = lib.quantize_weight(d["W"])
    fws = torch.empty(lib.qlora_fwd_workspace_size(M, N, K, r), dtype=torch.uint8, device=dev)
    bws = torch.empty(lib.qlora_bwd_dropout_workspace_size(M, N, K, r), dtype=torch.uint8, device=dev)
    Y, U, Xd = lib.qlora_linear_fwd_dropout(d["X"], W, d["A"], d["B"], s, p, 1, ws=fws)
    dX, dA, dB = lib.qlora_linear_bwd_dropout(d["dY"], Xd, U, W, d["A"], d["B"], s, p, 1, ws=bws)

    def with_dropout(i):
        lib.qlora_linear_fwd_dropout(d["X"], W, d["A"], d["B"], s, p, i, Y=Y, U=U, X_drop=Xd, ws=fws)
        lib.qlora_linear_bwd_dropout(d["dY"], Xd, U, W, d["A"], d["B"], s, p, i, dX=dX, dA=dA, dB=dB, ws=bws)

    def plain(i):
        lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], s, Y=Y, U=U, ws=fws)
        lib.qlora_linear_bwd(d["dY"], d["X"], U, W, d["A"], d["B"], s, dX=dX, dA=dA, dB=dB, ws=bws)

    out = {"p": p, "workload": "c2 (4096x4096, 4x1024 tokens, r=64): forward + backward"}
    fl = flops_fwd_bwd(M, N, K, r)
    for name, fn in (("dropout", with_dropout), ("plain", plain)):
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn(i + 1)
            e1.record()
            e1.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        out[name] = {"us": ms * 1e3, "tflops": fl / (ms * 1e-3) / 1e12}
    out["overhead"] = out["dropout"]["us"] / out["plain"]["us"] - 1.0
    return out


def adamw8_timing(lib, synth, torch, dev, flush, peaks, layers=10, reps=10):
    """AdamW with 8-bit states over the r=64 adapters of ``layers`` 65B-shaped
    layers (about 100M parameters, 1.2 GB streamed per step: larger than L2),
    states in device memory and in paged (managed, device-resident) memory.
    Algorithmic bytes per parameter: bf16 p read + write, fp32 gradient, two
    state bytes read + write, two fp32 scales per 256 read + write."""
    import statistics
    r = 64
    per_layer = sum(r * (lin.n_out + lin.k_in) for lin in synth.c5_layer_linears())
    n = per_layer * layers
    gen = torch.Generator(device=dev).manual_seed(5)
    p = (torch.randn(n, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    grad = torch.randn(n, generator=gen, device=dev) * 1e-3
    bytes_per = 2 + 2 + 4 + 2 + 2 + 16 / 256
    out = {"params": n, "layers": layers, "bytes_per_param": bytes_per}
    for paged in (False, True):
        st = lib.AdamW8State(n, paged=paged)
        st.prefetch(to_host=False)
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            lib.qlora_adamw8_step(p, grad, st, lr=2e-4, step=i + 1)
            e1.record()
            e1.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        gbs = n * bytes_per / (ms * 1e-3) / 1e9
        key = "paged" if paged else "device"
        out[key] = {"us": ms * 1e3, "gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"]}
        st.close()
    del p, grad
    return out


def run_case(args):
    """Profiler driver: time one entry point on one shape (no JSON contract).

    --case fwd:M:N:K or bwd:M:N:K (r=64, alpha=16), quant:N:K / dequant:N:K (NF4
    quantisation / dequantisation of an N x K weight), or adamw8:n (one 8-bit AdamW
    step over n parameters), --steps calls after 2 warm-up calls.
    """
    import torch

    import bit_nf4_quantized_26_b200 as lib
    import synth
    if args.case.startswith("adamw8:"):
        n = int(args.case.split(":")[1])
        gen = torch.Generator(device="cuda").manual_seed(5)
        p = (torch.randn(n, generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
        g = torch.randn(n, generator=gen, device="cuda") * 1e-3
        st = lib.AdamW8State(n, paged=False)
        for i in range(2 + args.steps):
            lib.qlora_adamw8_step(p, g, st, lr=2e-4, step=i + 1)
        torch.cuda.synchronize()
        st.close()
        print(json.dumps({"case": args.case, "ok": True}))
        return
    if args.case.startswith("dequant:"):
        _, N, K = args.case.split(":")
        w = synth.weight_bf16(int(N), int(K), seed=1, device="cuda")
        W = lib.quantize_weight(w)
        out = torch.empty(w.numel(), dtype=torch.bfloat16, device="cuda")
        del w
        for _ in range(2 + args.steps):
            lib.nf4_dequantize(W.codes, W.c8, W.s2, out.numel(), out=out)
        torch.cuda.synchronize()
        print(json.dumps({"case": args.case, "ok": True}))
        return
    if args.case.startswith("quant:"):
        _, N, K = args.case.split(":")
        w = synth.weight_bf16(int(N), int(K), seed=1, device="cuda")
        W = lib.quantize_weight(w)
        for _ in range(2 + args.steps):
            lib.nf4_quantize(w.view(-1), W.codes, W.c8, W.s2)
        torch.cuda.synchronize()
        print(json.dumps({"case": args.case, "ok": True}))
        return
    kind, M, N, K = args.case.split(":")
    M, N, K, r = int(M), int(N), int(K), 64
    d = {k: v.cuda() for k, v in synth.linear_inputs(synth.Linear("case", N, K), M, r, 0).items()}
    W = lib.quantize_weight(d["W"])
    Y, U = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.25)
    for _ in range(2 + args.steps):
        if kind == "fwd":
            lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.25, Y=Y, U=U)
        else:
            lib.qlora_linear_bwd(d["dY"], d["X"], U, W, d["A"], d["B"], 0.25)
    torch.cuda.synchronize()
    print(json.dumps({"case": args.case, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-sweep", action="store_true", help="skip the 65B-shaped forward sweep")
    ap.add_argument("--kernels-only", action="store_true",
                    help="only the timed steps (for profiler captures): no e2e, no NF4 stream test, no CPU baseline")
    ap.add_argument("--case", default=None,
                    help="profiler driver: fwd:M:N:K, bwd:M:N:K, quant:N:K, dequant:N:K or adamw8:n")
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
