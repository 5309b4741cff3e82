#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear hot path on B200.

Headline workload: the seven linears of a LLaMA-7B-shaped decoder layer
(q, k, v, o 4096x4096; gate, up 4096->11008; down 11008->4096), every weight
NF4 with FP8 double quantisation, LoRA r=64 alpha=16 on all seven,
8 x 2048 = 16384 tokens per GPU, synthetic seeded inputs.  One step, all
through the library's C ABI:

  * NF4 quantisation of the seven frozen bf16 weights (absmax per 64, FP8
    double quantisation per 256);
  * forward of every linear in layer order: U = X A^T, Y = X W'^T + s U B^T
    with W' dequantised inside the GEMM (q, k, v read the same input and so do
    gate and up; with grouping on they run as one call per group);
  * backward in reverse order: dU, dB, dX, dA (a group's dX is the sum over
    its members, the gradient of the shared input);
  * with N > 1 ranks, the sum of each linear's dA/dB over ranks (NCCL,
    issued as soon as that linear's backward is enqueued, so it overlaps the
    next linear's backward);
  * the 8-bit AdamW step on every adapter.

value = algorithmic fwd+bwd FLOPs of the seven linears (sum of
4MNK + 6MKr + 6MNr) / device time per step, summed over ranks (each rank runs
its own batch: weak scaling).  Quantisation and the optimizer step are in
the timed step but not in the FLOP count.

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
WORKLOAD_NAME = ("LLaMA-7B-shaped decoder layer, all 7 linears (q,k,v,o 4096x4096; gate,up 4096->11008; "
                 "down 11008->4096), NF4/64 + FP8/256, LoRA r=64 alpha=16 on every linear, 8x2048 = 16384 tokens")
M_TOKENS = 8 * 2048
RANK_R = 64
ALPHA = 16.0
# Earlier measurements on this GPU type, used when no measured-peaks file is
# present: copy bandwidth, cuBLAS bf16 as a burst, and the same GEMM held for
# seconds under the power cap (about 1.3 GHz).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NF4_BYTES_PER_PARAM = 2 + 0.5 + 1 / 64 + 4 / 16384
# Per-launch DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the
# CTA-pair GEMMs in the grouped layer step (mean over the step's 4 launches of
# each), from one ncu capture of the current kernels (the decoder-layer-step
# summary under profiles/); emptied whenever those kernels change.
NCU_TRAFFIC_BYTES = {"fused_fwd": 705.5e6, "fused_dx": 722.1e6}


def flops_fwd_bwd(M, N, K, r):
    return 4 * M * N * K + 6 * M * K * r + 6 * M * N * r


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

def cpu_cores():
    """(cores this process may run on, BLAS threads numpy uses)."""
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


_SAMPLE_CACHE = {}


def _sample_inputs(m_s, n_s):
    """Seeded inputs of the oracle's sample, drawn once per size."""
    import synth
    key = (m_s, n_s)
    if key not in _SAMPLE_CACHE:
        _SAMPLE_CACHE[key] = [
            {k: synth.bf16_bits(v) for k, v in
             synth.linear_inputs(synth.Linear("sample", n_s, lin.k_in), m_s, RANK_R, 10 + i).items()}
            for i, lin in enumerate(synth.LLAMA7B_LAYER)]
    return _SAMPLE_CACHE[key]


def cpu_oracle_layer_sample(m_s=512, n_s=1024):
    """Time the oracle on a bounded sample of the layer workload.

    Sample, for each of the seven linears: the first n_s output features of
    its weight (all K input features) and m_s tokens; NF4-quantise and
    dequantise those weight rows, then the fp64 forward and backward
    (U, Y, dU, dX, dA, dB) on (m_s tokens, n_s features, K, r=64).
    Returns (TFLOP/s on the sample's fwd+bwd FLOPs, seconds, description).
    """
    import synth
    from oracle import linear as ol
    from oracle import nf4
    s = ALPHA / RANK_R
    fl, dt = 0.0, 0.0
    for b, lin in zip(_sample_inputs(m_s, n_s), synth.LLAMA7B_LAYER):
        t0 = time.perf_counter()
        codes, c8, s2 = nf4.quantize(b["W"].reshape(-1))
        wd = nf4.dequantize(codes, c8, s2, b["W"].size).reshape(b["W"].shape)
        ol.linear_fwd(b["X"], wd, b["A"], b["B"], s)
        ol.linear_bwd(b["dY"], b["X"], wd, b["A"], b["B"], s)
        dt += time.perf_counter() - t0
        fl += flops_fwd_bwd(m_s, n_s, lin.k_in, RANK_R)
    desc = (f"per linear of the layer: quantize+dequantize {n_s} weight rows (all K), fp64 fwd+bwd on {m_s} "
            f"tokens x {n_s} output features x K, r={RANK_R}")
    return fl / dt / 1e12, dt, desc


def cpu_oracle_nf4_rates(n_rows=4096, k=8192, seed=0):
    """Oracle NF4 quantise and dequantise throughput on an n_rows x k weight:
    params/s and the equivalent GB/s at 2.5159 B/param (bf16 in, NF4 out)."""
    import synth
    from oracle import nf4
    wb = synth.bf16_bits(synth.weight_bf16(n_rows, k, seed)).reshape(-1)
    t0 = time.perf_counter()
    codes, c8, s2 = nf4.quantize(wb)
    tq = time.perf_counter() - t0
    t0 = time.perf_counter()
    nf4.dequantize(codes, c8, s2, wb.size)
    tdq = time.perf_counter() - t0
    n = wb.size
    return {"params": n, "quantize_params_per_s": n / tq, "quantize_gbs": n * NF4_BYTES_PER_PARAM / tq / 1e9,
            "dequantize_params_per_s": n / tdq, "dequantize_gbs": n * NF4_BYTES_PER_PARAM / tdq / 1e9,
            "seconds": tq + tdq}


# ------------------------------------------------------------ the layer step

# The decoder layer's linears by shared input: q/k/v read the attention
# input, gate/up the MLP input; o and down read their own.
LAYER_GROUPS = (("attn", (0, 1, 2)), ("o", (3,)), ("mlp", (4, 5)), ("down", (6,)))


class LayerStep:
    """The decoder layer's seven QLoRA linears on one GPU: buffers, and the
    quantise / forward / backward / optimizer phases of one training step.
    grouped: the linears that share an input run as one grouped call (their
    weights, adapters, outputs and gradients stacked along the output
    dimension, their input gradient summed); otherwise every linear is its
    own call."""

    def __init__(self, lib, synth, torch, dev, M, rank=0, world=1, grouped=True):
        self.lib, self.torch, self.dev = lib, torch, dev
        self.M, self.r, self.s = M, RANK_R, ALPHA / RANK_R
        self.world = world
        self.grouped = grouped and hasattr(lib, "qlora_group_fwd")
        self.lins = synth.LLAMA7B_LAYER
        r = self.r
        params = synth.decoder_layer_params(r, seed=0, device=dev)
        X, dY = synth.decoder_layer_activations(M, rank=rank, device=dev)
        self.X = X
        if self.grouped:
            units = [(name, idx) for name, idx in LAYER_GROUPS]
        else:
            units = [(synth.LAYER_INPUT_OF[i], (i,)) for i in range(len(self.lins))]
        self.units = []
        for name, idx in units:
            K = self.lins[idx[0]].k_in
            ns = [self.lins[i].n_out for i in idx]
            N = sum(ns)
            G = len(idx)
            u = {"x": name, "members": ns, "G": G, "N": N, "K": K}
            u["Wb"] = torch.cat([params[i]["W"] for i in idx], 0).contiguous() if G > 1 else params[idx[0]]["W"]
            nc, nb, nsz = lib.nf4_sizes(N * K)
            u["W"] = lib.NF4Weight(torch.empty(nc, dtype=torch.uint8, device=dev),
                                   torch.empty(nb, dtype=torch.uint8, device=dev),
                                   torch.empty(nsz, dtype=torch.float32, device=dev), N, K)
            # The stacked adapters A [G r, K] and B [N, r] are views of one flat
            # bf16 parameter, dA and dB of one flat fp32 gradient (one
            # all-reduce and one optimizer call per unit).
            p = torch.empty(G * r * K + N * r, dtype=torch.bfloat16, device=dev)
            p[: G * r * K].copy_(torch.cat([params[i]["A"] for i in idx], 0).reshape(-1))
            p[G * r * K:].copy_(torch.cat([params[i]["B"] for i in idx], 0).reshape(-1))
            gr = torch.empty_like(p, dtype=torch.float32)
            u.update(param=p, grad=gr, A=p[: G * r * K].view(G * r, K), B=p[G * r * K:].view(N, r),
                     dA=gr[: G * r * K].view(G * r, K), dB=gr[G * r * K:].view(N, r))
            u["dY"] = torch.cat([dY[i] for i in idx], 1).contiguous() if G > 1 else dY[idx[0]]
            u["U"] = torch.empty((M, G * r), dtype=torch.float32, device=dev)
            u["Y"] = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            u["dX"] = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
            u["opt"] = lib.AdamW8State(p.numel(), paged=False, device=dev)
            self.units.append(u)
        del params, dY
        wsf = max(lib.qlora_group_fwd_workspace_size(M, u["N"], u["K"], u["G"], r) if self.grouped else
                  lib.qlora_fwd_workspace_size(M, u["N"], u["K"], r) for u in self.units)
        wsb = max(lib.qlora_group_bwd_workspace_size(M, u["N"], u["K"], u["G"], r) if self.grouped else
                  lib.qlora_bwd_workspace_size(M, u["N"], u["K"], r) for u in self.units)
        self.ws_f = torch.empty(max(wsf, 16), dtype=torch.uint8, device=dev)
        self.ws_b = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)
        self.t = 0
        self.pending = []
        # Called with an input's key ("X_<name>" or "dY_<unit>") just before
        # the first call that reads it (the end-to-end step waits there for
        # that input's host-to-device copy).
        self.before_use = None

    def input_order(self):
        """Keys of the step's inputs in the order the step first reads them."""
        keys = [f"X_{u['x']}" for u in self.units] + [f"dY_{i}" for i in reversed(range(len(self.units)))]
        return list(dict.fromkeys(keys))

    @property
    def dY(self):
        return [u["dY"] for u in self.units]

    @property
    def grad(self):
        return [u["grad"] for u in self.units]

    def flops(self):
        return sum(flops_fwd_bwd(self.M, lin.n_out, lin.k_in, self.r) for lin in self.lins)

    def kernel_flops(self, name):
        """Algorithmic FLOPs per step of the named tensor-core kernel."""
        M, r = self.M, self.r
        tot = 0
        for lin in self.lins:
            N, K = lin.n_out, lin.k_in
            tot += {"fused_fwd": 2 * M * N * K + 2 * M * N * r, "fused_dx": 2 * M * N * K + 2 * M * K * r,
                    "lora_down": 2 * M * K * r, "lora_du": 2 * M * N * r, "lora_db": 2 * M * N * r,
                    "lora_da": 2 * M * K * r}.get(name, 0)
        return tot

    def quantize(self):
        for u in self.units:
            W = u["W"]
            self.lib.nf4_quantize(u["Wb"].reshape(-1), W.codes, W.c8, W.s2, status=self.status)

    def forward(self):
        lib = self.lib
        for u in self.units:
            X = self.X[u["x"]]
            if self.before_use is not None:
                self.before_use(f"X_{u['x']}")
            if self.grouped:
                lib.qlora_group_fwd(X, u["W"], u["members"], u["A"], u["B"], self.s, Y=u["Y"], U=u["U"],
                                    ws=self.ws_f, status=self.status)
            else:
                lib.qlora_linear_fwd(X, u["W"], u["A"], u["B"], self.s, Y=u["Y"], U=u["U"], ws=self.ws_f,
                                     status=self.status)

    def backward(self):
        lib = self.lib
        for i in reversed(range(len(self.units))):
            u = self.units[i]
            X = self.X[u["x"]]
            if self.before_use is not None:
                self.before_use(f"dY_{i}")
            if self.grouped:
                lib.qlora_group_bwd(u["dY"], X, u["U"], u["W"], u["members"], u["A"], u["B"], self.s, dX=u["dX"],
                                    dA=u["dA"], dB=u["dB"], ws=self.ws_b, status=self.status)
            else:
                lib.qlora_linear_bwd(u["dY"], X, u["U"], u["W"], u["A"], u["B"], self.s, dX=u["dX"], dA=u["dA"],
                                     dB=u["dB"], ws=self.ws_b, status=self.status)
            self._reduce(u)

    def _reduce(self, u):
        # Sum of the adapter gradients over ranks, issued right after this
        # unit's backward: NCCL's stream waits for it and then runs beside
        # the next unit's backward.
        if self.world > 1:
            import torch.distributed as dist
            self.pending.append(dist.all_reduce(u["grad"], async_op=True))

    def optimizer(self):
        for h in self.pending:
            h.wait()
        self.pending = []
        self.t += 1
        for u in self.units:
            self.lib.qlora_adamw8_step(u["param"], u["grad"], u["opt"], lr=2e-4, step=self.t, status=self.status)

    def step(self):
        self.quantize()
        self.forward()
        self.backward()
        self.optimizer()

    def close(self):
        for u in self.units:
            u["opt"].close()


def with_clocks(dev, fn):
    """Run fn() with the SM clock sampled beside it: (*result, clocks) for a
    tuple result, else (result, clocks)."""
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.2)
    try:
        res = fn()
    finally:
        clocks = sampler.stop()
    return (*res, clocks) if isinstance(res, tuple) else (res, clocks)


def time_steps(torch, step, stream, steps, flush, dist=None):
    """Per-step device times (ms) of `steps` steps, one event pair each, L2
    flushed (512 MB memset) before every step outside its events."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return [a.elapsed_time(b) for a, b in evs]


def kernel_table(records, steps):
    kern = {}
    for name, t in records:
        k = kern.setdefault(name, {"launches": 0, "ms_total": 0.0})
        k["launches"] += 1
        k["ms_total"] += t
    tot = sum(k["ms_total"] for k in kern.values()) or 1.0
    for k in kern.values():
        k["share"] = k["ms_total"] / tot
        k["ms_avg"] = k["ms_total"] / k["launches"]
        k["ms_per_step"] = k["ms_total"] / steps
    return kern


# ------------------------------------------------------------------ extras

def c2_step_timing(lib, synth, torch, dev, flush, reps=20):
    """The single 4096x4096 projection (4 x 1024 tokens, r=64): quantise +
    forward + backward, L2 flushed before each step."""
    wl = synth.WORKLOADS["c2"]
    lin = wl.linears[0]
    M, N, K, r, s = wl.m_tokens, lin.n_out, lin.k_in, wl.r, wl.s
    g = {k: v.to(dev) for k, v in synth.linear_inputs(lin, M, r, 0).items()}
    W = lib.quantize_weight(g["W"])
    out = {"Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
           "U": torch.empty((M, r), dtype=torch.float32, device=dev),
           "dX": torch.empty((M, K), dtype=torch.bfloat16, device=dev),
           "dA": torch.empty((r, K), dtype=torch.float32, device=dev),
           "dB": torch.empty((N, r), dtype=torch.float32, device=dev)}
    ws_f = torch.empty(lib.qlora_fwd_workspace_size(M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(lib.qlora_bwd_workspace_size(M, N, K, r), dtype=torch.uint8, device=dev)

    def step():
        lib.nf4_quantize(g["W"].reshape(-1), W.codes, W.c8, W.s2)
        lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], s, Y=out["Y"], U=out["U"], ws=ws_f)
        lib.qlora_linear_bwd(g["dY"], g["X"], out["U"], W, g["A"], g["B"], s, dX=out["dX"], dA=out["dA"],
                             dB=out["dB"], ws=ws_b)

    for _ in range(3):
        step()
    ts = time_steps(torch, step, torch.cuda.current_stream(), reps, flush)
    ms = statistics.median(ts)
    return {"workload": "4096x4096 projection, 4x1024 tokens, r=64: quantize + fwd + bwd (L2 flushed)",
            "ms": ms, "tflops": flops_fwd_bwd(M, N, K, r) / (ms * 1e-3) / 1e12}


def c5_forward_sweep(lib, synth, torch, dev, flush, peaks, reps=7):
    """Forward of the 65B-shaped 8192<->22016 linears over M in {1,16,128,2048,16384}.

    Per case: algorithmic bytes 0.5159 N K + 2 M K + 2 M N + 2 r (K + N) and
    FLOPs 2 M N K + 2 M K r + 2 M N r, over the median device time of the
    forward call (L2 flushed before each call).  Plain calls alternate with
    calls that bracket every kernel with events (the brackets serialise the
    kernels, which otherwise overlap through programmatic dependent launch),
    so both see the same clocks: kernels_ms is the per-kernel median over the
    bracketed calls and ms_bracketed their median outer time.
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

            def call():
                lib.qlora_linear_fwd(X, W, A, B, s, Y=Y, U=U, ws=ws)

            def timed():
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                call()
                e1.record()
                e1.synchronize()
                return e0.elapsed_time(e1)

            for _ in range(3):
                call()
            torch.cuda.synchronize()
            lib.profile_collect()
            ts, tb, per = [], [], {}
            for _ in range(reps):
                ts.append(timed())
                lib.profile_enable(True)
                tb.append(timed())
                lib.profile_enable(False)
                this = {}
                for name, kms in lib.profile_collect():
                    this[name] = this.get(name, 0.0) + kms
                for name, kms in this.items():
                    per.setdefault(name, []).append(kms)
            ms = float(statistics.median(ts))
            kern = {k: float(statistics.median(v)) for k, v in per.items()}
            byts = 0.51587 * N * K + 2 * M * K + 2 * M * N + 2 * r * (K + N)
            fl = 2 * M * N * K + 2 * M * K * r + 2 * M * N * r
            out[f"{lin.name}_{N}x{K}_M{M}"] = {
                "ms": round(ms, 5), "tflops": round(fl / ms / 1e9, 2), "gbs": round(byts / ms / 1e6, 1),
                "hbm_frac": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4),
                "tensor_frac": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4),
                "ms_bracketed": round(float(statistics.median(tb)), 5),
                "kernels_ms": {k: round(v, 5) for k, v in kern.items()}}
            del X, Y, U, ws
        del W, A, B
    return out


def c5_quantize_sweep(lib, synth, torch, dev):
    """NF4 quantisation of every linear weight of the 80-layer 65B-shaped
    model (hidden 8192, intermediate 22016; 64.76 G parameters).  Each layer's
    seven bf16 weights are drawn on the device, quantised, and dropped: only
    the NF4 storage (33.4 GB) stays resident.  GB/s counts 2.5159 B/param over
    the summed device time of the quantise calls; the wall time includes the
    random draws.  Weight seeds: 650000 + 10 * layer + index (the GPU test
    of this sweep redraws layers with the same seeds)."""
    t_wall = time.perf_counter()
    kept, total_ms, params = [], 0.0, 0
    for layer in range(synth.C5_LAYERS):
        for j, lin in enumerate(synth.c5_layer_linears()):
            w = synth.weight_bf16(lin.n_out, lin.k_in, seed=650000 + 10 * layer + j, device=dev)
            nc, nb, ns = lib.nf4_sizes(w.numel())
            codes = torch.empty(nc, dtype=torch.uint8, device=dev)
            c8 = torch.empty(nb, dtype=torch.uint8, device=dev)
            s2 = torch.empty(ns, dtype=torch.float32, device=dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            lib.nf4_quantize(w.reshape(-1), codes, c8, s2)
            e1.record()
            kept.append((codes, c8, s2, e0, e1))
            params += w.numel()
            del w
    torch.cuda.synchronize()
    for k in kept:
        total_ms += k[3].elapsed_time(k[4])
    wall = time.perf_counter() - t_wall
    resident = sum(k[0].numel() + k[1].numel() + 4 * k[2].numel() for k in kept)
    del kept
    return {"layers": synth.C5_LAYERS, "params": params, "resident_nf4_bytes": resident,
            "quantize_ms_total": total_ms, "quantize_gbs": params * NF4_BYTES_PER_PARAM / (total_ms * 1e-3) / 1e9,
            "wall_s_with_draws": wall}


def centered_cost(lib, synth, torch, dev, flush, reps=5):
    """What mean-centred double quantisation costs against the plain scheme,
    per kernel family (median device times, L2 flushed before each call):
    quantise and dequantise a 22016x8192 weight, the few-token forward (16
    tokens) on it, and the 4096x4096 forward + backward at 4096 tokens."""
    import statistics

    def med(fn):
        ts = []
        for i in range(reps + 2):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            if i >= 2:
                ts.append(e0.elapsed_time(e1))
        return statistics.median(ts) * 1e3

    out = {}
    w = synth.weight_bf16(22016, 8192, seed=99, device=dev)
    Wp = lib.quantize_weight(w)
    Wc = lib.quantize_weight_centered(w)
    ws = torch.empty(lib.nf4_centered_workspace_size(w.numel()), dtype=torch.uint8, device=dev)
    dq = torch.empty(w.numel(), dtype=torch.bfloat16, device=dev)
    out["quantize_us"] = {"plain": med(lambda: lib.nf4_quantize(w.reshape(-1), Wp.codes, Wp.c8, Wp.s2)),
                          "centered": med(lambda: lib.nf4_quantize_centered(w.reshape(-1), Wc.codes, Wc.c8, Wc.s2,
                                                                            Wc.mean, ws=ws))}
    out["dequantize_us"] = {"plain": med(lambda: lib.nf4_dequantize(Wp.codes, Wp.c8, Wp.s2, w.numel(), out=dq)),
                            "centered": med(lambda: lib.nf4_dequantize_centered(Wc.codes, Wc.c8, Wc.s2, Wc.mean,
                                                                                w.numel(), out=dq))}
    del dq, ws
    X = synth.normal_bf16((16, 8192), 1.0, seed=5, device=dev)
    A = synth.normal_bf16((64, 8192), 1.0 / 8192, seed=6, device=dev)
    B = synth.normal_bf16((22016, 64), synth.B_STD, seed=7, device=dev)
    Y = torch.empty((16, 22016), dtype=torch.bfloat16, device=dev)
    U = torch.empty((16, 64), dtype=torch.float32, device=dev)
    out["fwd_16_tokens_us"] = {k: med(lambda W=W: lib.qlora_linear_fwd(X, W, A, B, 0.25, Y=Y, U=U))
                               for k, W in (("plain", Wp), ("centered", Wc))}
    del w, Wp, Wc, X, A, B, Y, U
    d = {k: v.to(dev) for k, v in synth.linear_inputs(synth.Linear("c2", 4096, 4096), 4096, 64, 0).items()}
    Wp = lib.quantize_weight(d["W"])
    Wc = lib.quantize_weight_centered(d["W"])

    def fb(W):
        _, U2 = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.25)
        lib.qlora_linear_bwd(d["dY"], d["X"], U2, W, d["A"], d["B"], 0.25)
    out["fwd_bwd_4096_us"] = {k: med(lambda W=W: fb(W)) for k, W in (("plain", Wp), ("centered", Wc))}
    for k in list(out):
        out[k]["overhead"] = out[k]["centered"] / out[k]["plain"] - 1.0
    out["workload"] = ("22016x8192 weight (quantise, dequantise, 16-token forward); 4096x4096 forward + backward "
                       "at 4096 tokens, r=64")
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


def dropout_timing(lib, synth, torch, dev, flush, p=0.05, reps=10):
    """The c2 forward + backward with LoRA dropout (p = 0.05, the tutorial's
    lora_dropout) against the same step without it; L2 flushed before each."""
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


def nf4_stream_timing(lib, synth, torch, dev, flush, reps=5):
    """Standalone quantise and dequantise of a 22016x8192 weight (larger than
    L2), L2 flushed before each launch; median of the per-launch event times."""
    big = synth.weight_bf16(22016, 8192, seed=99, device=dev)
    bcodes, bc8, bs2 = lib.nf4_quantize(big.reshape(-1))
    bout = torch.empty(big.numel(), dtype=torch.bfloat16, device=dev)
    lib.profile_enable(True)
    for _ in range(reps):
        flush.zero_()
        lib.nf4_quantize(big.reshape(-1), bcodes, bc8, bs2)
        flush.zero_()
        lib.nf4_dequantize(bcodes, bc8, bs2, big.numel(), out=bout)
    torch.cuda.synchronize()
    lib.profile_enable(False)
    qrec = lib.profile_collect()
    nbytes = big.numel() * NF4_BYTES_PER_PARAM
    qt = [t for n, t in qrec if n == "nf4_quantize"]
    dqt = [t for n, t in qrec if n == "nf4_dequantize"]
    return nbytes / (statistics.median(qt) * 1e-3) / 1e9, nbytes / (statistics.median(dqt) * 1e-3) / 1e9


# ------------------------------------------------------------------ arms

def run_reference(args, rank, world):
    """The CPU oracle as the reference arm (rank 0 only), on a bounded sample
    of the layer workload per step."""
    if rank != 0:
        return
    cores, blas = cpu_cores()
    times, vals = [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        v, dt, desc = cpu_oracle_layer_sample(m_s=128, n_s=256)
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
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "blas_threads": blas, "kind": "oracle",
                         "sample": desc},
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
    M = args.tokens
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    dd = dist if world > 1 else None
    peaks = load_peaks()

    # The standalone NF4 streams first: quantisation runs when a model is
    # loaded, not in the power-capped wake of a training step, and both
    # kernels are issue- or bandwidth-bound, so they follow the SM clock
    # (sampled beside them).
    nf4_extras = {}
    if rank == 0 and not args.no_sweep:
        quant_gbs, dequant_gbs, nf4_clocks = with_clocks(
            dev, lambda: nf4_stream_timing(lib, synth, torch, dev, flush))
        nf4_extras["nf4_quantize_gbs"] = quant_gbs
        nf4_extras["nf4_dequantize_gbs"] = dequant_gbs
        nf4_extras["nf4_hbm_frac"] = {"quantize": quant_gbs / peaks["hbm_gbs"],
                                      "dequantize": dequant_gbs / peaks["hbm_gbs"], "peak_gbs": peaks["hbm_gbs"],
                                      "peak_source": peaks["source"], "clocks": nf4_clocks,
                                      "when": "before the layer-step phases"}

    layer = LayerStep(lib, synth, torch, dev, M, rank, world, grouped=not args.no_group)

    for _ in range(args.warmup):
        flush.zero_()
        layer.step()
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
    step_ms = time_steps(torch, layer.step, stream, args.steps, flush, dd)
    lib.profile_enable(True)
    step_ms_profiled = time_steps(torch, layer.step, stream, args.steps, flush, dd)
    lib.profile_enable(False)
    clocks = sampler.stop()
    records = lib.profile_collect()
    ms = float(sum(step_ms) / len(step_ms))
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    assert int(layer.status[0].item()) == 0, f"device status {int(layer.status[0].item())}"

    kern = kernel_table(records, args.steps)
    tc = {n: k for n, k in kern.items() if n in ("fused_fwd", "fused_dx")}
    roofline = None
    if tc:
        dom = max(tc, key=lambda n: tc[n]["ms_total"])
        for n in tc:
            kern[n]["tflops"] = layer.kernel_flops(n) / (kern[n]["ms_per_step"] * 1e-3) / 1e12
        ach = kern[dom]["tflops"]
        # The kernel is timed inside a step of about 12 ms repeated back to
        # back, under the power cap: the sustained GEMM figure is its peak; the
        # fraction of the burst figure is reported beside it.
        pk = peaks["bf16_tflops_sustained"]
        roofline = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": pk,
                    "unit": "TFLOP/s", "frac": ach / pk, "traffic": NCU_TRAFFIC_BYTES.get(dom),
                    "peak_source": f"{peaks['source']} bf16 sustained (kernel timed inside the step)",
                    "frac_of_burst": ach / peaks["bf16_tflops"], "burst_peak": peaks["bf16_tflops"],
                    "launches_per_step": kern[dom]["launches"] // args.steps,
                    "achieved_from": "algorithmic FLOPs of the kernel's launches in a step / their summed "
                                     "event time per step (phase B)"}

    if args.kernels_only:
        if rank == 0:
            print(json.dumps({"kernels_only": True, "ms_per_step": ms,
                              "ms_per_step_profiled": float(np.mean(step_ms_profiled)), "kernels": kern}), flush=True)
        layer.close()
        return

    # ------------------------------------------------------------- e2e
    # The same step through the same API, with the step's inputs (the four
    # layer inputs and the seven upstream gradients) copied in from pinned
    # host memory and its result (the summed adapter gradients) copied back,
    # inside the timed region.  The inputs go over a second stream in the
    # order the step reads them, once the previous step's work is enqueued
    # (the device buffers are reused), and each call waits only for its own
    # inputs, so the copies overlap the calls before them.
    host_in = {f"X_{k}": (v, torch.empty_like(v, device="cpu").pin_memory()) for k, v in layer.X.items()}
    host_in.update({f"dY_{i}": (v, torch.empty_like(v, device="cpu").pin_memory()) for i, v in enumerate(layer.dY)})
    for dv, hv in host_in.values():
        hv.copy_(dv)
    host_out = [(g, torch.empty_like(g, device="cpu").pin_memory()) for g in layer.grad]
    h2d = sum(hv.numel() * hv.element_size() for _, hv in host_in.values())
    d2h = sum(hv.numel() * hv.element_size() for _, hv in host_out)

    copy_stream = torch.cuda.Stream(device=dev)
    order = layer.input_order()
    assert sorted(order) == sorted(host_in), (order, list(host_in))
    landed = {k: torch.cuda.Event() for k in order}

    def e2e_step():
        cs = torch.cuda.current_stream()
        copy_stream.wait_stream(cs)
        with torch.cuda.stream(copy_stream):
            for k in order:
                dv, hv = host_in[k]
                dv.copy_(hv, non_blocking=True)
                landed[k].record(copy_stream)
        layer.before_use = lambda k: cs.wait_event(landed[k])
        try:
            layer.step()
        finally:
            layer.before_use = None
        for dv, hv in host_out:
            hv.copy_(dv, non_blocking=True)

    for _ in range(2):
        e2e_step()
    e2e_ms = time_steps(torch, e2e_step, stream, max(3, args.steps // 4), flush, dd)
    e2e = float(np.mean(e2e_ms))
    if world > 1:
        t = torch.tensor([e2e], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e = float(t.item())
    fl = layer.flops()
    grouped = layer.grouped
    layer.close()
    del layer, host_in, host_out

    extras = {}
    if rank == 0 and not args.no_sweep and grouped:
        # Grouped against per-linear calls, timed in alternation (rounds of a
        # few steps each) so that both see the same clocks and power state.
        # Rank 0 alone runs this: its layers are single-GPU ones (world 1, no
        # gradient all-reduce that the other ranks would never join).
        flat = LayerStep(lib, synth, torch, dev, M, rank, 1, grouped=False)
        again = LayerStep(lib, synth, torch, dev, M, rank, 1, grouped=True)
        for _ in range(3):
            flat.step()
            again.step()
        tg, tf = [], []
        for _ in range(4):
            tg += time_steps(torch, again.step, stream, max(2, args.steps // 4), flush)
            tf += time_steps(torch, flat.step, stream, max(2, args.steps // 4), flush)
        gms, fms = float(np.mean(tg)), float(np.mean(tf))
        extras["grouping_ab"] = {"per_linear_ms_per_step": fms, "per_linear_tflops": fl / (fms * 1e-3) / 1e12,
                                 "grouped_ms_per_step": gms, "grouped_tflops": fl / (gms * 1e-3) / 1e12,
                                 "grouped_speedup": fms / gms,
                                 "timing": "4 alternating rounds of K/4 steps each, L2 flushed before every step"}
        flat.close()
        again.close()
        del flat, again
    if rank == 0 and not args.no_sweep:
        extras.update(nf4_extras)
        # Each secondary measurement carries the SM clock it ran at.
        for key, fn in (("c2_step", lambda: c2_step_timing(lib, synth, torch, dev, flush)),
                        ("adamw8", lambda: adamw8_timing(lib, synth, torch, dev, flush, peaks)),
                        ("lora_dropout", lambda: dropout_timing(lib, synth, torch, dev, flush)),
                        ("c5_forward", lambda: c5_forward_sweep(lib, synth, torch, dev, flush, peaks)),
                        ("c5_quantize_sweep", lambda: c5_quantize_sweep(lib, synth, torch, dev)),
                        ("c1_graph", lambda: c1_graph_timing(lib, synth, torch, dev)),
                        ("centered_dq", lambda: centered_cost(lib, synth, torch, dev, flush))):
            res, clk = with_clocks(dev, fn)
            res["clocks"] = clk
            extras[key] = res
        extras["c5_quantize_sweep"]["hbm_frac"] = extras["c5_quantize_sweep"]["quantize_gbs"] / peaks["hbm_gbs"]

    value = world * fl / (ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cores, blas = cpu_cores()
        v, dt, desc = cpu_oracle_layer_sample()
        rates = cpu_oracle_nf4_rates()
        cpu = {"value": v, "unit": "TFLOP/s", "cores": cores, "blas_threads": blas, "kind": "oracle",
               "sample": desc, "seconds": dt, "nf4": rates}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAME, "tokens_per_gpu": M, "r": RANK_R, "alpha": ALPHA,
                       "linears": [[lin.name, lin.n_out, lin.k_in] for lin in synth.LLAMA7B_LAYER],
                       "parallelism": f"dp{world}", "global_batch_tokens": M * world,
                       "grouped_projections": grouped,
                       "step": "nf4_quantize x7 + forward x7 + backward x7 (+ dA/dB all-reduce per linear if N>1) "
                               "+ 8-bit AdamW on every adapter",
                       "flops_per_step_per_gpu": fl,
                       "l2": "flushed before every step (512 MB memset outside the step's events)",
                       "pdl": os.environ.get("QLORA_PDL", "1") != "0"},
            "pct_bf16_peak": value / world / peaks["bf16_tflops"],
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": world * fl / (e2e * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "pinned host -> device on a second stream in the order the step reads its "
                              "inputs, each call waiting for its own; gradients device -> host after the step"},
            "gpu_launches": len(records),
            "timing": {"value_from": "phase A: K steps, step-level events only",
                       "kernels_from": "phase B: the same K steps with per-kernel event brackets",
                       "ms_per_step_phase_b": float(np.mean(step_ms_profiled)),
                       "ms_per_step_min": float(min(step_ms)), "ms_per_step_max": float(max(step_ms))},
            "clocks": clocks,
            "kernels": {n: {kk: round(vv, 5) if isinstance(vv, float) else vv for kk, vv in k.items()}
                        for n, k in sorted(kern.items(), key=lambda x: -x[1]["ms_total"])},
            "peaks": peaks,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)


def run_case(args):
    """Profiler driver: time one entry point on one shape (no JSON contract).

    --case fwd:M:N:K or bwd:M:N:K (r=64, alpha=16), quant:N:K / dequant:N:K (NF4
    quantisation / dequantisation of an N x K weight), cquant:N:K (the same with
    mean-centred double quantisation), adamw8:n (one 8-bit AdamW
    step over n parameters), or layer:M (the decoder-layer step with M tokens);
    --steps calls after 2 warm-up calls.
    """
    import torch

    import bit_nf4_quantized_26_b200 as lib
    import synth
    dev = torch.device("cuda", 0)
    if args.case.startswith("layer:"):
        M = int(args.case.split(":")[1])
        layer = LayerStep(lib, synth, torch, dev, M, grouped=not args.no_group)
        for _ in range(2 + args.steps):
            layer.step()
        torch.cuda.synchronize()
        layer.close()
        print(json.dumps({"case": args.case, "ok": True}))
        return
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
    if args.case.startswith("cquant:"):
        _, N, K = args.case.split(":")
        w = synth.weight_bf16(int(N), int(K), seed=1, device="cuda")
        for _ in range(2 + args.steps):
            lib.nf4_quantize_centered(w.view(-1))
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
    ap.add_argument("--tokens", type=int, default=M_TOKENS, help="tokens per GPU (default 8 x 2048)")
    ap.add_argument("--no-group", action="store_true", help="run every linear as its own call")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-sweep", action="store_true", help="skip the extra measurements after the headline")
    ap.add_argument("--kernels-only", action="store_true",
                    help="only the timed steps (for profiler captures): no e2e, no extras, no CPU baseline")
    ap.add_argument("--case", default=None,
                    help="profiler driver: fwd:M:N:K, bwd:M:N:K, quant:N:K, cquant:N:K, dequant:N:K, adamw8:n or layer:M")
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
