#!/usr/bin/env python
"""MoE-layer forward benchmark on B200: tokens/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one full moe_layer_forward (route, top-K, stats, dispatch, both
expert GEMMs, combine, bias update where the workload has one) over one batch
of T synthetic tokens whose inputs already sit in HBM.  Inputs (2.8 GB of
expert weights for the default Mixtral-shaped decode workload) are larger
than L2, so no flush is needed between steps.  With N > 1 (torchrun), every
rank runs an independent replica of the layer (the path has no exchange
step), timing is the max over ranks and ``value`` counts all ranks' tokens.

The headline is the Mixtral-shaped decode layer (T = 256).  The same JSON
line also carries a second-long ``sustained`` run of it (the power cap has
settled) and, on one GPU, a ``workloads`` entry for each other layer shape of
the metric: Mixtral prefill (T = 16384, tensor-bound), the Qwen-like layer
with capacity, and the DeepSeek-like layer whose steps update the bias in
place and draw fresh tokens (step j takes the tokens of seed step j mod 10).
A last entry runs the DeepSeek-shaped layer with its experts offloaded to
host memory as INT4 and an LRU cache on the GPU (16-token decode steps).
Timed regions carry no per-stage events; each is followed by as many steps
with an event between every two stages, which give the stage split (and the
expert-GEMM time of the roofline).

``--impl reference`` times the CPU oracle (the plain fp64 implementation the
tests check against) on the host cores on a bounded token sample per step;
under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_layer_gemm_b200 import synth  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200 (Mixtral shape decode/prefill); % of roofline"
# steps between the ones that carry per-stage events (working runs); the
# bench's own timed regions carry none, and their stage split comes from a
# second run with events on every step (see time_with_stages)
STAGE_EVERY = 4
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="mixtral_decode", choices=sorted(synth.workloads().keys()))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=0, help="end-to-end steps (0: as many as --steps)")
    p.add_argument("--cpu-sample-tokens", type=int, default=96,
                   help="tokens per oracle run of the CPU baseline (a bounded sample of the batch)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--chunk-tokens", type=int, default=0,
                   help="run the chunked layer (moe_layer_forward_chunked) in chunks of this many tokens")
    p.add_argument("--no-extra", action="store_true",
                   help="time only the headline workload (not prefill, capacity and bias-loop entries)")
    p.add_argument("--no-sustained", action="store_true", help="skip the second-long sustained run")
    p.add_argument("--tokens", type=int, default=0,
                   help="override the workload's T (smaller cases for profiling); recorded in config")
    p.add_argument("--experts", type=int, default=0,
                   help="profiling case: keep only the first N experts (T scaled to keep the mean group "
                        "size unless --tokens is given); recorded in config")
    return p.parse_args()


# --------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except FileNotFoundError:
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
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        loaded = [r for r in rows if r[1].replace(".", "").isdigit() and float(r[3] or 0) > 250.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[5 + i].lower() == "active"})
        sm_loaded = [float(r[1]) for r in loaded if r[1].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm_loaded or sm), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3])}


L2_BYTES = 126 * 1024 * 1024


def l2_note(wl) -> str:
    """How the timed steps relate to the 126 MB L2 (no flush between steps)."""
    wbytes = wl.E * 3 * wl.d_model * wl.d_ff * 2
    if wbytes > L2_BYTES:
        return "inputs larger than L2 (expert weights %.2f GB)" % (wbytes / 1e9)
    return "inputs fit in L2 (expert weights %.1f MB), not flushed between steps: a parity-size case" % (wbytes / 1e6)


def layer_algorithmic(wl, counts: np.ndarray, kept: np.ndarray):
    """Algorithmic bytes / FLOPs of one layer step and of its expert GEMMs.

    Layer: weights of every expert with >= 1 kept row (3 d f bf16) + x (bf16)
    + y (fp32) + W_r (bf16); FLOPs 2 T d E (router) + 6 d f N_kept.
    Expert GEMMs (gate/up + down, one kernel): the touched weights; FLOPs
    6 d f N_kept.  The activations the GEMM kernel moves by design (x_perm
    in, H out and back in, y_perm out) are reported apart, as
    gemm_design_bytes, and are not counted as algorithmic work.
    """
    T, d, f, E = wl.T, wl.d_model, wl.d_ff, wl.E
    n_kept = int(kept.sum())
    touched = int((kept > 0).sum())
    wbytes = touched * 3 * d * f * 2
    layer_bytes = wbytes + T * d * 2 + T * d * 4 + d * E * 2
    layer_flops = 2 * T * d * E + 6 * d * f * n_kept
    gemm_flops = 6 * d * f * n_kept
    design = n_kept * (d * 2 + 2 * f * 2 + d * 4)
    return dict(n_kept=n_kept, touched=touched, layer_bytes=layer_bytes, layer_flops=layer_flops,
                gemm_bytes=wbytes, gemm_design_bytes=design, gemm_flops=gemm_flops)


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of the expert-GEMM kernel from the committed ncu
    summary profiles/<kernel>_<workload>.txt, or None when it is missing or
    was taken on a different kernel source."""
    import hashlib
    stem = kernel[:-len("_kernel")] if kernel.endswith("_kernel") else kernel
    path = os.path.join(ROOT, "profiles", f"{stem}_{workload}.txt")
    try:
        vals = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
        src = os.path.join(ROOT, "moe_layer_gemm_b200", "csrc", vals["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if vals.get("source_sha256_16") != h:
            return None
        return int(float(vals["dram_bytes_per_launch"]))
    except Exception:
        return None


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (the value itself without a
    process group).  Multi-GPU timings are reported as the slowest rank."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(T: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own T tokens per step."""
    return T * world / (ms_per_step * 1e-3)


# --------------------------------------------------------------- oracle timing

def time_oracle(wl, x_h, Wr_h, W1_h, W3_h, W2_h, tokens, bias32=None, steps=1):
    """Wall time of the CPU oracle on a token sample (routing all T tokens)."""
    sys.path.insert(0, ROOT)
    from oracle import moe_oracle as O
    x64 = x_h.double().numpy()
    Wr64 = Wr_h.double().numpy()

    class Slab:
        def __init__(self, t):
            self.t = t
            self.shape = tuple(t.shape)

        def __getitem__(self, e):
            return self.t[int(e)].numpy()   # fp32 view; the oracle widens to fp64

    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        O.moe_layer(x64, Wr64, Slab(W1_h), Slab(W3_h), Slab(W2_h), wl.K, wl.capacity_factor,
                    bias32=bias32, alpha=wl.alpha, tokens=tokens)
        times.append(time.perf_counter() - t0)
    return times


def host_inputs(wl, device):
    """x, Wr, W1, W3, W2 as host fp32 tensors (generated where it is fastest)."""
    x = synth.make_x(wl, device=device)
    Wr = synth.make_router(wl, device=device)
    W1, W3, W2 = synth.make_expert_weights(wl, device=device)
    return [t.to("cpu", torch.float32) for t in (x, Wr, W1, W3, W2)]


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------- arms

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synth.get_workload(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x_h, Wr_h, W1_h, W3_h, W2_h = host_inputs(wl, dev)
    S = min(args.cpu_sample_tokens, wl.T)
    tokens = np.linspace(0, wl.T - 1, S).astype(int).tolist()
    bias = np.zeros(wl.E, np.float32) if wl.use_bias else None
    steps = max(1, min(args.steps, 5))
    warm = min(args.warmup, 1)
    if warm:
        time_oracle(wl, x_h, Wr_h, W1_h, W3_h, W2_h, tokens, bias, warm)
    times = time_oracle(wl, x_h, Wr_h, W1_h, W3_h, W2_h, tokens, bias, steps)
    sec = statistics.mean(times)
    value = S / sec
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": warm, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "d_model": wl.d_model, "d_ff": wl.d_ff, "E": wl.E, "K": wl.K,
                   "capacity_factor": wl.capacity_factor, "parallelism": f"replicas x{args.gpus}", "l2": l2_note(wl)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{S} of {wl.T} tokens per step (routing, counts and capacity over all "
                                   f"{wl.T}); {steps} steps after {warm} warm-up (of {args.steps}/{args.warmup} "
                                   f"asked, bounded to minutes); numpy fp64 with the BLAS threads given in cores"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class Layer:
    """One workload's inputs, packed weights, workspace and outputs on the
    device, and the call that runs one step of the layer."""

    def __init__(self, wl, dev, chunk: int = 0, keep_host: bool = False):
        from moe_layer_gemm_b200 import abi
        self.abi = abi
        self.wl = wl
        self.dev = dev
        self.chunk = chunk
        self.dims = abi.Dims(wl.T, wl.d_model, wl.d_ff, wl.E, wl.K, wl.capacity_factor)
        # workloads with per-step tokens (the bias loop) draw fresh x each
        # step: step j uses the tokens of seed step j (cycled over wl.steps)
        nx = wl.steps if wl.steps > 1 else 1
        self.xs = [synth.make_x(wl, j, device=dev)[: wl.T].contiguous() for j in range(nx)]
        self.Wr = synth.make_router(wl, device=dev)
        W1, W3, W2 = synth.make_expert_weights(wl, device=dev)
        self.W13p, self.W2p = abi.pack_weights(self.dims, W1, W3, W2)
        torch.cuda.synchronize()
        self.host = None
        if keep_host:
            self.host = [t.to("cpu", torch.float32) for t in (self.xs[0], self.Wr, W1, W3, W2)]
        del W1, W3, W2
        torch.cuda.empty_cache()
        self.ws = abi.alloc_chunked_workspace(self.dims, chunk, dev) if chunk > 0 else abi.alloc_workspace(self.dims, dev)
        self.y = torch.empty(wl.T, wl.d_model, dtype=torch.float32, device=dev)
        E = wl.E
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.outs = dict(counts=torch.zeros(E, **i32), kept=torch.zeros(E, **i32), n_dropped=torch.zeros(1, **i32),
                         f=torch.zeros(E, **f32), P=torch.zeros(E, **f32), aux=torch.zeros(1, **f32))
        self.bias = torch.zeros(E, **f32) if wl.use_bias else None
        self.alpha = float(wl.alpha) if wl.use_bias else 0.0

    def run(self, x_in, y_out, evs=None):
        abi = self.abi
        if self.chunk > 0:   # per-stage events are not recorded by the chunked layer
            abi.moe_layer_forward_chunked(self.dims, self.chunk, x_in, self.Wr, self.bias, self.alpha, self.W13p,
                                          self.W2p, y_out, self.ws, self.outs)
        else:
            abi.moe_layer_forward(self.dims, x_in, self.Wr, self.bias, self.alpha, self.W13p, self.W2p, y_out,
                                  self.ws, self.outs, stage_events=evs)

    def step(self, i, evs=None):
        self.run(self.xs[i % len(self.xs)], self.y, evs)

    def launches(self) -> int:
        stats, upd = True, self.bias is not None and self.alpha != 0.0
        if self.chunk > 0:
            return self.abi.moe_layer_chunked_launch_count(self.dims, self.chunk, stats, upd)
        return self.abi.moe_layer_launch_count(self.dims, stats, upd)

    def check_status(self, where: str):
        st, detail = self.abi.moe_get_device_status(self.ws)
        if st != 0:
            raise RuntimeError(f"device-side status {st} ({detail}) {where}")


# per-stage events: [0] before routing, [1] after routing, [2] after
# dispatch, [3] after the expert GEMMs, [4] after the combine (whose extra
# CTA also computes the statistics and the bias update; event [5] marks the
# same point and is not reported)
STAGES = ("route", "dispatch", "expert_gemms", "combine_stats")


def time_steps(layer: Layer, K: int, barrier, clock_index: int, stage_every=None, start_step: int = 0):
    """Time K layer steps with CUDA events on the launching stream (barrier
    and device synchronisation on both sides); per-stage events ride on every
    stage_every-th step (an event between two kernels keeps the second from
    starting early, so the other steps run without them).  Clocks are
    sampled during the region."""
    from moe_layer_gemm_b200 import abi
    nev = abi.NUM_STAGE_EVENTS
    if stage_every is None:
        stage_every = 1 if len(layer.xs) > 1 else STAGE_EVERY
    sampled = list(range(0, K, stage_every)) if layer.chunk == 0 and stage_every > 0 else []
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(nev)] for i in sampled}
    s = torch.cuda.current_stream()
    for row in evs.values():   # create the underlying events before the timed region
        for e in row:
            e.record(s)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.reset_peak_memory_stats(layer.dev)
    clocks = ClockSampler(clock_index)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    start.record(s)
    for i in range(K):
        layer.step(start_step + i, evs.get(i))
    end.record(s)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms_total = max_over_ranks(start.elapsed_time(end), layer.dev)
    stage_ms = None
    if sampled:
        st = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(len(STAGES))] for i in sampled])
        stage_ms = st.mean(axis=0)
    layer.check_status("in the timed region")
    return dict(ms_total=ms_total, ms_step=ms_total / K, stage_ms=stage_ms, clocks=clk,
                peak_bytes=int(torch.cuda.max_memory_allocated(layer.dev)))


def time_with_stages(layer: Layer, K: int, barrier, clock_index: int, start_step: int, n_staged: int = 0):
    """The timed region (K steps, no per-stage events: an event between two
    kernels costs a few microseconds per step), then n_staged (default K)
    more steps with events on every step for the stage split, which covers
    every token set of a workload that draws fresh tokens per step."""
    res = time_steps(layer, K, barrier, clock_index, stage_every=0, start_step=start_step)
    if layer.chunk == 0:
        n = n_staged if n_staged > 0 else K
        st = time_steps(layer, n, barrier, clock_index, stage_every=1, start_step=start_step + K)
        res["stage_ms"] = st["stage_ms"]
        res["staged_ms_step"] = st["ms_step"]
    return res


def roofline_of(layer: Layer, res: dict, peaks: dict, peak_src: str):
    """The expert-GEMM roofline (touched weight bytes or FLOPs over the
    kernel's event-timed duration) and the layer roofline of one timed run."""
    from moe_layer_gemm_b200 import abi
    wl = layer.wl
    counts = layer.outs["counts"].cpu().numpy()
    kept = layer.outs["kept"].cpu().numpy()
    alg = layer_algorithmic(wl, counts, kept)
    ms_step, stage_ms = res["ms_step"], res["stage_ms"]
    sustained = res["ms_total"] > 1000.0
    tensor_peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    tensor_src = peak_src + (" sustained" if sustained else " burst")
    bw = peaks["hbm_gbs"]
    t_bytes = alg["layer_bytes"] / (bw * 1e9)
    t_flops = alg["layer_flops"] / (tensor_peak * 1e12)
    layer_roof = {"bound": "hbm" if t_bytes >= t_flops else "tensor", "t_roof_ms": max(t_bytes, t_flops) * 1e3,
                  "t_meas_ms": ms_step, "frac": max(t_bytes, t_flops) * 1e3 / ms_step, "bytes": alg["layer_bytes"],
                  "flops": alg["layer_flops"]}
    # the expert GEMMs' own work and time; the chunked layer records no
    # per-stage events, so there the whole layer's work over its time
    per_stage = stage_ms is not None
    gemm_ms = float(stage_ms[2]) if per_stage else ms_step
    w_bytes = alg["gemm_bytes"] if per_stage else alg["layer_bytes"]
    w_flops = alg["gemm_flops"] if per_stage else alg["layer_flops"]
    if w_bytes / (bw * 1e9) >= w_flops / (tensor_peak * 1e12):
        achieved = w_bytes / (gemm_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": bw, "unit": "GB/s", "frac": achieved / bw,
                "peak_source": f"{peak_src} copy bandwidth"}
    else:
        achieved = w_flops / (gemm_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": achieved / tensor_peak, "peak_source": f"{tensor_src} bf16 GEMM"}
    kernel = abi.moe_ffn_kernel(layer.dims)
    full = synth.get_workload(wl.name)
    traffic = profile_traffic(kernel, wl.name) if layer.chunk == 0 and (wl.T, wl.E) == (full.T, full.E) else None
    roof.update({
        "traffic": traffic,
        "kernel": (f"{kernel} (gate/up and down in one launch)" if per_stage else
                   f"whole chunked layer (no per-stage events; {kernel} once per chunk)"),
        "algorithmic_per_step": w_bytes if roof["bound"] == "hbm" else w_flops,
        "algorithmic_what": ("touched expert weights (bytes)" if roof["bound"] == "hbm" else
                             "6 d_model d_ff N_kept (FLOPs)") if per_stage else "whole layer",
        "design_activation_bytes": alg["gemm_design_bytes"] if per_stage else None,
        "ms_per_step": gemm_ms})
    routing = {"n_kept": alg["n_kept"], "experts_touched": alg["touched"],
               "max_over_mean_load": float(counts.max() / (wl.T * wl.K / wl.E)),
               "count_cv": float(counts.std() / counts.mean()), "n_dropped": int(layer.outs["n_dropped"].item())}
    return roof, layer_roof, routing


def stage_dict(stage_ms):
    return None if stage_ms is None else {k: float(v) for k, v in zip(STAGES, stage_ms)}


EXTRA_WORKLOADS = ("mixtral_prefill", "qwen_capacity", "deepseek_bias")

# Expert offloading: the DeepSeek-shaped layer at a decode batch of 16 tokens
# (about 65 distinct experts a step), 160 of its 256 experts cached on the GPU
OFFLOAD_TOKENS = 16
OFFLOAD_SLOTS = 160
OFFLOAD_PREFETCH = 32


def run_offload_entry(dev, steps: int, warmup: int, barrier, clock_index: int):
    """The DeepSeek-shaped layer at a decode batch with its experts offloaded:
    all 256 experts in page-locked host memory as group-wise INT4, a cache of
    OFFLOAD_SLOTS experts on the GPU, OFFLOAD_PREFETCH predicted experts
    loaded ahead after each step; every step draws fresh tokens."""
    from moe_layer_gemm_b200 import abi
    from moe_layer_gemm_b200.offload import OffloadedLayer, quantize_experts_to_host
    wl = synth.get_workload("deepseek_bias")
    T = OFFLOAD_TOKENS
    dims = abi.Dims(T, wl.d_model, wl.d_ff, wl.E, wl.K)
    Wr = synth.make_router(wl, device=dev)
    W1, W3, W2 = synth.make_expert_weights(wl, device=dev)
    q = quantize_experts_to_host(dims, W1, W3, W2)
    del W1, W3, W2
    torch.cuda.empty_cache()
    layer = OffloadedLayer(dims, Wr, *q, n_slots=OFFLOAD_SLOTS, prefetch=OFFLOAD_PREFETCH)
    xs = [synth.normal_bf16((T, wl.d_model), 7000 + j, synth.STREAM_X, wl.x_std, dev) for j in range(warmup + steps)]
    y = torch.empty(T, wl.d_model, dtype=torch.float32, device=dev)
    for j in range(warmup):
        layer.forward(xs[j], y)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s = torch.cuda.current_stream()
    clocks = ClockSampler(clock_index)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start.record(s)
    for j in range(steps):
        layer.forward(xs[warmup + j], y)
    end.record(s)
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) * 1e3 / steps
    clk = clocks.stop()
    ms = start.elapsed_time(end) / steps
    recs = layer.log[warmup:]
    need = sum(len(r["needed"]) for r in recs)
    hits = sum(len(r["hits"]) for r in recs)
    phits = sum(len(r["prefetch_hits"]) for r in recs)
    miss = sum(len(r["misses"]) for r in recs)
    host_bytes = sum(r["unpacked_bytes"] for r in recs) / steps
    return {"value": T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps, "warmup": warmup,
            "config": {"T": T, "d_model": wl.d_model, "d_ff": wl.d_ff, "E": wl.E, "K": wl.K, "cache_slots": OFFLOAD_SLOTS,
                       "prefetch": OFFLOAD_PREFETCH, "int4_bytes_per_expert": layer.bytes_per_expert,
                       "bf16_bytes_per_expert": 3 * wl.d_model * wl.d_ff * 2, "fresh_tokens_per_step": True},
            "cache": {"needed_per_step": need / steps, "hit_rate": (hits + phits) / max(need, 1),
                      "resident_hit_rate": hits / max(need, 1), "prefetch_hit_rate": phits / max(need, 1),
                      "misses_per_step": miss / steps},
            "host_link": {"bytes_per_step": host_bytes, "GB_per_s": host_bytes / (ms * 1e-3) / 1e9},
            "host_ms_per_step": wall, "clocks": clk}



def run_ours(args):
    from moe_layer_gemm_b200 import abi
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = False
    if world > 1:
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
        pg = True

    def barrier():
        if pg:
            torch.distributed.barrier()

    peaks, peak_src = load_peaks()
    wl = synth.get_workload(args.workload)
    if args.experts > 0:
        if args.experts < wl.K:
            raise SystemExit("--experts must be at least the workload's K")
        wl.T = max(1, wl.T * args.experts // wl.E)
        wl.E = args.experts
    if args.tokens > 0:
        wl.T = args.tokens
    reduced = args.tokens > 0 or args.experts > 0
    chunk = args.chunk_tokens
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline and not reduced
    layer = Layer(wl, dev, chunk, keep_host=want_cpu)
    abi.moe_reset_device_status(layer.ws)
    for i in range(args.warmup):
        layer.step(i)
    torch.cuda.synchronize()
    layer.check_status("during warm-up")

    # ---- timed region: K steps of the headline workload
    K = args.steps
    res = time_with_stages(layer, K, barrier, local, start_step=args.warmup)
    roof, layer_roof, routing = roofline_of(layer, res, peaks, peak_src)
    ms_step = res["ms_step"]

    # ---- the same workload over at least a second of steps (the power cap
    # settles in): its own timed region and clock record
    sustained = None
    if not args.no_sustained and chunk == 0:
        n_sus = max(K, int(np.ceil(1100.0 / max(ms_step, 1e-3))))
        rs = time_with_stages(layer, n_sus, barrier, local, start_step=args.warmup + 2 * K, n_staged=K)
        r2, l2, _ = roofline_of(layer, rs, peaks, peak_src)
        sustained = {"steps": n_sus, "ms_per_step": rs["ms_step"],
                     "value": job_tokens_per_s(wl.T, world, rs["ms_step"]), "timed_ms": rs["ms_total"],
                     "roofline_frac": r2["frac"], "roofline_bound": r2["bound"], "gemm_ms": r2["ms_per_step"],
                     "layer_roofline_frac": l2["frac"], "stage_ms": stage_dict(rs["stage_ms"]),
                     "clocks": rs["clocks"]}

    # ---- end to end through the public API with host buffers: every step
    # copies its input in from pinned host memory and its result y back out.
    # Two buffer sets and two copy streams pipeline the copies of one step
    # with the layer of another, as a serving loop would.
    s = torch.cuda.current_stream()
    x0 = layer.xs[0]
    x_host = [xx.cpu().pin_memory() for xx in layer.xs]
    y_host = [torch.empty(wl.T, wl.d_model, dtype=torch.float32).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x0) for _ in range(2)]
    y_dev = [torch.empty_like(layer.y) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):
        ev_done[b].record(s)
        ev_out[b].record(s)
    E2E = max(1, args.e2e_steps if args.e2e_steps > 0 else K)

    def e2e_step(i):
        b = i % 2
        s_in.wait_event(ev_done[b])          # x_dev[b] no longer read by step i - 2
        with torch.cuda.stream(s_in):
            x_dev[b].copy_(x_host[i % len(x_host)], non_blocking=True)
        ev_in[b].record(s_in)
        s.wait_event(ev_in[b])
        s.wait_event(ev_out[b])               # y_dev[b] copied out by step i - 2
        layer.run(x_dev[b], y_dev[b])
        ev_done[b].record(s)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            y_host[b].copy_(y_dev[b], non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    s_in.wait_event(e0)
    for i in range(E2E):
        e2e_step(i)
    for b in range(2):
        s.wait_event(ev_out[b])
    e1.record(s)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / E2E, dev)
    layer.check_status("in the end-to-end steps")
    launches = layer.launches() * K

    cpu = None
    if layer.host is not None:
        S = min(args.cpu_sample_tokens, wl.T)
        tokens = np.linspace(0, wl.T - 1, S).astype(int).tolist()
        b32 = np.zeros(wl.E, np.float32) if wl.use_bias else None
        times = time_oracle(wl, *layer.host, tokens, b32, steps=2)
        sec = min(times)
        cpu = {"value": S / sec, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"{S} of {wl.T} tokens (routing over all {wl.T}), best of 2 runs of {sec:.1f}-"
                         f"{max(times):.1f} s; numpy fp64 with the BLAS threads given in cores"}
    line_cfg = {"workload": wl.name, "T": wl.T, "d_model": wl.d_model, "d_ff": wl.d_ff, "E": wl.E, "K": wl.K,
                "capacity_factor": wl.capacity_factor, "parallelism": f"replicas x{world}",
                "l2": l2_note(wl), **({"chunk_tokens": chunk} if chunk > 0 else {}),
                **({"reduced_for_profiling": True} if reduced else {})}
    memory = {"workspace_bytes": int(layer.ws.numel()), "peak_device_bytes": res["peak_bytes"],
              **({"workspace_bytes_whole_batch": abi.moe_workspace_size(layer.dims)} if chunk > 0 else {})}
    del layer, x_host, y_host, x_dev, y_dev
    torch.cuda.empty_cache()

    # ---- the other workloads of the metric (prefill, capacity, bias loop):
    # same step, same timing, one entry each; 1-GPU runs only
    extras = {}
    if world == 1 and not args.no_extra and args.workload == "mixtral_decode" and not reduced and chunk == 0:
        for name in EXTRA_WORKLOADS:
            wx = synth.get_workload(name)
            lx = Layer(wx, dev)
            abi.moe_reset_device_status(lx.ws)
            for i in range(args.warmup):
                lx.step(i)
            torch.cuda.synchronize()
            lx.check_status(f"during warm-up ({name})")
            rx = time_with_stages(lx, K, barrier, local, start_step=args.warmup)
            rf, lr, rt = roofline_of(lx, rx, peaks, peak_src)
            extras[name] = {"value": job_tokens_per_s(wx.T, world, rx["ms_step"]), "unit": "tokens/s",
                            "ms_per_step": rx["ms_step"], "steps": K, "warmup": args.warmup,
                            "config": {"T": wx.T, "d_model": wx.d_model, "d_ff": wx.d_ff, "E": wx.E, "K": wx.K,
                                       "capacity_factor": wx.capacity_factor, "bias_update": wx.use_bias,
                                       "fresh_tokens_per_step": len(lx.xs) > 1, "l2": l2_note(wx)},
                            "roofline": rf, "layer_roofline": lr, "stage_ms": stage_dict(rx["stage_ms"]),
                            "routing": rt, "clocks": rx["clocks"], "gpu_launches_per_step": lx.launches()}
            del lx
            torch.cuda.empty_cache()
        extras["deepseek_offload"] = run_offload_entry(dev, max(1, min(K, 20)), max(3, min(args.warmup, 5)), barrier,
                                                       local)
        torch.cuda.empty_cache()

    if pg:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    value = job_tokens_per_s(wl.T, world, ms_step)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": line_cfg,
        "memory": memory,
        "roofline": roof,
        "layer_roofline": layer_roof,
        "stage_ms": stage_dict(res["stage_ms"]),
        "routing": routing,
        "sustained": sustained,
        "cpu_baseline": cpu,
        "e2e": {"value": job_tokens_per_s(wl.T, world, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x0.numel() * 2), "d2h_bytes_per_step": int(wl.T * wl.d_model * 4)},
        "gpu_launches": launches,
        "clocks": res["clocks"],
        "workloads": extras or None,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
