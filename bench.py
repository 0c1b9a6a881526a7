#!/usr/bin/env python3
"""Throughput of the OLMoE-shape MoE layer forward on B200.

Workload: one MoE layer with OLMoE's shapes, T=4096 tokens (one 4096-token
context), d_model 2048, 64 experts, top-8, SwiGLU width 1024, bf16 activations
and weights with fp32 accumulation; seeded synthetic inputs (unit-RMS token
rows, N(0, 0.02^2) weights). A step is one moe_forward: router, dispatch,
gate/up grouped GEMM with SwiGLU, down grouped GEMM, combine, and both losses.
Weights and tokens are resident in HBM; the 805 MB of expert weights read by
every step exceed the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

At N=1 the line also carries the other OLMoE-shape workloads, each timed on
the device: "decode" (T = 1, 8, 32, 64; CUDA-graph replays with the L2 flushed
before each, HBM GB/s of the touched experts' weights), "train" (T = 16384
forward + backward) and "stack" (16 layers, T = 8192, Zipf-skewed routing).

N > 1 runs as torchrun, one process per GPU, each on its own batch (weak
scaling, no data-path collective); the device time is the max over ranks and
`value` counts the tokens of all ranks. `--impl reference` times the fp64 CPU
oracle on the host cores on a bounded sample of the same workload.
Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and TFLOP/s (fwd, fwd+bwd) as % of bf16/HBM roofline on 1 B200"
UNIT = "tokens/s"
WORKLOAD = "OLMoE MoE layer forward, T=4096 (1x4096 context), d_model=2048, E=64, top-8, d_ff=1024, bf16"
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# router (which also ranks the dispatch), dispatch permute, gate/up GEMM, down GEMM,
# combine; plus one memset of the router's ticket word (not a kernel)
KERNELS_PER_STEP = 5


# ----------------------------------------------------------------------------- shapes


def layer_flops_per_token(d, E, k, f):
    """Router 2dE plus k experts of (gate/up 4df + down 2fd)."""
    return 2 * d * E + k * (4 * d * f + 2 * f * d)


def gate_up_flops(T, d, k, f):
    return 2.0 * T * k * d * (2 * f)


def layer_bytes(T, d, E, k, f, esize=2):
    """Algorithmic bytes of one forward: every expert's weights once (all are
    touched at this T), router weight, tokens in, output out, top-k out."""
    return E * 3 * d * f * esize + E * d * esize + 2 * T * d * esize + T * k * 8


# ----------------------------------------------------------------------------- ranks


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world, backend):
    if world <= 1:
        return None
    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


def reduce_max(dist, value, device="cpu"):
    """Max of a float over ranks (the measurement itself is per rank)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finish_line(rank, line):
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "gpu_idle": "nvmlClocksEventReasonGpuIdle",
        "applications_clocks_setting": "nvmlClocksEventReasonApplicationsClocksSetting",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "sync_boost": "nvmlClocksEventReasonSyncBoost",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, device_index, period_s=0.002):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # no NVML: report that, do not guess
            self.nv = None
            self.error = str(exc)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS.items():
                    if mask & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        return {
            "sm_mhz": statistics.median(self.samples) if self.samples else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": sorted(self.reasons - {"gpu_idle"}),
            "samples": len(self.samples),
        }


# ----------------------------------------------------------------------------- peaks


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return {k: p[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def committed_traffic(kernel_file, key):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, valid only
    while the kernel source is unchanged (sha256 recorded beside it)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "sparse_moe_transformer_route_b200", "csrc", kernel_file)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    with open(path) as fh:
        rec = json.load(fh).get(key)
    if not rec:
        return None
    with open(src, "rb") as fh:
        digest = hashlib.sha256(fh.read()).hexdigest()
    return rec.get("bytes_per_launch") if rec.get("source_sha256") == digest else None


# ----------------------------------------------------------------------------- oracle leg


def oracle_sample(n_tokens_max, budget_s, steps=None, seed=1):
    """Time the fp64 CPU oracle on contiguous token samples of the workload.

    Returns (tokens/s, tokens per sample, seconds per sample list, threads)."""
    import numpy as np
    import torch
    from oracle import moe_oracle as O
    from sparse_moe_transformer_route_b200 import synthetic as S

    inp = S.layer_inputs(S.PREFILL_4096, seed=seed)
    k = inp.shape.top_k
    x = inp.x.to(torch.float64).numpy()
    wr = inp.w_router.to(torch.float64).numpy()
    wgu = inp.w_gate_up.to(torch.float64).numpy()
    wd = inp.w_down.to(torch.float64).numpy()

    def one(t0, n):
        xs = x[t0:t0 + n]
        s = time.perf_counter()
        O.moe_forward(xs, wr, wgu, wd, k)
        return time.perf_counter() - s

    probe = 16
    one(0, probe)  # warm the BLAS threads
    per_tok = one(probe, probe) / probe
    n = int(max(probe, min(n_tokens_max, budget_s / max(per_tok, 1e-9))))
    times = []
    reps = steps if steps is not None else 1
    for i in range(reps):
        t0 = (i * n) % max(1, x.shape[0] - n + 1)
        times.append(one(t0, n))
    threads = 0
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 0) for i in threadpool_info()), default=0)
    except Exception:
        pass
    threads = threads or (os.cpu_count() or 1)
    return n / statistics.mean(times), n, times, threads


def workload_config(T, world, d=2048, E=64, k=8, f=1024):
    """The `config` object of the bench line (both arms)."""
    return {
        "workload": WORKLOAD if T == 4096 else WORKLOAD.replace("T=4096 (1x4096 context)", f"T={T}"),
        "T": T, "d_model": d, "n_experts": E, "top_k": k, "d_ff": f,
        "global_batch_tokens": world * T, "parallelism": f"replicas{world}",
        "l2": "no flush: each step reads 805 MB of expert weights, above the 126 MB L2",
    }


def run_reference(args, rank, world):
    """The reference arm: the oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    per_step_budget = max(1.0, 120.0 / max(1, args.steps + args.warmup))
    v, n, times, threads = oracle_sample(4096, per_step_budget, steps=args.steps + args.warmup)
    timed = times[args.warmup:] or times
    value = n / statistics.mean(timed)
    sample = f"{n} contiguous tokens of the T=4096 workload per step (routing, experts, losses), fp64"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.mean(timed) * 4096 / n,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": dict(workload_config(4096, world), sample_tokens=n),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    finish_line(rank, line)
    return 0


# ----------------------------------------------------------------------------- B200 leg


def _percentiles(xs):
    xs = sorted(xs)
    q = lambda f: xs[min(len(xs) - 1, int(f * (len(xs) - 1) + 0.5))]
    return statistics.median(xs), q(0.1), q(0.9)


def bench_decode(M, S, dev, weights, reps, peaks):
    """Decode-shaped layers (T = 1, 8, 32, 64): the forward captured in a CUDA
    graph and replayed, the L2 flushed before every replay so the touched
    experts' weights come from HBM. Algorithmic bytes: the touched experts'
    weights, the router weight, x, y and the top-k outputs."""
    import torch
    wr, wgu, wd = weights
    E, d = wr.shape
    f = wd.shape[2]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {}
    for T in S.DECODE_TOKENS:
        k = S.OLMOE_TOP_K
        x = S.make_tokens(S.LayerShape(T=T), seed=700 + T).to(dev)
        cfg = M.config(T, d, E, k, f)
        ws = M.workspace(cfg, False, dev)
        y = torch.empty_like(x)
        losses = torch.empty(2, device=dev)
        idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        wts = torch.empty(T, k, device=dev)
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            M.moe_forward(cfg, x, wr, None, wgu, wd, y, losses, idx, wts, False, ws)
            torch.cuda.synchronize(dev)
            with torch.cuda.graph(graph, stream=side):
                M.moe_forward(cfg, x, wr, None, wgu, wd, y, losses, idx, wts, False, ws)
        torch.cuda.current_stream(dev).wait_stream(side)
        for _ in range(5):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize(dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in evs:
            flush.zero_()
            a.record()
            graph.replay()
            b.record()
        torch.cuda.synchronize(dev)
        us = [a.elapsed_time(b) * 1e3 for a, b in evs]
        med, p10, p90 = _percentiles(us)
        touched = int(torch.unique(idx).numel())
        nbytes = touched * 3 * d * f * 2 + E * d * 2 + 2 * T * d * 2 + T * k * 8
        gbs = nbytes / (med * 1e-6) / 1e9
        status = M.moe_get_device_status(ws)
        if status != 0:
            raise RuntimeError(f"device check failed in the decode runs: 0x{status:x}")
        del graph
        out[f"T{T}"] = {
            "us_median": med, "us_p10": p10, "us_p90": p90, "replays": reps, "experts_touched": touched,
            "bytes": nbytes, "GB_per_s": gbs, "frac_of_8TBs": gbs / NOMINAL_HBM_GBS,
            "frac_of_measured_hbm": gbs / peaks["hbm_gbs"], "tokens_per_s": T / (med * 1e-6),
        }
    out["timing"] = "CUDA-graph replay of moe_forward, L2 flushed (256 MB write) before each replay"
    return out


def bench_decode_stack(M, S, dev, reps, peaks):
    """The 16-layer skewed stack at decode batch sizes (T = 1, 4, 8). Up to 4
    tokens one persistent launch walks all 16 layers (RMSNorm, routing, experts
    and the residual add of each); at 8 each layer runs the layered tensor-core
    path. The L2 is flushed before each call; bytes are the touched experts'
    weights of every layer plus the router weights."""
    import torch
    out = {}
    _, layers = S.stack_inputs(S.LayerShape(T=1), S.STACK_LAYERS, seed=8)
    layers = [{n: (v.to(dev) if v is not None else None) for n, v in L.items()} for L in layers]
    E, d = layers[0]["w_router"].shape
    f = layers[0]["w_down"].shape[2]
    k = S.OLMOE_TOP_K
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for T in (1, 4, 8):
        sh = S.LayerShape(T=T)
        x0 = S.make_tokens(sh, seed=90 + T, dtype=torch.float32, normalised=False).to(dev)
        cfg = M.config(T, d, E, k, f)
        ws = M.workspace(cfg, False, dev)
        resid = torch.empty_like(x0)
        idx = torch.empty(len(layers), T, k, dtype=torch.int32, device=dev)
        resid.copy_(x0)
        M.moe_stack_forward_trace(cfg, layers, resid, ws, topk_idx=idx)
        torch.cuda.synchronize(dev)
        touched = [int(torch.unique(idx[l]).numel()) for l in range(len(layers))]
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i in range(reps + 3):
            resid.copy_(x0)
            flush.zero_()
            if i >= 3:
                evs[i - 3][0].record()
            M.moe_stack_forward(cfg, layers, resid, ws)
            if i >= 3:
                evs[i - 3][1].record()
        torch.cuda.synchronize(dev)
        status = M.moe_get_device_status(ws)
        if status != 0:
            raise RuntimeError(f"device check failed in the decode stack: 0x{status:x}")
        us = [a.elapsed_time(b) * 1e3 for a, b in evs]
        med, p10, p90 = _percentiles(us)
        nbytes = sum(t * 3 * d * f * 2 for t in touched) + len(layers) * (E * d * 2 + 2 * T * d * 4)
        gbs = nbytes / (med * 1e-6) / 1e9
        out[f"T{T}"] = {
            "us_median": med, "us_p10": p10, "us_p90": p90, "us_per_layer": med / len(layers),
            "layers": len(layers), "experts_touched_per_layer": touched, "bytes": nbytes, "GB_per_s": gbs,
            "frac_of_8TBs": gbs / NOMINAL_HBM_GBS, "frac_of_measured_hbm": gbs / peaks["hbm_gbs"],
            "tokens_per_s": T / (med * 1e-6),
            "path": "one persistent launch" if T <= 4 else "layered, per layer",
        }
    out["timing"] = "CUDA events around one moe_stack_forward, L2 flushed (256 MB write) before each"
    return out


def bench_train(M, S, dev, steps, peaks):
    """One training step at T = 16384: moe_forward (saving for backward) and
    moe_backward, with the OLMoE loss weights, an N(0, 1) upstream gradient and
    fp32 weight gradients."""
    import torch
    sh = S.TRAIN_16384
    inp = S.layer_inputs(sh, seed=3, with_grad=True)
    T, d, E, k, f = sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff
    x, wr, wgu, wd, dy = (t.to(dev) for t in (inp.x, inp.w_router, inp.w_gate_up, inp.w_down, inp.dy))
    del inp
    cfg = M.config(T, d, E, k, f, alpha_lb=S.ALPHA_LB, beta_z=S.BETA_Z, grad_dtype=torch.float32)
    ws = M.workspace(cfg, True, dev)
    y = torch.empty_like(x)
    losses = torch.empty(2, device=dev)
    dx = torch.empty_like(x)
    dwr, dwgu, dwd = (torch.empty_like(t, dtype=torch.float32) for t in (wr, wgu, wd))

    def fwd():
        M.moe_forward(cfg, x, wr, None, wgu, wd, y, losses, None, None, True, ws)

    def bwd():
        M.moe_backward(cfg, dy, x, wr, wgu, wd, dx, dwr, dwgu, dwd, ws)

    for _ in range(3):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e0, e1, e2 in evs:
        e0.record()
        fwd()
        e1.record()
        bwd()
        e2.record()
    torch.cuda.synchronize(dev)
    status = M.moe_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device check failed in the training step: 0x{status:x}")
    f_ms = statistics.median(a.elapsed_time(b) for a, b, _ in evs)
    b_ms = statistics.median(b.elapsed_time(c) for _, b, c in evs)
    s_ms = statistics.median(a.elapsed_time(c) for a, _, c in evs)
    fl_fwd = layer_flops_per_token(d, E, k, f) * T
    # backward: twice the expert forward (data and weight gradients) plus the
    # router's two products (dx += dh W_r and dW_r = dh^T x)
    fl_bwd = 2.0 * k * (6 * d * f) * T + 4.0 * T * d * E
    peak = peaks["bf16_tflops"]
    return {
        "T": T, "ms_forward": f_ms, "ms_backward": b_ms, "ms_step": s_ms, "steps": steps,
        "tokens_per_s": T / (s_ms * 1e-3),
        "tflops_step": (fl_fwd + fl_bwd) / (s_ms * 1e-3) / 1e12,
        "tflops_forward": fl_fwd / (f_ms * 1e-3) / 1e12, "tflops_backward": fl_bwd / (b_ms * 1e-3) / 1e12,
        "frac_of_2250TF": (fl_fwd + fl_bwd) / (s_ms * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS,
        "frac_of_measured_bf16": (fl_fwd + fl_bwd) / (s_ms * 1e-3) / 1e12 / peak,
        "flops_step": fl_fwd + fl_bwd, "weight_grads": "fp32",
    }


def bench_stack(M, S, dev, steps, peaks):
    """The 16-layer skewed stack at T = 8192 (pre-RMSNorm, fp32 residual, Zipf
    router offset), each step from the same input residual."""
    import torch
    sh = S.STACK_8192
    T, d, E, k, f = sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff
    x0, layers = S.stack_inputs(sh, S.STACK_LAYERS, seed=8)
    x0 = x0.to(dev)
    layers = [{n: (v.to(dev) if v is not None else None) for n, v in L.items()} for L in layers]
    cfg = M.config(T, d, E, k, f)
    ws = M.workspace(cfg, False, dev)
    resid = torch.empty_like(x0)
    for _ in range(3):
        resid.copy_(x0)
        M.moe_stack_forward(cfg, layers, resid, ws)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        resid.copy_(x0)
        a.record()
        M.moe_stack_forward(cfg, layers, resid, ws)
        b.record()
    torch.cuda.synchronize(dev)
    status = M.moe_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device check failed in the stack: 0x{status:x}")
    ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    flops = S.STACK_LAYERS * layer_flops_per_token(d, E, k, f) * T
    return {
        "T": T, "layers": S.STACK_LAYERS, "ms": ms, "steps": steps, "tokens_per_s": T / (ms * 1e-3),
        "tflops": flops / (ms * 1e-3) / 1e12, "frac_of_2250TF": flops / (ms * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS,
        "frac_of_measured_bf16": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "flops": flops,
    }


def bench_expert_choice(M, S, dev, cfg, x, weights, steps, peaks, ms_token_choice):
    """The same T=4096 layer (weights, tokens) under expert-choice routing: every
    expert takes its C = T*k/E best tokens, so the expert GEMMs do the same work
    as token choice on perfectly even groups. CUDA events per stage, as the
    headline; inputs larger than L2 (805 MB of weights per step)."""
    import torch
    wr, wgu, wd = weights
    T, E = cfg.T, cfg.n_experts
    C = M.moe_expert_choice_capacity(cfg)
    ws = M.workspace(cfg, False, dev)
    y = torch.empty_like(x)
    losses = torch.empty(2, device=dev)
    for _ in range(3):
        M.moe_forward_expert_choice(cfg, x, wr, None, wgu, wd, y, losses, None, None, ws)
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(M.binding.STAGE_EVENTS)] for _ in range(steps)]
    for row in ev:
        for e in row:
            e.record()
    torch.cuda.synchronize(dev)
    for i in range(steps):
        M.moe_set_stage_events(ev[i])
        M.moe_forward_expert_choice(cfg, x, wr, None, wgu, wd, y, losses, None, None, ws)
    torch.cuda.synchronize(dev)
    status = M.moe_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device check failed under expert choice: 0x{status:x}")
    ms = statistics.median(ev[i][0].elapsed_time(ev[i][-1]) for i in range(steps))
    stage_ms = {name: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(steps))
                for j, name in enumerate(("router", "select_gather", "gate_up", "down", "combine"))}
    gu = 2.0 * E * C * cfg.d_model * 2 * cfg.d_ff
    return {
        "T": T, "capacity": C, "ms": ms, "steps": steps, "tokens_per_s": T / (ms * 1e-3),
        "stage_ms": stage_ms, "vs_token_choice": ms_token_choice / ms,
        "gate_up_tflops": gu / (stage_ms["gate_up"] * 1e-3) / 1e12,
        "gate_up_frac_of_measured": gu / (stage_ms["gate_up"] * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "timing": "CUDA events per stage, median over steps, no L2 flush (weights exceed L2)",
    }


def run_b200(args, rank, world, local):
    import torch
    import sparse_moe_transformer_route_b200 as M
    from sparse_moe_transformer_route_b200 import synthetic as S

    torch.cuda.set_device(local)
    dist = init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    sh = S.LayerShape(T=args.tokens)
    T, d, E, k, f = sh.T, sh.d_model, sh.n_experts, sh.top_k, sh.d_ff
    inp = S.layer_inputs(sh, seed=1 + rank)
    x = inp.x.to(dev)
    wr, wgu, wd = inp.w_router.to(dev), inp.w_gate_up.to(dev), inp.w_down.to(dev)
    cfg = M.config(T, d, E, k, f)
    ws = M.workspace(cfg, False, dev)
    y = torch.empty_like(x)
    losses = torch.empty(2, device=dev)

    expert_choice = args.routing == "expert"

    def step():
        if expert_choice:
            M.moe_forward_expert_choice(cfg, x, wr, None, wgu, wd, y, losses, None, None, ws)
        else:
            M.moe_forward(cfg, x, wr, None, wgu, wd, y, losses, None, None, False, ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    status = M.moe_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device check failed during warm-up: 0x{status:x}")

    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    barrier(dist, local)
    torch.cuda.synchronize()
    sampler.start()
    start.record()
    for i in range(K):
        step()
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(dist, local)
    ms = start.elapsed_time(end) / K
    ms_max = reduce_max(dist, ms, dev)

    # The same K steps again with CUDA events between the stages (on the
    # layer's stream), for the per-stage times and the gate/up kernel's duration;
    # kept out of the headline loop because an event between two kernels stops
    # the next one's launch from overlapping the previous one's tail.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(M.binding.STAGE_EVENTS)] for _ in range(K)]
    for row in ev:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    for i in range(K):
        M.moe_set_stage_events(ev[i])
        step()
    torch.cuda.synchronize()
    stage_ms = {}
    for s_, name in enumerate(M.binding.STAGES):
        stage_ms[name] = statistics.mean(ev[i][s_].elapsed_time(ev[i][s_ + 1]) for i in range(K))
    gate_up_ms = reduce_max(dist, stage_ms["gate_up"], dev)
    status = M.moe_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device check failed in the timed region: 0x{status:x}")

    # End to end through the host-buffer entry point: every step copies its
    # tokens in from pinned host memory, runs the layer and copies y and the
    # losses back. Two steps are in flight on two streams (each with its own
    # workspace and output buffers), so one step's transfers overlap the other's
    # kernels, as a serving loop would run it.
    streams = [torch.cuda.Stream(dev) for _ in range(2)]
    wss = [ws, M.workspace(cfg, False, dev)]
    xh = [inp.x.clone().pin_memory() for _ in range(2)]
    yh = [torch.empty_like(xh[0]).pin_memory() for _ in range(2)]
    lh = [torch.empty(2).pin_memory() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            j = i & 1
            M.moe_forward_host_async(cfg, xh[j], wr, None, wgu, wd, yh[j], lh[j], wss[j], stream=streams[j])
        for st_ in streams:
            st_.synchronize()

    e2e_steps(4)
    barrier(dist, local)
    t0 = time.perf_counter()
    e2e_steps(K)
    e2e_s = (time.perf_counter() - t0) / K
    e2e_s = reduce_max(dist, e2e_s, dev)
    for j in range(2):
        status = M.moe_get_device_status(wss[j])
        if status != 0:
            raise RuntimeError(f"device check failed in the end-to-end steps: 0x{status:x}")
    del wss, xh, yh, lh

    peaks, peak_src = measured_peaks()
    timed_region_s = ms * K / 1000.0
    burst = timed_region_s < 1.0
    peak_tf = peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]
    gu_flops = gate_up_flops(T, d, k, f)
    achieved = gu_flops / (gate_up_ms * 1e-3) / 1e12
    layer_flops = layer_flops_per_token(d, E, k, f) * T
    layer_tflops = layer_flops / (ms_max * 1e-3) / 1e12
    lbytes = layer_bytes(T, d, E, k, f)
    floor_ms_nominal = max(layer_flops / (NOMINAL_BF16_TFLOPS * 1e12), lbytes / (NOMINAL_HBM_GBS * 1e9)) * 1e3
    floor_ms_measured = max(layer_flops / (peak_tf * 1e12), lbytes / (peaks["hbm_gbs"] * 1e9)) * 1e3

    line = {
        "metric": METRIC,
        "value": world * T / (ms_max * 1e-3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(T, world, d, E, k, f),
        "tflops": layer_tflops,
        "layer_roofline": {
            "floor_ms_nominal": floor_ms_nominal, "frac_nominal": floor_ms_nominal / ms_max,
            "floor_ms_measured": floor_ms_measured, "frac_measured": floor_ms_measured / ms_max,
        },
        "stage_ms": stage_ms,
        "roofline": {
            "kernel": "grouped GEMM gate/up + SwiGLU (tcgen05)",
            "bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
            "frac": achieved / peak_tf, "traffic": committed_traffic("grouped_gemm.cu", "gate_up_T4096"),
            "peak_source": f"{peak_src} bf16_tflops{'' if burst else '_sustained'}",
        },
        "e2e": {
            "value": world * T / e2e_s, "unit": UNIT,
            "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2 + 8,
            "call": "moe_forward_host_async, pinned host buffers, two steps in flight on two streams",
            "timing": "host wall clock over K steps, both streams synchronised at the end",
        },
        "gpu_launches": (KERNELS_PER_STEP + (1 if expert_choice else 0)) * K,
        "clocks": clocks,
    }
    if expert_choice:
        line["config"]["routing"] = "expert choice (profiling run; the headline is token choice)"
    extras = [] if args.no_extras else [e for e in args.extras.split(",") if e]
    if world == 1 and extras:
        # the other OLMoE-shape workloads on this GPU, each reported beside the headline
        if "ec" in extras and not expert_choice:
            line["expert_choice"] = bench_expert_choice(M, S, dev, cfg, x, (wr, wgu, wd), 50, peaks, ms)
            torch.cuda.empty_cache()
        if "decode" in extras:
            line["decode"] = bench_decode(M, S, dev, (wr, wgu, wd), 200, peaks)
            torch.cuda.empty_cache()
        if "decode_stack" in extras:
            line["decode_stack"] = bench_decode_stack(M, S, dev, 50, peaks)
            torch.cuda.empty_cache()
        del x, wr, wgu, wd, ws, y
        torch.cuda.empty_cache()
        if "train" in extras:
            line["train"] = bench_train(M, S, dev, 10, peaks)
            torch.cuda.empty_cache()
        if "stack" in extras:
            line["stack"] = bench_stack(M, S, dev, 5, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, times, threads = oracle_sample(4096, args.cpu_budget / 2, steps=2)
        line["cpu_baseline"] = {
            "value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} contiguous tokens of the same workload, fp64 numpy, 2 repeats",
        }
    finish_line(rank, line)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("b200", "reference"), default="b200")
    ap.add_argument("--tokens", type=int, default=4096,
                    help="tokens per layer call (4096 is the benchmarked workload; others are for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the expert-choice, decode, training-step and 16-layer stack workloads (N=1 only)")
    ap.add_argument("--extras", default="ec,decode,decode_stack,train,stack",
                    help="comma list of the extra workloads to run at N=1 (ec, decode, decode_stack, train, stack)")
    ap.add_argument("--routing", choices=("token", "expert"), default="token",
                    help="token choice (OLMoE, the benchmarked layer) or expert choice (for profiling)")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_b200(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
