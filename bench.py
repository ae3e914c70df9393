#!/usr/bin/env python
"""Throughput of the DeepSeekMoE layer forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload dsv3]

A step is one pass of the whole hot path over one batch: router + top-K,
1x128 quantisation, permutation, routed grouped GEMMs (SwiGLU + requant fused),
shared expert, combine, and the per-batch expert-bias update (written to a
separate buffer, so every step routes with the configured bias b = 0).  Inputs are
synthetic (seeded) with the DeepSeek-V3 layer shape: T=4096 tokens, hidden 7168,
256 routed + 1 shared expert, top-8 with 8 groups / 4 kept, expert intermediate
2048, routed_scaling_factor 2.5; all 257 experts' E4M3 weights (11.3 GB) are
resident in HBM, far larger than L2, so no L2 flush is needed between steps.

Multi-GPU: replicas only (the layer is timed on each GPU independently; value
is the tokens of all ranks divided by the slowest rank's time).

--impl reference times the CPU float64 oracle on the host cores instead (a
bounded sample of the same workload, scaled to tokens/s).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE layer tokens/s at DSV3 shape; grouped FP8 GEMM TFLOP/s & % of peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(s: synth.MoEShape) -> str:
    return (f"{s.name}: T={s.T} H={s.H} E={s.E}+1 shared K={s.K} groups {s.n_group}/{s.topk_group} "
            f"I={s.I} rho={s.rho}")


# ----------------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def reduce_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.start = 0          # samples written before the region began
        self.after = False      # the region held no sample: the next one is used

    def _lines(self) -> int:
        try:
            with open(self.path) as f:
                return f.read().count("\n")
        except OSError:
            return 0

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # nvidia-smi takes a moment to start: wait (bounded) for its first
        # sample, so that every sample after `start` falls in the region
        deadline = time.time() + 10.0
        while self.proc is not None and self.proc.poll() is None and self._lines() == 0 \
                and time.time() < deadline:
            time.sleep(0.02)
        self.start = self._lines()
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            # a region shorter than the 200 ms period may hold no sample; then
            # the first sample after it (at most 200 ms later) stands for it
            deadline = time.time() + 1.0
            while self._lines() <= self.start and self.proc.poll() is None and time.time() < deadline:
                self.after = True
                time.sleep(0.01)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path).readlines()[self.start:]:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        loaded = [v for v in sm if mx and v > 0.5 * max(mx)] or sm
        out = {"sm_mhz": statistics.median(loaded) if loaded else None,
               "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}
        if self.after:
            out["window"] = "region shorter than the 200 ms sampling period: the first sample after it"
        return out


# ----------------------------------------------------------------- GPU arm
def build_layer(shape: synth.MoEShape, T: int, qw=None, offset=None):
    """The layer of `shape` for T tokens: its router and bias from the shape's
    seeds; expert weights drawn and quantised here unless `qw` (the resident
    E4M3 weights of another layer of the same sizes) is given."""
    import sparse_moe_layer_group_b200 as moe
    H, E, I = shape.H, shape.E, shape.I

    def master(kind, e):
        if e < 0:
            tid = synth.SH13 if kind == "w13" else synth.SH2
        else:
            tid = synth.W13 if kind == "w13" else synth.W2
        rows, cols = (2 * I, H) if kind == "w13" else (H, I)
        return synth.expert_weight(rows, cols, shape.w_std, synth.seed_of(shape, tid, max(e, 0)), device="cuda")

    if qw is None:
        qw = moe.QuantWeights.from_master(master, E, H, I, device="cuda")
    wr = synth.router_weights(E, H, shape.wr_std, synth.seed_of(shape, synth.WR), device="cuda")
    b = synth.expert_bias(E, shape.bias_range, synth.seed_of(shape, synth.BIAS), device="cuda")
    layer = moe.MoELayer(T, H, E, shape.K, shape.n_group, shape.topk_group, I, shape.rho, wr, b, qw,
                         router_offset=offset)
    return layer


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "grouped_gemm_w13_dsv3_traffic.txt")
# the grouped GEMM's code (the header only declares entry points, so new ones
# elsewhere do not mark the record stale)
GEMM_SOURCES = ("sparse_moe_layer_group_b200/csrc/common.cuh", "sparse_moe_layer_group_b200/csrc/tc_util.cuh",
                "sparse_moe_layer_group_b200/csrc/gemm_fp8.cu")


def gemm_sources_sha256() -> str:
    """sha256 of the GEMM's sources with comments and blank space removed, so
    that an edit of comments alone does not mark the traffic record stale."""
    import re
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(os.path.join(ROOT, p)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("".join(src.split()).encode())
    return h.hexdigest()


def recorded_w13_traffic(algorithmic_bytes: int):
    """DRAM bytes (read + write) of one W13 launch from the committed ncu record,
    or None when the kernel's sources changed since the record was taken or the
    record is for another workload (different algorithmic bytes)."""
    try:
        with open(TRAFFIC_RECORD) as f:
            lines = f.read().splitlines()
        digest = gemm_sources_sha256()
    except OSError:
        return None
    rec = dict(l.split(": ", 1) for l in lines if l and not l.startswith("#") and ": " in l)
    if rec.get("kernel_sources_sha256") != digest:
        return None
    if int(rec.get("algorithmic_bytes_per_launch", -1)) != algorithmic_bytes:
        return None
    return int(rec["traffic_bytes_per_launch"])


def gemm1_bytes(layer, touched: int) -> int:
    """Algorithmic HBM bytes of the W13 grouped GEMM launch: W13 of the touched
    routed experts and of the shared expert, the A rows it reads (codes +
    scales: the T token rows when it gathers them, else the T*K + T rows of the
    permuted copy) and the requantised output rows (codes + scales)."""
    T, H, K, I = layer.T, layer.H, layer.K, layer.I
    w = (touched + 1) * (2 * I * H + (2 * I // 128) * (H // 128) * 4)
    a = (T if layer.gather else T * K + T) * (H + (H // 128) * 4)
    o = (T * K + T) * (I + (I // 128) * 4)
    return w + a + o


def run_gpu(args, rank, world, local):
    import sparse_moe_layer_group_b200 as moe
    shape = synth.DSV3
    T = shape.T
    torch.cuda.set_device(local)
    layer = build_layer(shape, T)
    gamma = 0.001
    x = synth.activations(T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac, device="cuda")
    stream = torch.cuda.current_stream()
    pk, pk_kind = peaks()

    # the GEMM launches are bracketed with events on the same stream
    g_events = []
    b_next = layer.e_bias.clone()

    def step(record=False):
        ev = None
        if record:
            ev = tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
            g_events.append(ev)
        layer.forward(x, gemm_events=ev)
        # the bias update runs every step; its result goes to b_next so the
        # workload keeps the configured routing bias b = 0
        layer.bias_update(gamma, bias=b_next)

    launches_per_step = layer.launches_per_forward + 1
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step(record=True)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    ms_max = reduce_max(ms, world)
    status = int(layer.status.item())
    g1_ms = sum(a.elapsed_time(b) for a, b, _ in g_events) / len(g_events)
    g2_ms = sum(b.elapsed_time(c) for _, b, c in g_events) / len(g_events)
    load = layer.load.cpu().numpy()
    touched = int((load > 0).sum())
    seq_loss, entropy = layer.balance_stats(T, 0.001)     # one 4096-token sequence per step
    balance = {"max_over_mean_load": round(float(load.max() / load.mean()), 3),
               "load_entropy": round(float(entropy.item()), 5), "uniform_entropy": round(float(np.log(layer.E)), 5),
               "seq_balance_loss": float(seq_loss[0].item())}

    # end to end through the C ABI with host buffers: moe_layer_run_host takes K
    # pinned host batches (four distinct seeded batches in rotation), uploads
    # each on a stream of its own, runs the forward and the bias update on the
    # compute stream and downloads each output on a third stream, the copies of
    # neighbouring steps overlapping each forward (device input and output
    # double-buffered)
    n_src = 4
    x_src = [x.cpu().pin_memory()] + [
        synth.activations(T, shape.H, synth.seed_of(shape, synth.X) + 1000 + i, shape.x_outlier_frac).pin_memory()
        for i in range(n_src - 1)]
    out_host = [torch.empty(T, shape.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x), torch.empty_like(x)]
    out_dev = [torch.empty_like(x), torch.empty_like(x)]

    def e2e_steps(n):
        layer.run_host([x_src[i % n_src] for i in range(n)], [out_host[i % 2] for i in range(n)], x_dev, out_dev,
                       stream=stream, bias_out=b_next, gamma=gamma)

    e2e_steps(max(1, args.warmup))
    torch.cuda.synchronize()
    # a short idle first: right after the device-only region the GPU runs at
    # power-capped clocks, which would be charged to the host copies
    time.sleep(1.0)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk_e2e:
        e0.record(stream)
        e2e_steps(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), world)

    if rank != 0:
        return None
    fl = layer.flops()
    tokens = T * args.steps * world
    value = tokens / (ms_max / 1e3)
    gemm_flops_step = fl["routed"] + fl["shared"]
    fp8_peak = 2.0 * pk["bf16_tflops"]          # nominal fp8:bf16 ratio 2 on the measured bf16 burst
    g1_bytes = gemm1_bytes(layer, touched)
    g1_gbs = g1_bytes / (g1_ms / 1e3) / 1e9
    g1_tflops = 2 * (T * layer.K + T) * 2 * layer.I * layer.H / (g1_ms / 1e3) / 1e12
    rec = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic (seeded N(0,1) activations with 0.1% x50 outlier channels; N(0,0.006) weights)",
        "config": {"workload": workload_desc(shape), "global_batch": T * world, "parallelism": f"replicas{world}",
                   "l2": "no flush: 11.3 GB of resident expert weights per step exceed the 126 MB L2",
                   "weights_gb": round(layer.qw.nbytes / 1e9, 3)},
        "gemm_tflops": round(gemm_flops_step / (ms_max / args.steps / 1e3) / 1e12, 1),
        "gemm_pct_fp8_peak": round(100 * gemm_flops_step / (ms_max / args.steps / 1e3) / 1e12 / fp8_peak, 1),
        "roofline": {
            "kernel": "grouped_gemm_kernel (W13 of 256 routed + 1 shared expert, SwiGLU+requant epilogue)",
            "bound": "hbm", "achieved": round(g1_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(g1_gbs / pk["hbm_gbs"], 3), "traffic": recorded_w13_traffic(g1_bytes),
            "traffic_unit": "bytes per launch", "peak_kind": pk_kind,
            "launch_ms": round(g1_ms, 4), "algorithmic_bytes": g1_bytes, "touched_experts": touched,
            "tensor_tflops": round(g1_tflops, 1), "tensor_frac_of_fp8": round(g1_tflops / fp8_peak, 3),
        },
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * shape.H * 2, "d2h_bytes_per_step": T * shape.H * 2,
                "how": "moe_layer_run_host (C ABI) over the K steps: each step's pinned-host input (4 distinct "
                       "batches in rotation) uploaded on its own stream, forward + bias update on the compute "
                       "stream, output downloaded on a third stream; copies of neighbouring steps overlap each "
                       "forward (double-buffered device input/output)",
                "clocks": clk_e2e.summary()},
        "w2_launch_ms": round(g2_ms, 4),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "device_status": status,
        "balance": balance,
    }
    if world == 1 and not args.no_workloads:
        rec["workloads"] = run_workloads(layer.qw, pk, pk_kind, layer.offsets_all, layer)
    return rec


# ----------------------------------------------------------------- further workloads
def _gemm_flops(T: int, K: int, H: int, I: int):
    rows = T * K + T                   # routed (token, slot) rows + the shared expert's T rows
    return 2 * rows * 2 * I * H, 2 * rows * H * I


def leg_prefill(qw, pk, steps: int = 20) -> dict:
    """Prefill-scale skewed routing: T = 32768 at the DeepSeek-V3 shape, router
    logits offset by a Zipf(1.1) ranking (initial max/mean expert load ~20),
    `steps` consecutive forwards each followed by the bias update (gamma 0.001)
    that feeds back into the next step's routing; a fresh batch every step."""
    s = synth.PREFILL
    T, H, E, K, I = s.T, s.H, s.E, s.K, s.I
    off = synth.zipf_offset(E, synth.zipf_kappa_default(), synth.seed_of(s, synth.ZIPF), device="cuda")
    layer = build_layer(s, T, qw=qw, offset=off)
    xs = [synth.activations(T, H, synth.seed_of(s, synth.X) + 1000 * i, s.x_outlier_frac, device="cuda")
          for i in range(steps)]
    b0 = layer.e_bias.clone()
    layer.forward(xs[0])                       # warm-up, then back to the initial bias
    layer.e_bias.copy_(b0)
    hist = torch.empty(steps, E, dtype=torch.int32, device="cuda")
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        layer.forward(xs[i], gemm_events=ev[i])
        layer.bias_update(0.001)
        hist[i].copy_(layer.load, non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    w13 = [a.elapsed_time(b) for a, b, _ in ev]
    w2 = [b.elapsed_time(c) for _, b, c in ev]
    f13, f2 = _gemm_flops(T, K, H, I)
    loads = hist.cpu().numpy().astype(np.float64)
    ratio = loads.max(axis=1) / loads.mean(axis=1)
    peak = 2.0 * pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    del xs, layer
    return {"workload": workload_desc(s) + " + Zipf(1.1) router offset, bias update fed back each step",
            "steps": steps, "ms_per_step": round(ms, 4), "tokens_per_s": round(T / (ms / 1e3), 1),
            "w13_ms": round(statistics.mean(w13), 4), "w2_ms": round(statistics.mean(w2), 4),
            "w13_tflops": round(f13 / statistics.mean(w13) / 1e9, 1),
            "w2_tflops": round(f2 / statistics.mean(w2) / 1e9, 1),
            "gemm_tflops": round((f13 + f2) / (statistics.mean(w13) + statistics.mean(w2)) / 1e9, 1),
            "gemm_frac_of_fp8_peak": round((f13 + f2) / (statistics.mean(w13) + statistics.mean(w2)) / 1e9 / peak, 3),
            "fp8_peak_tflops": peak, "fp8_peak_kind": "2 x bf16_tflops_sustained (measured)",
            "max_over_mean_load_first": round(float(ratio[0]), 3),
            "max_over_mean_load_last": round(float(ratio[-1]), 3)}


def leg_decode(qw, pk, steps: int = 50) -> dict:
    """Decode-sized batch: T = 128 tokens at the DeepSeek-V3 shape, all 257
    experts' E4M3 weights resident; measured against the HBM bandwidth of the expert
    weights the step actually touches (every expert with a routed token, plus
    the shared expert), read by the two grouped GEMMs."""
    s = synth.DECODE
    T, H, E, K, I = s.T, s.H, s.E, s.K, s.I
    layer = build_layer(s, T, qw=qw)
    x = synth.activations(T, H, synth.seed_of(s, synth.X), s.x_outlier_frac, device="cuda")
    for _ in range(3):
        layer.forward(x)
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        layer.forward(x, gemm_events=ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    gemm_ms = statistics.mean(a.elapsed_time(c) for a, _, c in ev)
    touched = int((layer.load.cpu().numpy() > 0).sum()) + 1
    per_expert = 3 * I * H + ((2 * I // 128) * (H // 128) + (H // 128) * (I // 128)) * 4
    wbytes = touched * per_expert
    gbs = wbytes / (gemm_ms / 1e3) / 1e9
    del layer
    return {"workload": workload_desc(s), "steps": steps, "ms_per_step": round(ms, 4),
            "tokens_per_s": round(T / (ms / 1e3), 1), "gemm_ms": round(gemm_ms, 4),
            "touched_experts": touched, "touched_weight_bytes": wbytes,
            "weight_gbs": round(gbs, 1), "weight_frac_of_hbm": round(gbs / pk["hbm_gbs"], 3),
            "l2": "no flush: ~11 GB of touched weights per step exceed the 126 MB L2"}


def leg_gemm_dense(pk, M: int = 4096, N: int = 18432, K: int = 7168, iters: int = 20) -> dict:
    """Dense FP8 block-scaled GEMM of the sweep: A [M, K] bf16 N(0,1) with 1 % of
    the entries x100, quantised 1x128; B [N, K] N(0, 0.02) in 128x128 blocks;
    C bf16.  Each launch is timed alone after an L2 flush (a 256 MB write)."""
    import sparse_moe_layer_group_b200 as moe
    abi = moe.abi
    a = synth.heavy_tailed(M, K, 71, device="cuda")
    qa = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    sa = torch.empty(M, K // 128, dtype=torch.float32, device="cuda")
    abi.fp8_quant_1x128(a, qa, sa)
    b = synth.normal((N, K), 0.02, 72, device="cuda", dtype=torch.bfloat16)
    qb = torch.empty(1, N, K, dtype=torch.uint8, device="cuda")
    sb = torch.empty(1, N // 128, K // 128, dtype=torch.float32, device="cuda")
    abi.fp8_quant_128x128(b, qb[0], sb[0])
    del a, b
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor([0, M], dtype=torch.int32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    run = lambda: abi.fp8_grouped_gemm_blockscaled(1, offs, M, N, K, qa, sa, qb, sb, abi.MOE_EPI_BF16, C)
    for _ in range(3):
        run()
    times = []
    for _ in range(iters):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    tflops = 2 * M * N * K / (ms / 1e3) / 1e12
    peak = 2.0 * pk["bf16_tflops"]
    return {"workload": f"dense FP8 block-scaled GEMM M={M} N={N} K={K}, bf16 out", "launches": iters,
            "ms": round(ms, 4), "tflops": round(tflops, 1), "frac_of_fp8_peak": round(tflops / peak, 3),
            "fp8_peak_tflops": peak, "fp8_peak_kind": "2 x bf16_tflops burst (measured)",
            "l2": "flushed before every launch (256 MB write)"}


def leg_gemm_sweep(pk, qw, iters: int = 10) -> list:
    """The FP8 block-scaled GEMM sweep: dense C = A B^T for (N, K) in {(4096, 7168),
    (7168, 2048), (18432, 7168), (7168, 18432)} and M in {128, 1024, 4096, 16384}
    (A N(0,1) with 1 % of the entries x100, B N(0, 0.02)), and each shape as a
    256-group GEMM with 8M rows split by a seeded uniform random composition
    (sorted uniform cut points, empty groups allowed) over 256 weight matrices
    (the layer's resident experts for its two shapes W13 and W2, drawn N(0, 0.02)
    for the other two).  Each launch timed alone after a
    256 MB L2 flush, median of `iters`; TFLOP/s against 2 x the measured bf16
    burst and algorithmic bytes (A, B and scales read, C written) against the
    HBM copy peak."""
    import sparse_moe_layer_group_b200 as moe
    abi = moe.abi
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    peak = 2.0 * pk["bf16_tflops"]

    def timed(run):
        for _ in range(2):
            run()
        t = []
        for _ in range(iters):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            run()
            e1.record()
            e1.synchronize()
            t.append(e0.elapsed_time(e1))
        return statistics.median(t)

    def row(kind, M, N, K, G, ms, nbytes):
        fl = 2 * M * N * K
        return {"kind": kind, "M": M, "N": N, "K": K, "groups": G, "ms": round(ms, 4),
                "tflops": round(fl / ms / 1e9, 1), "frac_of_fp8_peak": round(fl / ms / 1e9 / peak, 3),
                "gbs": round(nbytes / ms / 1e6, 1), "frac_of_hbm": round(nbytes / ms / 1e6 / pk["hbm_gbs"], 3)}

    out = []
    Ms = (128, 1024, 4096, 16384)
    for N, K in ((4096, 7168), (7168, 2048), (18432, 7168), (7168, 18432)):
        b = synth.normal((N, K), 0.02, 72, device="cuda", dtype=torch.bfloat16)
        qb = torch.empty(1, N, K, dtype=torch.uint8, device="cuda")
        sb = torch.empty(1, N // 128, K // 128, dtype=torch.float32, device="cuda")
        abi.fp8_quant_128x128(b, qb[0], sb[0])
        del b
        for M in Ms:
            a = synth.heavy_tailed(M, K, 71, device="cuda")
            qa = torch.empty(M, K, dtype=torch.uint8, device="cuda")
            sa = torch.empty(M, K // 128, dtype=torch.float32, device="cuda")
            abi.fp8_quant_1x128(a, qa, sa)
            del a
            C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            offs = torch.tensor([0, M], dtype=torch.int32, device="cuda")
            ms = timed(lambda: abi.fp8_grouped_gemm_blockscaled(1, offs, M, N, K, qa, sa, qb, sb, abi.MOE_EPI_BF16,
                                                                C))
            nbytes = M * K + N * K + M * (K // 128) * 4 + (N // 128) * (K // 128) * 4 + 2 * M * N
            out.append(row("dense", M, N, K, 1, ms, nbytes))
            del qa, sa, C
        del qb, sb
    # 256 groups, 8M rows in a seeded uniform random composition; the two layer shapes
    # reuse the resident expert weights, the other two draw 256 weight matrices
    G = 256
    for N, K in ((4096, 7168), (7168, 2048), (18432, 7168), (7168, 18432)):
        if (N, K) == tuple(qw.w13.shape[1:]):
            name, W, S = "W13", qw.w13, qw.s13
        elif (N, K) == tuple(qw.w2.shape[1:]):
            name, W, S = "W2", qw.w2, qw.s2
        else:
            name = f"{N}x{K}"
            W = torch.empty(G, N, K, dtype=torch.uint8, device="cuda")
            S = torch.empty(G, N // 128, K // 128, dtype=torch.float32, device="cuda")
            for e in range(G):
                b = synth.normal((N, K), 0.02, 1000 + e, device="cuda", dtype=torch.bfloat16)
                abi.fp8_quant_128x128(b, W[e], S[e])
                del b
        for M in Ms:
            rows = 8 * M
            g = synth.gen(900 + M, "cpu")
            cuts = torch.sort(torch.randint(0, rows + 1, (G - 1,), generator=g)).values
            offs_h = torch.cat([torch.zeros(1, dtype=torch.int64), cuts, torch.tensor([rows])])
            offs = offs_h.to(torch.int32).cuda()
            a = synth.heavy_tailed(rows, K, 73, device="cuda")
            qa = torch.empty(rows, K, dtype=torch.uint8, device="cuda")
            sa = torch.empty(rows, K // 128, dtype=torch.float32, device="cuda")
            abi.fp8_quant_1x128(a, qa, sa)
            del a
            C = torch.empty(rows, N, dtype=torch.bfloat16, device="cuda")
            ms = timed(lambda: abi.fp8_grouped_gemm_blockscaled(G, offs, rows, N, K, qa, sa, W, S, abi.MOE_EPI_BF16,
                                                                C))
            touched = int(((offs_h[1:] - offs_h[:-1]) > 0).sum())
            nbytes = (rows * K + touched * (N * K + (N // 128) * (K // 128) * 4) + rows * (K // 128) * 4
                      + 2 * rows * N)
            out.append(row(f"grouped {name}", rows, N, K, G, ms, nbytes))
            del qa, sa, C
        del W, S
        torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return out


def leg_wgrad(offsets_all, pk, iters: int = 5) -> dict:
    """Backward weight gradient of W13 at the DeepSeek-V3 layer shape: dW13 [257,
    2I, H] = dY^T X per expert over the layer's own expert segments (the T*K
    routed rows in expert order, then the T shared rows), dY bf16 [T*K + T, 2I]
    and X bf16 [T*K + T, H] seeded N(0,1); one step = the two 128x1 quantisations
    and the wgrad GEMM.  Bound by HBM: the fp32 gradient alone is 30 GB."""
    import sparse_moe_layer_group_b200 as moe
    abi = moe.abi
    s = synth.DSV3
    H, I = s.H, s.I
    offs = offsets_all
    G = offs.numel() - 1
    M = int(offs[-1].item())
    dy = synth.normal((M, 2 * I), 1.0, 81, device="cuda", dtype=torch.bfloat16)
    x = synth.activations(M, H, 82, device="cuda")
    p_cap, t_cap = abi.wgrad_capacities(M, G)
    dq = torch.empty(2 * I, p_cap, dtype=torch.uint8, device="cuda")
    ds = torch.empty(t_cap, 2 * I, dtype=torch.float32, device="cuda")
    xq = torch.empty(H, p_cap, dtype=torch.uint8, device="cuda")
    xs = torch.empty(t_cap, H, dtype=torch.float32, device="cuda")
    dW = torch.empty(G, 2 * I, H, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(ev=None):
        abi.fp8_quant_128x1_grouped(dy, offs, dq, ds, st)
        abi.fp8_quant_128x1_grouped(x, offs, xq, xs, st)
        if ev is not None:
            ev[0].record()
        abi.fp8_grouped_gemm_wgrad(offs, M, dq, ds, xq, xs, dW, st)
        if ev is not None:
            ev[1].record()

    step()
    torch.cuda.synchronize()
    time.sleep(0.5)              # after the prefill and decode legs: let the clocks recover
    evs = []
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record()
        for _ in range(iters):
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            evs.append(ev)
            step(ev)
        t1.record()
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / iters
    g_ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    flops = 2.0 * M * 2 * I * H
    out_bytes = G * 2 * I * H * 4
    in_bytes = (2 * I + H) * (p_cap + 4 * t_cap)
    status = int(st.item())
    del dy, x, dq, ds, xq, xs, dW
    torch.cuda.empty_cache()
    return {"workload": f"wgrad of W13 at the DSV3 layer shape: {G} groups (256 routed + shared), {M} rows, "
                        f"dW fp32 [{G}, {2 * I}, {H}]", "iters": iters, "ms_per_step": round(ms, 4),
            "gemm_ms": round(g_ms, 4), "gemm_tflops": round(flops / g_ms / 1e9, 1),
            "gemm_gbs": round((out_bytes + in_bytes) / g_ms / 1e6, 1),
            "gemm_frac_of_hbm": round((out_bytes + in_bytes) / g_ms / 1e6 / pk["hbm_gbs"], 3),
            "algorithmic_bytes": out_bytes + in_bytes, "device_status": status, "clocks": clk.summary()}


def leg_gather(layer, pk, iters: int = 10) -> dict:
    """W13 of the DeepSeek-V3 step two ways on the step's own routing: over the
    materialised permuted rows (the layer's default, as timed in the step) and
    with the routed rows fetched through tok_of by TMA row gathers (the fused
    dispatch variant, which drops the permute's row-copy kernel and its
    T*K x H copy)."""
    import sparse_moe_layer_group_b200 as moe
    abi = moe.abi
    T, H, K, I, E = layer.T, layer.H, layer.K, layer.I, layer.E
    M = T * K + T
    qw = layer.qw
    a_map = torch.cat([layer.tok_of, torch.arange(T, dtype=torch.int32, device="cuda")])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def plain():
        abi.fp8_grouped_gemm_blockscaled(E + 1, layer.offsets_all, M, 2 * I, H, layer.aq, layer.as_, qw.w13, qw.s13,
                                         abi.MOE_EPI_SWIGLU_REQUANT, layer.actq, layer.acts, st)

    def gather():
        abi.fp8_grouped_gemm_blockscaled_gather(E + 1, layer.offsets_all, M, 2 * I, H, layer.xq, layer.xs, a_map,
                                                qw.w13, qw.s13, abi.MOE_EPI_SWIGLU_REQUANT, layer.actq, layer.acts,
                                                st)

    out = {"workload": "W13 grouped GEMM of the DSV3 step (T=4096, 257 groups, 36864 rows): materialised "
                       "permuted A vs A rows gathered through tok_of (tile::gather4)", "iters": iters}
    for name, fn in (("materialised_ms", plain), ("gather_ms", gather)):
        fn()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for _ in range(iters):
            fn()
        ev[1].record()
        torch.cuda.synchronize()
        out[name] = round(ev[0].elapsed_time(ev[1]) / iters, 4)
    out["device_status"] = int(st.item())
    return out


def leg_combine(layer, pk, iters: int = 10) -> dict:
    """The second half of the DSV3 step two ways on the step's own routing and
    activations: W2 storing its bf16 rows + the combine kernel (the layer's
    default), and W2 with the combine in its epilogue (gates scattered into row
    order, gated rows added into an fp32 accumulator at the L2) + the finishing
    pass that rounds to bf16 and re-zeroes the accumulator (f3 combine half)."""
    import sparse_moe_layer_group_b200 as moe
    abi = moe.abi
    T, H, K, I, E = layer.T, layer.H, layer.K, layer.I, layer.E
    M = T * K + T
    qw = layer.qw
    row_gate = torch.ones(M, dtype=torch.float32, device="cuda")
    acc = torch.zeros(T, H, dtype=torch.float32, device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def stored():
        abi.fp8_grouped_gemm_blockscaled(E + 1, layer.offsets_all, M, H, I, layer.actq, layer.acts, qw.w2, qw.s2,
                                         abi.MOE_EPI_BF16, layer.yperm, None, st)
        abi.moe_combine(layer.d, layer.yperm, layer.row_of, layer.topk_w, layer.ysh, out)

    def fused():
        abi.moe_ep_scatter(layer.row_of, layer.topk_w.view(torch.int32), row_gate[:T * K].view(torch.int32))
        abi.fp8_grouped_gemm_blockscaled_combine(E + 1, layer.offsets_all, M, H, I, layer.actq, layer.acts, qw.w2,
                                                 qw.s2, layer.rows_tok, row_gate, acc, st)
        abi.moe_combine_finish(acc, out, None, True)

    res = {"workload": "W2 + combine of the DSV3 step (T=4096, 257 groups, 36864 rows): bf16 rows stored and "
                       "combined vs combine in the W2 epilogue (fp32 L2 reductions) + bf16 finish", "iters": iters}
    for name, fn in (("stored_ms", stored), ("fused_ms", fused)):
        fn()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        for _ in range(iters):
            fn()
        ev[1].record()
        torch.cuda.synchronize()
        res[name] = round(ev[0].elapsed_time(ev[1]) / iters, 4)
    res["device_status"] = int(st.item())
    return res


def run_workloads(qw, pk, pk_kind, offsets_all=None, layer=None) -> dict:
    """The other configurations of the layer, each timed with CUDA events only:
    prefill with skewed routing, decode, and the dense GEMM sweep's largest
    compute-bound shape, and the backward wgrad of W13 over the DSV3 step's own
    expert segments.  The layer legs reuse the resident DeepSeek-V3 expert
    weights (same sizes); their routers and inputs come from their own seeds."""
    # the dense GEMM first, after a short idle: run after the long prefill leg it
    # would be timed at power-capped clocks against the burst peak
    time.sleep(1.0)
    with ClockSampler(torch.cuda.current_device()) as clk:
        dense = leg_gemm_dense(pk)
    dense["clocks"] = clk.summary()
    with ClockSampler(torch.cuda.current_device()) as clk:
        sweep = leg_gemm_sweep(pk, qw)
    out = {"gemm_dense": dense, "gemm_sweep": {"shapes": sweep, "clocks": clk.summary()},
           "prefill_skew": leg_prefill(qw, pk), "decode": leg_decode(qw, pk)}
    if offsets_all is not None:
        out["wgrad"] = leg_wgrad(offsets_all, pk)
    if layer is not None and not layer.gather and not layer.fused_combine:
        out["gather"] = leg_gather(layer, pk)
        out["combine"] = leg_combine(layer, pk)
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------- CPU oracle arm
def time_oracle_sample(shape: synth.MoEShape, n_experts: int = 2, seed: int = 0) -> dict:
    """Time the float64 oracle on a bounded sample of one layer step and scale
    it to tokens/s: the router, quantisation and permutation of all T tokens,
    plus the expert FFNs of `n_experts` routed experts (their own rows) whose
    per-row time is scaled to all T*K + T expert rows of the step."""
    import oracle
    from threadpoolctl import threadpool_info
    T, H, E, K, I = shape.T, shape.H, shape.E, shape.K, shape.I
    x = synth.activations(T, H, synth.seed_of(shape, synth.X), shape.x_outlier_frac).float().numpy()
    wr = synth.router_weights(E, H, shape.wr_std, synth.seed_of(shape, synth.WR)).numpy()
    b = synth.expert_bias(E, shape.bias_range, synth.seed_of(shape, synth.BIAS)).numpy()
    t0 = time.perf_counter()
    s32 = oracle.router_scores(x, wr).astype(np.float32)
    idx, w = oracle.select_experts(s32, b, shape.n_group, shape.topk_group, K, shape.rho)
    load, offs, tok_of, row_of = oracle.permute(idx, E)
    xq, xs = oracle.quant_1x128(x)
    t_route = time.perf_counter() - t0
    rows = 0
    t_ffn = 0.0
    for j in range(n_experts):
        e = int(np.argsort(-load)[j * 7 % E])
        w13 = synth.expert_weight(2 * I, H, shape.w_std, synth.seed_of(shape, synth.W13, e)).float().numpy()
        w2 = synth.expert_weight(H, I, shape.w_std, synth.seed_of(shape, synth.W2, e)).float().numpy()
        q13, s13 = oracle.quant_128x128(w13)
        q2, s2 = oracle.quant_128x128(w2)
        r0, r1 = int(offs[e]), int(offs[e + 1])
        sel = tok_of[r0:r1]
        t1 = time.perf_counter()
        oracle.expert_ffn(xq[sel], xs[sel], q13, s13, q2, s2)
        t_ffn += time.perf_counter() - t1
        rows += r1 - r0
    per_row = t_ffn / max(rows, 1)
    t_step = t_route + per_row * (T * K + T)
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    return {"value": T / t_step, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": (f"router+top-K+permute+quant of all {T} tokens ({t_route:.2f} s) and the FFNs of "
                       f"{n_experts} routed experts ({rows} rows, {t_ffn:.2f} s) scaled to {T * K + T} "
                       f"expert rows; est. {t_step:.1f} s per step")}


def oracle_step_sampler(shape: synth.MoEShape, tok: int = 256, rows: int = 128):
    """The reference arm's step: the float64 oracle on a bounded slice of one
    layer step, scaled to the whole step -- router, top-K, permutation and
    quantisation of `tok` tokens (a different slice each step) and the FFN of
    one routed expert on `rows` tokens (128 = the mean expert load T*K/E at the
    layer shape; the slice is repeated when tok < rows), per-token and per-row times
    scaled to T tokens and T*K + T expert rows.  Inputs and the expert's
    quantised weights are prepared once, outside the timing."""
    import oracle
    T, H, E, K, I = shape.T, shape.H, shape.E, shape.K, shape.I
    x = synth.activations(T, H, synth.seed_of(shape, synth.X), shape.x_outlier_frac).float().numpy()
    wr = synth.router_weights(E, H, shape.wr_std, synth.seed_of(shape, synth.WR)).numpy()
    b = synth.expert_bias(E, shape.bias_range, synth.seed_of(shape, synth.BIAS)).numpy()
    w13 = synth.expert_weight(2 * I, H, shape.w_std, synth.seed_of(shape, synth.W13, 0)).float().numpy()
    w2 = synth.expert_weight(H, I, shape.w_std, synth.seed_of(shape, synth.W2, 0)).float().numpy()
    q13, s13 = oracle.quant_128x128(w13)
    q2, s2 = oracle.quant_128x128(w2)

    def step(i: int) -> float:
        lo = (i * tok) % T
        xs_ = x[lo:lo + tok]
        t0 = time.perf_counter()
        s32 = oracle.router_scores(xs_, wr).astype(np.float32)
        idx, _ = oracle.select_experts(s32, b, shape.n_group, shape.topk_group, K, shape.rho)
        oracle.permute(idx, E)
        xq, xsc = oracle.quant_1x128(xs_)
        t_route = time.perf_counter() - t0
        sel = np.arange(rows) % len(xs_)
        t1 = time.perf_counter()
        oracle.expert_ffn(xq[sel], xsc[sel], q13, s13, q2, s2)
        t_ffn = time.perf_counter() - t1
        t_step = t_route * (T / len(xs_)) + t_ffn / rows * (T * K + T)
        return T / t_step

    return step


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from threadpoolctl import threadpool_info
    shape = synth.DSV3
    tok, rows = 256, 128
    step = oracle_step_sampler(shape, tok, rows)
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    vals = [step(args.warmup + i) for i in range(max(1, args.steps))]
    wall = time.perf_counter() - t0
    v = statistics.median(vals)
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    cb = {"value": round(v, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
          "sample": (f"per step: router+top-K+permute+quant of {tok} of the {shape.T} tokens and the FFN of one "
                     f"routed expert on {rows} rows, scaled to {shape.T} tokens and {shape.T * shape.K + shape.T} "
                     f"expert rows; median over {len(vals)} steps ({wall:.1f} s of host time)")}
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(shape.T / v * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload_desc(shape), "global_batch": shape.T,
                                         "parallelism": "host cores"},
        "cpu_baseline": cb,
        "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------- single-kernel cases
def run_case(args):
    """One kernel alone on a profiling-sized case (a few GB on the device):
    gemm1 = routed W13 GEMM with the SwiGLU+requant epilogue and gemm2 = routed
    W2 GEMM, both on 64 experts x 128 rows at the DSV3 hidden/intermediate
    sizes (1.9 GB / 0.9 GB of weights, larger than L2); gemm1_gather = gemm1_skew
    with its A rows gathered through a seeded row map from T/8 source rows (the
    layer's fan-out of 8 slots per token); wgrad = the wgrad GEMM of W13 for 8
    experts of ~144 rows (dW 0.94 GB); router = moe_route at T=4096, H=7168, E=256."""
    import sparse_moe_layer_group_b200 as moe
    abi = moe.abi
    shape = synth.DSV3
    H, I = shape.H, shape.I
    E, rows = 64, 128
    dev = "cuda"
    ev = []
    if args.case in ("gemm1", "gemm2", "gemm1_x256", "gemm1_skew", "gemm1_gather"):
        N, K = (H, I) if args.case == "gemm2" else (2 * I, H)
        w = torch.empty(E, N, K, dtype=torch.uint8, device=dev)
        sw = torch.empty(E, N // 128, K // 128, dtype=torch.float32, device=dev)
        for e in range(E):
            m = synth.expert_weight(N, K, shape.w_std, synth.seed_of(shape, synth.W13, e), device=dev)
            abi.fp8_quant_128x128(m, w[e], sw[e])
        if args.case == "gemm1_x256":
            sizes = [2 * rows] * E
        elif args.case in ("gemm1_skew", "gemm1_gather"):
            # log-normal expert loads with mean 128 rows (spread like an unbalanced router)
            g = synth.gen(11, "cpu")
            wts = torch.exp(0.6 * torch.randn(E, generator=g, dtype=torch.float64))
            sizes = torch.floor(wts / wts.sum() * E * rows).to(torch.int64).tolist()
        else:
            sizes = [rows] * E
        Mrows = int(sum(sizes))
        a_bf = synth.activations(Mrows, K, 5, device=dev)
        a = torch.empty(Mrows, K, dtype=torch.uint8, device=dev)
        sa = torch.empty(Mrows, K // 128, dtype=torch.float32, device=dev)
        abi.fp8_quant_1x128(a_bf, a, sa)
        offs = torch.tensor([0] + list(np.cumsum(sizes)), dtype=torch.int32, device=dev)
        mode = {"auto": 0, "single": abi.MOE_GEMM_SINGLE_CTA, "pair": abi.MOE_GEMM_PAIR_CTA}[args.gemm_mode]
        if args.case == "gemm1_gather":
            n_src = max(1, Mrows // 8)
            a_map = torch.randint(0, n_src, (Mrows,), generator=synth.gen(13, "cpu"), dtype=torch.int32).to(dev)
            src_q, src_s = a[:n_src].contiguous(), sa[:n_src].contiguous()
            out = torch.empty(Mrows, N // 2, dtype=torch.uint8, device=dev)
            so = torch.empty(Mrows, N // 256, dtype=torch.float32, device=dev)
            run = lambda: abi.fp8_grouped_gemm_blockscaled_gather(E, offs, Mrows, N, K, src_q, src_s, a_map, w, sw,
                                                                 abi.MOE_EPI_SWIGLU_REQUANT, out, so)
        elif args.case != "gemm2":
            out = torch.empty(Mrows, N // 2, dtype=torch.uint8, device=dev)
            so = torch.empty(Mrows, N // 256, dtype=torch.float32, device=dev)
            run = lambda: abi.fp8_grouped_gemm_blockscaled(E, offs, Mrows, N, K, a, sa, w, sw,
                                                          abi.MOE_EPI_SWIGLU_REQUANT | mode, out, so)
        else:
            out = torch.empty(Mrows, N, dtype=torch.bfloat16, device=dev)
            run = lambda: abi.fp8_grouped_gemm_blockscaled(E, offs, Mrows, N, K, a, sa, w, sw,
                                                          abi.MOE_EPI_BF16 | mode, out)
        nbytes = E * N * K + Mrows * K + Mrows * (2 * N if args.case == "gemm2" else N // 2)
        flops = 2 * Mrows * N * K
    elif args.case == "wgrad":
        G, N, K = 8, 2 * I, H
        g = synth.gen(14, "cpu")
        sizes = (torch.full((G,), 144) + torch.randint(-40, 41, (G,), generator=g)).tolist()
        M = int(sum(sizes))
        offs = torch.tensor([0] + list(np.cumsum(sizes)), dtype=torch.int32, device=dev)
        dy = synth.normal((M, N), 1.0, 81, device=dev, dtype=torch.bfloat16)
        xx = synth.activations(M, K, 82, device=dev)
        p_cap, t_cap = abi.wgrad_capacities(M, G)
        dq = torch.empty(N, p_cap, dtype=torch.uint8, device=dev)
        ds = torch.empty(t_cap, N, dtype=torch.float32, device=dev)
        xq = torch.empty(K, p_cap, dtype=torch.uint8, device=dev)
        xs = torch.empty(t_cap, K, dtype=torch.float32, device=dev)
        dW = torch.empty(G, N, K, dtype=torch.float32, device=dev)
        abi.fp8_quant_128x1_grouped(dy, offs, dq, ds)
        abi.fp8_quant_128x1_grouped(xx, offs, xq, xs)
        run = lambda: abi.fp8_grouped_gemm_wgrad(offs, M, dq, ds, xq, xs, dW)
        nbytes = G * N * K * 4 + (N + K) * (p_cap + 4 * t_cap)
        flops = 2 * M * N * K
    elif args.case == "router":
        T, E2 = shape.T, shape.E
        x = synth.activations(T, H, 1, device=dev)
        wr = synth.router_weights(E2, H, shape.wr_std, 2, device=dev)
        b = torch.zeros(E2, dtype=torch.float32, device=dev)
        d = abi.dims(T, H, E2, shape.K, shape.n_group, shape.topk_group, I, shape.rho)
        idx = torch.empty(T, shape.K, dtype=torch.int32, device=dev)
        wt = torch.empty(T, shape.K, dtype=torch.float32, device=dev)
        sc = torch.empty(T, E2, dtype=torch.float32, device=dev)
        ws = torch.empty(abi.workspace_size(d), dtype=torch.uint8, device=dev)
        run = lambda: abi.moe_route(d, x, wr, b, None, idx, wt, sc, ws)
        nbytes = T * H * 2 + E2 * H * 4 + T * E2 * 4
        flops = 2 * T * E2 * H
    else:
        raise SystemExit(f"unknown case {args.case}")
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    print(json.dumps({"case": args.case, "ms": round(ms, 4), "GB/s": round(nbytes / ms / 1e6, 1),
                      "TFLOP/s": round(flops / ms / 1e9, 1), "algorithmic_bytes": nbytes, "flops": flops}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the prefill / decode / dense-GEMM legs reported under 'workloads'")
    ap.add_argument("--case", default=None,
                    help="time one kernel alone: gemm1 | gemm1_x256 | gemm1_skew | gemm1_gather | gemm2 | wgrad | router")
    ap.add_argument("--gemm-mode", default="auto", choices=["auto", "single", "pair"])
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    if args.impl == "reference":
        # the oracle runs on the host cores of rank 0 alone; other ranks exit at once
        # (no process group: nothing is exchanged and rank 0 runs for minutes)
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rec = run_reference(args, rank, world)
        if rec is not None:
            print(json.dumps(rec), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    rec = run_gpu(args, rank, world, local)
    if rec is not None and world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = time_oracle_sample(synth.DSV3)
    if rec is not None:
        print(json.dumps(rec), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
