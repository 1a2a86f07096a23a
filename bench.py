#!/usr/bin/env python
"""Benchmark of the union-of-experts 4-bit SwitchGLU layer on B200.

Workload: the GLM-5.3-Flash-shaped layer of "gather_qmm at M=1 streams 4-bit
expert weights at ~half the bandwidth of M=4" (mlx issue 4509, "Numbers" and
the moe_bench.py script): E=288 experts, top-8, hidden 4096, intermediate 2048,
4-bit affine group 64 with bf16 scale and bias (14,155,776 B per expert), bf16
activations ~N(0,1), each token's 8 experts drawn uniformly without
replacement.  One bank of 288 experts is shared by 42 layers with 42 distinct
routings, as the script does.  One step = the 42-layer chain at T=1 followed by
the 42-layer chain at T=4 (both rows of the page's table), launched back to back
with no host synchronisation (captured once in a CUDA graph).

Metric: effective HBM GB/s over unique-expert bytes (u * 14,155,776 B per layer,
u = distinct experts of the layer's window), and us/layer.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs its own replica of the workload on its own GPU
(no data-path collective; "scaling": "weak"); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

K_TOP, HIDDEN, INTER = 8, 4096, 2048
E = 288     # experts in the bank (--experts changes it, for small profiling cases only)
LAYERS = 42  # chained layers per T (--layers changes it, for small profiling cases only)
TS = (1, 4)
SEED = 2000
BYTES_PER_EXPERT = 3 * (INTER * HIDDEN // 2 + 2 * 2 * INTER * HIDDEN // 64)  # 14,155,776
METRIC = "us/layer and effective HBM GB/s (unique-expert bytes) at T=1..16, % of B200 peak"
L2_BYTES = 126 * 1024 * 1024
# what the small-window kernel computes in: 4-bit affine codes times bf16 activations held
# as 16-bit block fixed point per 32 columns (exact for values within 8 binades of their
# chunk's largest), integer dot products, fp32 scaling and accumulation
DTYPE_LABEL = ("u4 affine weights x bf16 act as 16-bit block fixed point per 32 columns "
               "(exact int dot), f32 accum")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


KERNEL_SOURCES = ("layer.cuh", "common.cuh", "union.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "layer_kernel_full_glm_e96_t1_t4.txt")


def captured_traffic():
    """DRAM traffic of the layer kernel from the committed ncu summary: (read bytes per
    unique expert, write bytes per launch), or None once the kernel sources differ from
    those the counters were taken on."""
    import hashlib
    try:
        kv = {}
        for line in open(TRAFFIC_FILE):
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        want = kv["kernel_sources_sha256"].split()
        have = [hashlib.sha256(open(os.path.join(ROOT, "quantized_expert_gather_b200", "csrc",
                                                 f), "rb").read()).hexdigest()
                for f in KERNEL_SOURCES]
        if want != have:
            return None
        return (float(kv["traffic_read_bytes_per_unique_expert"]),
                float(kv["traffic_write_bytes_per_launch"]))
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------------ distributed ---
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ clocks ---
class ClockSampler:
    """nvidia-smi samples (every 50 ms) while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.first = threading.Event()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())
            self.first.set()

    def wait_first(self, timeout: float = 5.0):
        """Block until nvidia-smi has printed its first sample (it starts slowly)."""
        self.first.wait(timeout)

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        rows = [[c.strip() for c in ln.split(",")] for ln in self.lines]
        rows = [f for f in rows if len(f) >= 9]
        indices = sorted(set(f[0] for f in rows))
        want = str(self.gpu) if str(self.gpu) in indices else (indices[0] if indices else None)
        for f in rows:
            if f[0] != want:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"error": (self.lines[:2] if self.lines else "no nvidia-smi output")}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- workload ---
ROUTING = "uniform"  # --routing markov: adjacent-overlap chain at p=0.40 (profiling)
# speculative-verify pair: adjacent-token overlap at random (3 %), in shallow layers, the
# mean, in deep layers and the maximum of the pages' router recording
VERIFY_PS = (0.03, 0.21, 0.34, 0.45, 0.52)
# verify-window sweep: window sizes, and the layers of the stack (GLM-5.2's MoE depth)
WINDOW_TS = (2, 3, 5, 8, 16)
WINDOW_LAYERS = 78


def graph_us_per_layer(issue, n_layers: int, reps: int = 5) -> float:
    """Device time per layer of `issue()` (n_layers launches, no host synchronisation)
    captured once in a CUDA graph: one warm replay, then `reps` replays between CUDA
    events on the current stream."""
    import torch
    issue()  # first calls outside the capture (per-device set-up)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        issue()
    g.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / (reps * n_layers)
    del g
    return us


def window_layer_seed(T: int, layer: int) -> int:
    return SEED + 10000 + 100 * T + layer


def window_stack(T: int, dev, qeg, synth, layers: int = None):
    """The verify-window stack at window size T: per layer an adjacent-overlap routing at
    p = 0.40 over E=256 experts, and a bank compacted to the u experts that window routes
    to (drawn on the device, seed per layer; routing ids remapped to 0..u-1), its own x,
    workspace and output buffer.  Returns {"layers": [...], "unique": [u per layer]}."""
    import torch
    layers = layers or WINDOW_LAYERS
    out, uniq = [], []
    for l in range(layers):
        seed = window_layer_seed(T, l)
        idx, w = synth.route_markov(T, 256, K_TOP, 0.40, seed)
        used, remap = np.unique(idx, return_inverse=True)
        u = int(used.size)
        cidx = remap.reshape(idx.shape).astype(np.int32)

        def mat(rows, cols, mid):
            q = torch.empty((u, rows, cols // 8), dtype=torch.int32, device=dev)
            s_ = torch.empty((u, rows, cols // 64), dtype=torch.int16, device=dev)
            b_ = torch.empty_like(s_)
            synth.fill_bank_device(q, s_, b_, rows, cols, seed, mid)
            return q, s_.view(torch.bfloat16), b_.view(torch.bfloat16)
        bank = qeg.QuantBank(*mat(INTER, HIDDEN, 0), *mat(INTER, HIDDEN, 1),
                             *mat(HIDDEN, INTER, 2))
        out.append({
            "bank": bank, "seed": seed, "idx_host": cidx, "w_host": w,
            "idx": torch.from_numpy(cidx).to(dev), "w": torch.from_numpy(w).to(dev),
            "x": torch.from_numpy(synth.x_bf16(T, HIDDEN, seed).view(np.int16)).to(dev)
            .view(torch.bfloat16),
            "ws": torch.zeros(qeg.moe_workspace_size(T, K_TOP, u, HIDDEN, INTER),
                              dtype=torch.uint8, device=dev),
            "out": torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=dev)})
        uniq.append(u)
    torch.cuda.synchronize()
    return {"layers": out, "unique": uniq}


def routings():
    import synth
    out = {}
    for T in TS:
        if ROUTING == "markov":
            out[T] = [synth.route_markov(T, E, K_TOP, 0.40, SEED + 100 * T + l)
                      for l in range(LAYERS)]
        elif ROUTING == "identical":  # every token on experts 8l .. 8l+7 (mod E)
            out[T] = [(np.tile((np.arange(K_TOP) + K_TOP * l) % E, (T, 1)).astype(np.int32),
                       np.full((T, K_TOP), 1.0 / K_TOP, np.float32)) for l in range(LAYERS)]
        else:
            out[T] = [synth.route_uniform(T, E, K_TOP, SEED + 100 * T + l) for l in range(LAYERS)]
    return out


def uniques(routes):
    return {T: [int(np.unique(r[0]).size) for r in routes[T]] for T in TS}


def cpu_cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def parity_of(got: np.ndarray, ref: np.ndarray):
    """(rel-L2, max-abs / rms(ref)) of a layer output against the oracle's: the parity
    measures of the GPU tests (bar: 5e-3 and 3e-2)."""
    d = got - ref
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return rel, float(np.abs(d).max() / rms) if rms > 0 else float(np.abs(d).max())


def run_oracle_sample(routes, budget_s: float = 15.0, gpu_outs=None):
    """Time the oracle (all host threads) on whole layers of the workload until about
    `budget_s` of CPU work: every layer of the chain once, then (if time is left) the
    last T=1 and T=4 layers again.  Each layer the oracle computes is also compared with
    the GPU's kept output of the same chained layer (gpu_outs[T][l], bf16 bits), outside
    the timed call.  Returns (GB/s over unique bytes, layers timed, seconds, threads,
    parity summary)."""
    import oracle
    import synth
    threads = cpu_cores()
    done, secs, nbytes = 0, 0.0, 0
    order = [(T, l) for l in range(LAYERS) for T in TS]
    last = {}
    checked, worst_rel, worst_mx = [], 0.0, 0.0

    def timed(T, l, bank, used):
        nonlocal done, secs, nbytes, worst_rel, worst_mx
        idx, w = routes[T][l]
        x = synth.x_bf16(T, HIDDEN, SEED + T)
        t0 = time.perf_counter()
        ref = oracle.switchglu(x, idx, w, bank, E, n_threads=threads)
        secs += time.perf_counter() - t0
        done += 1
        nbytes += len(used) * BYTES_PER_EXPERT
        if gpu_outs is not None and (T, l) not in checked:
            got = synth.bf16_bits_to_f32(gpu_outs[T][l]).astype(np.float64)
            rel, mx = parity_of(got, ref)
            worst_rel, worst_mx = max(worst_rel, rel), max(worst_mx, mx)
            checked.append((T, l))

    for T, l in order:
        used = sorted(set(routes[T][l][0].ravel().tolist()))
        bank = {"gate": synth.fill_bank_host(E, INTER, HIDDEN, SEED, synth.MATRIX_GATE, used),
                "up": synth.fill_bank_host(E, INTER, HIDDEN, SEED, synth.MATRIX_UP, used),
                "down": synth.fill_bank_host(E, HIDDEN, INTER, SEED, synth.MATRIX_DOWN, used)}
        timed(T, l, bank, used)
        last[T] = (l, bank, used)
        if secs >= budget_s:
            break
    while secs < budget_s:
        for T in TS:
            l, bank, used = last[T]
            timed(T, l, bank, used)
    parity = None
    if gpu_outs is not None:
        parity = {"layers_checked": len(checked), "max_rel_l2": worst_rel,
                  "max_abs_over_rms": worst_mx,
                  "pass": bool(worst_rel <= 5e-3 and worst_mx <= 3e-2),
                  "what": "the GPU outputs of the chained layers kept from the timed graph "
                          "replays, against the oracle on the same inputs"}
    return nbytes / secs / 1e9, done, secs, threads, parity


def reference_arm(args, world, rank):
    """The oracle, as it stands, timed on the host cores: each step one bounded sample
    (one T=1 and one T=4 layer of the workload)."""
    if rank != 0:
        return 0
    import oracle
    import synth
    routes = routings()
    threads = cpu_cores()
    cache = {}
    plan = []
    for s in range(args.warmup + args.steps):
        l = s % min(LAYERS, 4)  # a few distinct layers, reused: bounded host-side set-up
        layer = []
        for T in TS:
            idx, w = routes[T][l]
            used = sorted(set(idx.ravel().tolist()))
            if (T, l) not in cache:
                cache[(T, l)] = {
                    "gate": synth.fill_bank_host(E, INTER, HIDDEN, SEED, 0, used),
                    "up": synth.fill_bank_host(E, INTER, HIDDEN, SEED, 1, used),
                    "down": synth.fill_bank_host(E, HIDDEN, INTER, SEED, 2, used)}
            layer.append((synth.x_bf16(T, HIDDEN, SEED + T), idx, w, cache[(T, l)], len(used)))
        plan.append(layer)
    times, nbytes = [], 0
    for s, layer in enumerate(plan):
        t0 = time.perf_counter()
        for x, idx, w, bank, u in layer:
            oracle.switchglu(x, idx, w, bank, E, n_threads=threads)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            nbytes += sum(u for *_, u in layer) * BYTES_PER_EXPERT
    tot = sum(times)
    gbs = nbytes / tot / 1e9
    ms = tot / len(times) * 1e3
    line = {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "GLM-5.3-Flash-shaped union-of-experts SwitchGLU layer "
                                   "E=288 top-8 4096/2048 q4g64", "sample": "one T=1 and one "
                                   "T=4 layer per step", "T": list(TS)},
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": "one T=1 and one T=4 layer of the 42-layer workload per "
                                       "step, all host threads"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def large_window_only(args, local):
    """Profiling run of the grouped path alone: one T-token layer (T from --ts, default
    512) on an E=256 bank (3.6 GB; with --mxfp4 an mxfp4 bank of the same shape, 3.4 GB),
    3 warm calls then 1 timed; for ncu captures of the grouped kernels on a small device
    footprint."""
    import torch
    import quantized_expert_gather_b200 as qeg
    import synth
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    EL = 256
    TL = int(args.ts) if args.ts else 512

    def mat(rows, cols, mid):
        q = torch.empty((EL, rows, cols // 8), dtype=torch.int32, device=dev)
        s = torch.empty((EL, rows, cols // 64), dtype=torch.int16, device=dev)
        b = torch.empty_like(s)
        synth.fill_bank_device(q, s, b, rows, cols, SEED, mid)
        return q, s.view(torch.bfloat16), b.view(torch.bfloat16)
    def matm(rows, cols, mid):
        q = torch.empty((EL, rows, cols // 8), dtype=torch.int32, device=dev)
        e8 = torch.empty((EL, rows, cols // 32), dtype=torch.uint8, device=dev)
        synth.fill_bank_mxfp4_device(q, e8, rows, cols, SEED, mid)
        return q, e8
    if args.mxfp4:  # the same shape on an mxfp4 bank (3.4 GB)
        bank = qeg.MxBank(*matm(INTER, HIDDEN, 0), *matm(INTER, HIDDEN, 1),
                          *matm(HIDDEN, INTER, 2))
        size = qeg.moe_workspace_size_mxfp4

        def call(x, il, wl, ws, out):
            qeg.moe_switchglu_forward_mxfp4_ws(x, il, wl, bank, ws, out=out)
    else:
        bank = qeg.QuantBank(*mat(INTER, HIDDEN, 0), *mat(INTER, HIDDEN, 1),
                             *mat(HIDDEN, INTER, 2))
        size = qeg.moe_workspace_size

        def call(x, il, wl, ws, out):
            qeg.moe_switchglu_forward_ws(x, il, wl, bank, ws, out=out)
    r = synth.route_uniform(TL, EL, K_TOP, SEED + 900 + TL)
    x = torch.from_numpy(synth.x_bf16(TL, HIDDEN, SEED + TL).view(np.int16)).to(dev) \
        .view(torch.bfloat16)
    il, wl = torch.from_numpy(r[0]).to(dev), torch.from_numpy(r[1]).to(dev)
    out = torch.empty((TL, HIDDEN), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(size(TL, K_TOP, EL, HIDDEN, INTER), dtype=torch.uint8, device=dev)
    for _ in range(3):
        call(x, il, wl, ws, out)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    call(x, il, wl, ws, out)
    b.record()
    torch.cuda.synchronize()
    return {"large_window_only": True, "T": TL, "mxfp4": bool(args.mxfp4),
            "us_per_layer": a.elapsed_time(b) * 1e3, "status": qeg.moe_read_device_status()}


def our_arm(args, world, rank, local):
    global E, LAYERS, TS, ROUTING
    E, LAYERS, ROUTING = args.experts, args.layers, args.routing
    if args.ts:
        TS = tuple(int(t) for t in args.ts.split(","))
    import torch
    import quantized_expert_gather_b200 as qeg
    import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    routes = routings()
    uq = uniques(routes)

    # bank: drawn on the device by the generator's CUDA twin (same bits as the host one)
    def mat(rows, cols, mid):
        q = torch.empty((E, rows, cols // 8), dtype=torch.int32, device=dev)
        s = torch.empty((E, rows, cols // 64), dtype=torch.int16, device=dev)
        b = torch.empty_like(s)
        synth.fill_bank_device(q, s, b, rows, cols, SEED, mid)
        return q, s.view(torch.bfloat16), b.view(torch.bfloat16)
    g, u, d = mat(INTER, HIDDEN, 0), mat(INTER, HIDDEN, 1), mat(HIDDEN, INTER, 2)
    bank = qeg.QuantBank(*g, *u, *d)
    torch.cuda.synchronize()

    xs = {T: torch.from_numpy(synth.x_bf16(T, HIDDEN, SEED + T).view(np.int16)).to(dev)
          .view(torch.bfloat16) for T in TS}
    idx = {T: [torch.from_numpy(r[0]).to(dev) for r in routes[T]] for T in TS}
    wts = {T: [torch.from_numpy(r[1]).to(dev) for r in routes[T]] for T in TS}
    outs = {T: [torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=dev)
                for _ in range(LAYERS)] for T in TS}
    ws = torch.zeros(max(qeg.moe_workspace_size(T, K_TOP, E, HIDDEN, INTER) for T in TS),
                     dtype=torch.uint8, device=dev)  # barrier words must start at zero

    def step():
        for T in TS:
            for l in range(LAYERS):
                qeg.moe_switchglu_forward_ws(xs[T], idx[T][l], wts[T][l], bank, ws,
                                             out=outs[T][l])

    launches_per_step = LAYERS * len(TS)  # one layer kernel per layer
    step()  # first call: per-device set-up, outside any capture
    torch.cuda.synchronize()
    if qeg.moe_read_device_status() != qeg.MOE_OK:
        raise RuntimeError("device error word set during warm-up")

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    total_bytes = sum(sum(uq[T]) for T in TS) * BYTES_PER_EXPERT
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        clk.wait_first()
        e0.record()
        for _ in range(args.steps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world)
    # every chained layer's output of the last timed replay, kept for the parity check
    kept = {T: [o.view(torch.int16).cpu().numpy().view(np.uint16) for o in outs[T]] for T in TS}
    ms_step = ms_total / args.steps
    all_bytes = sum_over_ranks(total_bytes * args.steps, world)
    gbs = all_bytes / (ms_total * 1e-3) / 1e9

    if args.quick:  # profiling runs: the timed graph replays only
        del graph
        return ({"quick": True, "value": gbs, "ms_per_step": ms_step, "clocks": clk.summary(),
                 "us_per_layer": ms_step * 1e3 / (LAYERS * len(TS))} if rank == 0 else None)
    # per-layer times (events between layers, chained; and isolated with an L2 flush)
    per = {}
    flush = torch.empty(4 * L2_BYTES, dtype=torch.uint8, device=dev)
    for T in TS:
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(LAYERS + 1)]
        ev[0].record()
        for l in range(LAYERS):
            qeg.moe_switchglu_forward_ws(xs[T], idx[T][l], wts[T][l], bank, ws, out=outs[T][l])
            ev[l + 1].record()
        torch.cuda.synchronize()
        chained = [ev[l].elapsed_time(ev[l + 1]) * 1e3 for l in range(LAYERS)]
        iso = []
        for l in range(LAYERS):
            flush.fill_(l & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            qeg.moe_switchglu_forward_ws(xs[T], idx[T][l], wts[T][l], bank, ws, out=outs[T][l])
            b.record()
            torch.cuda.synchronize()
            iso.append(a.elapsed_time(b) * 1e3)
        byt = [u_ * BYTES_PER_EXPERT for u_ in uq[T]]
        per[T] = {
            "mean_unique_experts": float(np.mean(uq[T])),
            "chained_us_per_layer": float(np.mean(chained)),
            "chained_gbs": sum(byt) / (sum(chained) * 1e-6) / 1e9,
            "isolated_us_per_layer_median": float(np.median(iso)),
            "isolated_gbs": sum(byt) / (sum(iso) * 1e-6) / 1e9,
        }
    graph_per_layer = {}
    for T in TS:
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            for l in range(LAYERS):
                qeg.moe_switchglu_forward_ws(xs[T], idx[T][l], wts[T][l], bank, ws,
                                             out=outs[T][l])
        g2.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            g2.replay()
        b.record()
        torch.cuda.synchronize()
        us = a.elapsed_time(b) * 1e3 / (5 * LAYERS)
        per[T]["graph_us_per_layer"] = us
        per[T]["graph_gbs"] = sum(uq[T]) * BYTES_PER_EXPERT / LAYERS / (us * 1e-6) / 1e9
        del g2

    # speculative-verify pair (E=256): a T=2 window against its first token alone, 42
    # chained layers each, CUDA graph, swept over the adjacent-token overlap p of the
    # pages' measurements; the target is T=2 <= 1.7 x T=1 at p = 0.34
    verify = None
    E2 = 256
    bank2 = None
    if not args.no_verify_pair:
        def mat2(rows, cols, mid):
            q = torch.empty((E2, rows, cols // 8), dtype=torch.int32, device=dev)
            s_ = torch.empty((E2, rows, cols // 64), dtype=torch.int16, device=dev)
            b_ = torch.empty_like(s_)
            synth.fill_bank_device(q, s_, b_, rows, cols, SEED + 1, mid)
            return q, s_.view(torch.bfloat16), b_.view(torch.bfloat16)
        bank2 = qeg.QuantBank(*mat2(INTER, HIDDEN, 0), *mat2(INTER, HIDDEN, 1),
                              *mat2(HIDDEN, INTER, 2))
        x2 = torch.from_numpy(synth.x_bf16(2, HIDDEN, SEED + 2).view(np.int16)).to(dev) \
            .view(torch.bfloat16)
        ws2 = torch.zeros(qeg.moe_workspace_size(2, K_TOP, E2, HIDDEN, INTER), dtype=torch.uint8,
                          device=dev)
        verify = {"E": E2, "target_ratio": 1.7, "target_p": 0.34, "layers": LAYERS, "p": {}}
        for p in VERIFY_PS:
            pairs = [synth.route_verify_pair(E2, K_TOP, p, SEED + 500 + int(p * 1000) + l)
                     for l in range(LAYERS)]
            runs = {}
            for T2 in (1, 2):
                ids = [torch.from_numpy(np.ascontiguousarray(r[0][:T2])).to(dev) for r in pairs]
                wv = [torch.from_numpy(np.ascontiguousarray(r[1][:T2])).to(dev) for r in pairs]
                o2 = [torch.empty((T2, HIDDEN), dtype=torch.bfloat16, device=dev) for _ in pairs]
                xs2 = x2[:T2]
                runs[T2] = graph_us_per_layer(
                    lambda: [qeg.moe_switchglu_forward_ws(xs2, ids[l], wv[l], bank2, ws2,
                                                          out=o2[l]) for l in range(LAYERS)],
                    LAYERS)
            u2 = float(np.mean([np.unique(r[0]).size for r in pairs]))
            verify["p"][str(p)] = {
                "t1_us_per_layer": runs[1], "t2_us_per_layer": runs[2],
                "ratio_t2_over_t1": runs[2] / runs[1], "mean_unique_t2": u2,
                "t2_gbs": u2 * BYTES_PER_EXPERT / (runs[2] * 1e-6) / 1e9,
                "t1_gbs": 8 * BYTES_PER_EXPERT / (runs[1] * 1e-6) / 1e9}
        del ws2
        torch.cuda.synchronize()

    # verify-window sweep: T in {2,3,5,8,16} on an adjacent-overlap chain at p = 0.40, a
    # stack of 78 layers with independent seeded weights per layer; each layer's bank is
    # compacted to the experts its window routes to (fresh memory per layer, ids remapped),
    # so no expert repeats across the stack and L2 gives no reuse; graph of the stack
    window = None
    if not args.no_window_sweep:
        window = {"E": E2, "p": 0.40, "layers": WINDOW_LAYERS, "per_T": {}}
        for TW in WINDOW_TS:
            stack = window_stack(TW, dev, qeg, synth)
            us = graph_us_per_layer(
                lambda: [qeg.moe_switchglu_forward_ws(st["x"], st["idx"], st["w"], st["bank"],
                                                      st["ws"], out=st["out"])
                         for st in stack["layers"]], len(stack["layers"]))
            ub = stack["unique"]
            window["per_T"][str(TW)] = {
                "us_per_layer": us, "us_per_stack": us * len(ub),
                "mean_unique": float(np.mean(ub)),
                "gbs": float(np.sum(ub)) * BYTES_PER_EXPERT / (us * len(ub) * 1e-6) / 1e9,
                "frac_of_hbm_peak": float(np.sum(ub)) * BYTES_PER_EXPERT
                / (us * len(ub) * 1e-6) / 1e9 / measured_peaks()[0],
                "stack_bytes": float(np.sum(ub)) * BYTES_PER_EXPERT}
            del stack
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        # the all-identical extreme: every token of a T=16 window routes to the same 8
        # experts (16 pairs per expert), which must still stream once; 42 chained layers,
        # layer l on experts 8l .. 8l+7 of the E=256 bank (mod 256), so consecutive layers
        # share no expert
        wsame = np.full((16, K_TOP), 1.0 / K_TOP, np.float32)
        ws3 = torch.zeros(qeg.moe_workspace_size(16, K_TOP, E2, HIDDEN, INTER), dtype=torch.uint8,
                          device=dev)
        xi = torch.from_numpy(synth.x_bf16(16, HIDDEN, SEED + 16).view(np.int16)).to(dev) \
            .view(torch.bfloat16)
        ii = [torch.from_numpy(np.tile((np.arange(K_TOP) + K_TOP * l) % E2, (16, 1))
                               .astype(np.int32)).to(dev) for l in range(LAYERS)]
        wi = torch.from_numpy(wsame).to(dev)
        oi = [torch.empty((16, HIDDEN), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        us = graph_us_per_layer(
            lambda: [qeg.moe_switchglu_forward_ws(xi, ii[l], wi, bank2, ws3, out=oi[l])
                     for l in range(LAYERS)], LAYERS)
        window["all_identical_T16"] = {
            "us_per_layer": us, "unique": K_TOP, "pairs_per_expert": 16,
            "gbs": K_TOP * BYTES_PER_EXPERT / (us * 1e-6) / 1e9,
            "frac_of_hbm_peak": K_TOP * BYTES_PER_EXPERT / (us * 1e-6) / 1e9
            / measured_peaks()[0]}
        del ws3
    # mxfp4 banks: GLM-5.2's routed bank (E=256, hidden 6144, intermediate 2048, e2m1
    # codes with one e8m0 scale per 32 columns, 20,054,016 B per expert), drawn on the
    # device; 42 chained layers with distinct adjacent-overlap routings (p = 0.34) per
    # window size, CUDA graph; GB/s over unique-expert mxfp4 bytes
    mxfp4 = None
    if not args.no_mxfp4:
        EM, HM, IM = 256, 6144, 2048
        bpe_mx = 3 * (IM * HM // 2 + IM * HM // 32)

        def matm(rows, cols, mid):
            q = torch.empty((EM, rows, cols // 8), dtype=torch.int32, device=dev)
            e8 = torch.empty((EM, rows, cols // 32), dtype=torch.uint8, device=dev)
            synth.fill_bank_mxfp4_device(q, e8, rows, cols, SEED + 3, mid)
            return q, e8
        bank_mx = qeg.MxBank(*matm(IM, HM, 0), *matm(IM, HM, 1), *matm(HM, IM, 2))
        mxfp4 = {"E": EM, "hidden": HM, "inter": IM, "bytes_per_expert": bpe_mx, "p": 0.34,
                 "layers": LAYERS, "per_T": {}}
        for TM in (1, 2, 4, 16):
            rts = [synth.route_markov(TM, EM, K_TOP, 0.34, SEED + 7000 + 100 * TM + l)
                   for l in range(LAYERS)]
            xm = torch.from_numpy(synth.x_bf16(TM, HM, SEED + 60 + TM).view(np.int16)).to(dev) \
                .view(torch.bfloat16)
            im = [torch.from_numpy(r[0]).to(dev) for r in rts]
            wm = [torch.from_numpy(r[1]).to(dev) for r in rts]
            om = [torch.empty((TM, HM), dtype=torch.bfloat16, device=dev) for _ in rts]
            wsm = torch.zeros(qeg.moe_workspace_size_mxfp4(TM, K_TOP, EM, HM, IM),
                              dtype=torch.uint8, device=dev)
            us = graph_us_per_layer(
                lambda: [qeg.moe_switchglu_forward_mxfp4_ws(xm, im[l], wm[l], bank_mx, wsm,
                                                            out=om[l]) for l in range(LAYERS)],
                LAYERS)
            um = float(np.mean([np.unique(r[0]).size for r in rts]))
            gb = um * bpe_mx / (us * 1e-6) / 1e9
            mxfp4["per_T"][str(TM)] = {"us_per_layer": us, "mean_unique": um, "gbs": gb,
                                       "frac_of_hbm_peak": gb / measured_peaks()[0]}
            del wsm
        # a large window on the same bank: T=512, uniform top-8 routing (every expert
        # used), the grouped tensor-core path; 3 layers between CUDA events after a warm
        # pass; bytes = unique experts, flops = 6 P H I
        if not args.no_large_t:
            TL, nl = 512, 3
            rl = [synth.route_uniform(TL, EM, K_TOP, SEED + 7900 + l) for l in range(nl)]
            xl = torch.from_numpy(synth.x_bf16(TL, HM, SEED + 79).view(np.int16)).to(dev) \
                .view(torch.bfloat16)
            il = [torch.from_numpy(r[0]).to(dev) for r in rl]
            wl = [torch.from_numpy(r[1]).to(dev) for r in rl]
            ol = torch.empty((TL, HM), dtype=torch.bfloat16, device=dev)
            wsl = torch.zeros(qeg.moe_workspace_size_mxfp4(TL, K_TOP, EM, HM, IM),
                              dtype=torch.uint8, device=dev)
            for l in range(nl):  # warm
                qeg.moe_switchglu_forward_mxfp4_ws(xl, il[l], wl[l], bank_mx, wsl, out=ol)
            torch.cuda.synchronize()
            a5, b5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a5.record()
            for l in range(nl):
                qeg.moe_switchglu_forward_mxfp4_ws(xl, il[l], wl[l], bank_mx, wsl, out=ol)
            b5.record()
            torch.cuda.synchronize()
            us = a5.elapsed_time(b5) * 1e3 / nl
            ul = float(np.mean([np.unique(r[0]).size for r in rl]))
            gbl = ul * bpe_mx / (us * 1e-6) / 1e9
            mxfp4["large_window"] = {
                "T": TL, "us_per_layer": us, "mean_unique": ul, "gbs": gbl,
                "frac_of_hbm_peak": gbl / measured_peaks()[0],
                "tflops": 6.0 * TL * K_TOP * HM * IM / (us * 1e-6) / 1e12,
                "path": "grouped tcgen05 kernels (5 launches per layer)"}
            del wsl
        del bank_mx
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    # large windows (the grouped tensor-core path): T=512 and T=2048 on the E=256 bank,
    # a few layers each, CUDA events; bytes = unique experts, flops = 6 P H I
    large = None
    if bank2 is not None and not args.no_large_t:
        large = {}
        for TL, nl in ((512, 3), (2048, 2)):
            rl = [synth.route_uniform(TL, E2, K_TOP, SEED + 900 + TL + l) for l in range(nl)]
            xl = torch.from_numpy(synth.x_bf16(TL, HIDDEN, SEED + TL).view(np.int16)).to(dev) \
                .view(torch.bfloat16)
            il = [torch.from_numpy(r[0]).to(dev) for r in rl]
            wl = [torch.from_numpy(r[1]).to(dev) for r in rl]
            ol = torch.empty((TL, HIDDEN), dtype=torch.bfloat16, device=dev)
            wsl = torch.zeros(qeg.moe_workspace_size(TL, K_TOP, E2, HIDDEN, INTER),
                              dtype=torch.uint8, device=dev)
            for l in range(nl):  # warm
                qeg.moe_switchglu_forward_ws(xl, il[l], wl[l], bank2, wsl, out=ol)
            torch.cuda.synchronize()
            a4, b4 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a4.record()
            for l in range(nl):
                qeg.moe_switchglu_forward_ws(xl, il[l], wl[l], bank2, wsl, out=ol)
            b4.record()
            torch.cuda.synchronize()
            us = a4.elapsed_time(b4) * 1e3 / nl
            ul = float(np.mean([np.unique(r[0]).size for r in rl]))
            fl = 6.0 * TL * K_TOP * HIDDEN * INTER
            gbl = ul * BYTES_PER_EXPERT / (us * 1e-6) / 1e9
            large[str(TL)] = {"us_per_layer": us, "mean_unique": ul, "unique_gbs": gbl,
                              "frac_of_hbm_peak": gbl / measured_peaks()[0],
                              "tflops": fl / (us * 1e-6) / 1e12,
                              "path": "grouped tcgen05 kernels (5 launches per layer)"}
            del wsl
    if bank2 is not None:
        del bank2

    # the router step ahead of the layer (top-k of softmax, renormalised): 20 calls
    # captured in a CUDA graph, replayed 20 times between CUDA events (device time,
    # no per-call host overhead); also the per-call time through the Python binding
    router = None
    try:
        rt, rt_host = {}, {}
        for TR in (1, 4, 16):
            lg = torch.from_numpy(np.random.default_rng(SEED + 70 + TR).standard_normal(
                (TR, E)).astype(np.float32)).to(dev)
            ri = torch.empty((TR, K_TOP), dtype=torch.int32, device=dev)
            rw = torch.empty((TR, K_TOP), dtype=torch.float32, device=dev)
            for _ in range(10):
                qeg.moe_router_topk(lg, K_TOP, topk_idx=ri, topk_w=rw)
            torch.cuda.synchronize()
            a5, b5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a5.record()
            for _ in range(200):
                qeg.moe_router_topk(lg, K_TOP, topk_idx=ri, topk_w=rw)
            b5.record()
            torch.cuda.synchronize()
            rt_host[str(TR)] = a5.elapsed_time(b5) * 1e3 / 200
            g5 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g5):
                for _ in range(20):
                    qeg.moe_router_topk(lg, K_TOP, topk_idx=ri, topk_w=rw)
            g5.replay()
            torch.cuda.synchronize()
            a5.record()
            for _ in range(20):
                g5.replay()
            b5.record()
            torch.cuda.synchronize()
            rt[str(TR)] = a5.elapsed_time(b5) * 1e3 / 400
            del g5
        # the router fused into the layer (one launch) against the router kernel then the
        # layer (two), 42 chained layers each on the bench bank, CUDA graph; per layer
        fused, two = {}, {}
        for TR in (1, 4, 16):
            lgs = [torch.from_numpy(np.random.default_rng(SEED + 80 + 100 * TR + l)
                                    .standard_normal((TR, E)).astype(np.float32)).to(dev)
                   for l in range(LAYERS)]
            xr = torch.from_numpy(synth.x_bf16(TR, HIDDEN, SEED + TR).view(np.int16)).to(dev) \
                .view(torch.bfloat16)
            orr = torch.empty((TR, HIDDEN), dtype=torch.bfloat16, device=dev)
            ri = torch.empty((TR, K_TOP), dtype=torch.int32, device=dev)
            rw = torch.empty((TR, K_TOP), dtype=torch.float32, device=dev)
            wsr = torch.zeros(qeg.moe_workspace_size(TR, K_TOP, E, HIDDEN, INTER),
                              dtype=torch.uint8, device=dev)
            fused[str(TR)] = graph_us_per_layer(
                lambda: [qeg.moe_switchglu_forward_routed(xr, lgs[l], K_TOP, bank, workspace=wsr,
                                                          out=orr, topk_idx=ri, topk_w=rw)
                         for l in range(LAYERS)], LAYERS)

            def two_step():
                for l in range(LAYERS):
                    qeg.moe_router_topk(lgs[l], K_TOP, topk_idx=ri, topk_w=rw)
                    qeg.moe_switchglu_forward_ws(xr, ri, rw, bank, wsr, out=orr)
            two[str(TR)] = graph_us_per_layer(two_step, LAYERS)
            del wsr
        router = {"E": E, "k": K_TOP, "renormalize": True, "us_per_call_graph": rt,
                  "us_per_call_python": rt_host,
                  "router_and_layer_us_per_layer_graph": {"fused_one_launch": fused,
                                                          "router_then_layer": two}}
    except Exception as ex:  # report, never lose the headline line
        router = {"error": repr(ex)}

    # end to end through the public call: pinned host inputs in, outputs back, each step
    pin_x = {T: torch.from_numpy(synth.x_bf16(T, HIDDEN, SEED + T).view(np.int16)).pin_memory()
             for T in TS}
    pin_idx = {T: torch.from_numpy(np.stack([r[0] for r in routes[T]])).pin_memory() for T in TS}
    pin_w = {T: torch.from_numpy(np.stack([r[1] for r in routes[T]])).pin_memory() for T in TS}
    pin_out = {T: torch.empty((LAYERS, T, HIDDEN), dtype=torch.bfloat16).pin_memory() for T in TS}
    d_idx = {T: torch.empty((LAYERS, T, K_TOP), dtype=torch.int32, device=dev) for T in TS}
    d_w = {T: torch.empty((LAYERS, T, K_TOP), dtype=torch.float32, device=dev) for T in TS}
    d_out = {T: torch.empty((LAYERS, T, HIDDEN), dtype=torch.bfloat16, device=dev) for T in TS}
    h2d = sum(pin_x[T].numel() * 2 + pin_idx[T].numel() * 4 + pin_w[T].numel() * 4 for T in TS)
    d2h = sum(pin_out[T].numel() * 2 for T in TS)

    def e2e_step():
        for T in TS:
            xs[T].view(torch.int16).copy_(pin_x[T], non_blocking=True)
            d_idx[T].copy_(pin_idx[T], non_blocking=True)
            d_w[T].copy_(pin_w[T], non_blocking=True)
            for l in range(LAYERS):
                qeg.moe_switchglu_forward(xs[T], d_idx[T][l], d_w[T][l], bank, out=d_out[T][l])
            pin_out[T].copy_(d_out[T], non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        e2e_step()
    b.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b), world)
    e2e_gbs = sum_over_ranks(total_bytes * args.steps, world) / (e2e_ms * 1e-3) / 1e9
    status = qeg.moe_read_device_status()
    if status != qeg.MOE_OK:
        raise RuntimeError(f"device error word: {qeg.moe_status_str(status)}")

    peak, peak_kind = measured_peaks()
    layer_bytes = {T: float(np.mean(uq[T])) * BYTES_PER_EXPERT for T in TS}
    # dominant kernel: the layer kernel (one launch per layer); algorithmic bytes per
    # launch = u * 14,155,776, time = its average duration inside graph replays
    tot_b = sum(layer_bytes[T] for T in TS)
    tot_us = sum(per[T]["graph_us_per_layer"] for T in TS)
    achieved = tot_b / (tot_us * 1e-6) / 1e9
    tr = captured_traffic()
    # per launch, averaged like `achieved` over the launches of a step (scaled by the
    # launches' unique experts from the small-case capture)
    traffic = (None if tr is None else
               tr[0] * sum(float(np.mean(uq[T])) for T in TS) / len(TS) + tr[1])
    result = None
    chained_parity = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cgbs, nl, secs, thr, chained_parity = run_oracle_sample(
                routes, budget_s=args.cpu_budget, gpu_outs=kept)
            cpu = {"value": cgbs, "unit": "GB/s", "cores": thr, "kind": "oracle",
                   "sample": f"{nl} whole layers of the workload (each of the 84 layers once, "
                             f"then the last T=1 and T=4 layers again), {secs:.1f} s of "
                             f"oracle time, unique-expert bytes"}
        result = {
            "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE_LABEL,
            "data": "synthetic",
            "config": {"workload": "GLM-5.3-Flash-shaped union-of-experts SwitchGLU layer: "
                                   "E=288 top-8 hidden 4096 inter 2048 q4 affine g64 bf16 "
                                   "scale/bias; 42 chained layers at T=1 then 42 at T=4 per step",
                       "T": list(TS), "layers_per_T": LAYERS, "routing": "uniform top-8",
                       "bytes_per_expert": BYTES_PER_EXPERT,
                       "l2": "inputs larger than L2 (4.08 GB bank; >20 GB streamed per step)",
                       "timing": "CUDA graph of the 84 layer calls, CUDA events",
                       "parallelism": f"replicas x{world}"},
            "us_per_layer": {str(T): per[T]["graph_us_per_layer"] for T in TS},
            "per_T": {str(T): per[T] for T in TS},
            "frac_of_peak": gbs / peak, "frac_of_nominal_8TBs": gbs / 8000.0,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind,
                         "kernel": "layer_kernel (one launch per layer)",
                         "traffic": traffic,
                         "algorithmic_bytes_per_launch": tot_b / len(TS),
                         "traffic_source": "ncu dram__bytes_read.sum+dram__bytes_write.sum of a "
                                           "T=1 and a T=4 launch (E=96 bank), scaled per unique "
                                           "expert to this workload"},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h),
                    "how": "moe_switchglu_forward per layer, pinned host inputs copied in and "
                           "all layer outputs copied back every step"},
            "chained_parity": chained_parity,
            "verify_pair": verify,
            "verify_window": window,
            "mxfp4": mxfp4,
            "large_window": large,
            "router": router,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
    del graph
    return result


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--layers", type=int, default=42, help="chained layers per T (profiling)")
    ap.add_argument("--experts", type=int, default=288, help="bank size (profiling)")
    ap.add_argument("--quick", action="store_true", help="timed graph only (profiling)")
    ap.add_argument("--no-large-t", action="store_true",
                    help="skip the T=512 / T=2048 grouped-path measurement")
    ap.add_argument("--no-verify-pair", action="store_true",
                    help="skip the T=2 / T=1 speculative-verify measurement")
    ap.add_argument("--no-mxfp4", action="store_true",
                    help="skip the mxfp4 (GLM-5.2 bank) measurement")
    ap.add_argument("--no-window-sweep", action="store_true",
                    help="skip the verify-window sweep (T=2..16, 78-layer stacks)")
    ap.add_argument("--ts", default="", help="comma-separated window sizes (profiling)")
    ap.add_argument("--mxfp4", action="store_true",
                    help="with --large-window-only: the same shape on an mxfp4 bank")
    ap.add_argument("--large-window-only", action="store_true",
                    help="one grouped-path layer alone (T from --ts, default 512; profiling)")
    ap.add_argument("--routing", default="uniform", choices=("uniform", "markov", "identical"),
                    help="routing model (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            return reference_arm(args, world, rank)
        res = large_window_only(args, local) if args.large_window_only else \
            our_arm(args, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
