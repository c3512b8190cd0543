#!/usr/bin/env python
"""Benchmark of the SALAD hybrid-attention forward layer (one layer = one step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of synthetic input:
gate, Top-K selection (or ST-SWA regrouping), linear-attention state, and the
sparse attention kernel with the fused gated linear term.  The default
workload is the 480p-like Top-K layer (B=1, H=12, d=128, N=31200, 488 blocks,
k=49, ~90% sparsity).

Metric: effective TFLOP/s counting only computed work -- 4*d*64^2 per kept
(query block, key block) pair plus 6*N*d^2 + 4*N*d per head for the linear
branch -- over the device time of K back-to-back steps (CUDA events, max over
ranks).  ms per layer is reported beside it.  Inputs (Q, K, V, X: 384 MB at the
default size) exceed the 126 MB L2, so no flush is inserted between steps.

Multi-GPU (torchrun): every rank runs an independent replica of the layer on
its own GPU (weak scaling, no collective on the data path); NCCL is used only
for the barrier and the max-over-ranks reduction of the elapsed time.

--impl reference times the CPU oracle on a bounded sample of the same
workload (rank 0 only) and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ms/layer & effective TFLOP/s, SALAD attn fwd N=31200 90% sparse; % roofline"
UNIT = "effective TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ work ---
def step_flops(w) -> dict:
    """Algorithmic work of one layer (counted, not executed, flops)."""
    B, H, N, d, bs = w.B, w.H, w.N, w.d, w.block
    nb = w.nb
    if w.mode == "topk":
        pairs = B * H * nb * w.topk
        sparse = 4.0 * d * bs * bs * pairs
    elif w.mode == "swa":
        # Exact (query, key) pairs inside the window, clipped at the ends.
        W = w.window
        per_head = sum(min(N - 1, r + W) - max(0, r - W) + 1 for r in range(N))
        sparse = 4.0 * d * per_head * B * H
    else:
        sparse = 4.0 * d * N * N * B * H
    linear = (6.0 * N * d * d + 4.0 * N * d) * B * H
    # The attention kernel itself: the sparse branch plus phi(Q) (H W_lin).
    attn_kernel = sparse + 2.0 * N * d * d * B * H
    dense = 4.0 * d * N * N * B * H
    return {"sparse": sparse, "linear": linear, "total": sparse + linear,
            "attn_kernel": attn_kernel, "dense": dense}


def input_bytes(w) -> int:
    """Bytes of one layer's inputs: Q, K, V, X, the gate weight and W_lin (bf16)."""
    return 2 * (3 * w.B * w.H * w.N * w.d + w.B * w.N * w.D + w.D + w.H * w.d * w.d)


def config_of(w, world: int) -> dict:
    """The workload's `config` dict, identical in both arms of the benchmark."""
    fl = step_flops(w)
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
            "block": w.block, "mode": w.mode, "topk": w.topk, "window": w.window,
            "nb": w.nb, "D": w.D,
            "sparsity": round(1 - fl["sparse"] / fl["dense"], 4),
            "parallelism": f"replicas{world}",
            "l2": "no flush: inputs (Q,K,V,X) %.0f MB > 126 MB L2" % (input_bytes(w) / 1e6)}


def choose_peak(peaks: dict, timed_ms: float, clk: dict):
    """The bf16 peak a kernel timed inside this run is held to.

    The burst figure (a GEMM timed alone at full clocks) applies when the
    timed region is short -- under a second -- and the SM clock sampled
    during it stayed at its maximum; a seconds-long region, or one whose
    clock sagged under the power cap, is held to the sustained figure.
    Returns (peak, label)."""
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained") or burst)
    mhz, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    at_max = mhz is not None and mx is not None and mhz >= 0.97 * mx
    if timed_ms < 1000.0 and (at_max or mhz is None):
        return burst, "bf16 burst"
    return sustained, "bf16 sustained"


def launches_per_step(w) -> int:
    # gate (2) + [pool, scores, selection | gather] + linear state and
    # reduce+fold (2) + attention (1)
    if w.mode == "topk":
        return 2 + 3 + 2 + 1
    if w.mode == "swa":
        return 2 + (1 if w.space_major_heads else 0) + 2 + 1
    return 2 + 2 + 1


def load_peaks() -> tuple:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("attn.cu", "common.cuh", "internal.h"):
        with open(os.path.join(ROOT, "sparse_linear_hybrid_top_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, if the
    kernel source is unchanged since it was captured; else None."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    ent = rec.get(workload)
    if not ent or ent.get("attn_source_hash") != attn_source_hash():
        return None
    return ent.get("bytes_per_launch")


# ---------------------------------------------------------------- clocks ---
class ClockSampler:
    """SM clock and throttle reasons sampled during a region.

    A thread polls NVML about every half millisecond (a timed region of a
    few dozen steps lasts only tens of milliseconds, shorter than
    nvidia-smi's own sampling period); where NVML cannot be opened, an
    `nvidia-smi -lms 100` child is the fallback and `start()` waits for its
    first sample. Reading clocks changes nothing on the GPU."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits.
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.first = threading.Event()
        self.sm, self.mx, self.reasons = [], [], set()
        self.source = None
        self.nvml = None
        self.handle = None

    def _nvml_handle(self):
        import pynvml
        import torch
        p = torch.cuda.get_device_properties(self.dev)
        pynvml.nvmlInit()
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            pci = pynvml.nvmlDeviceGetPciInfo(h)
            if (pci.domain, pci.bus, pci.device) == (p.pci_domain_id, p.pci_bus_id, p.pci_device_id):
                return pynvml, h
        pynvml.nvmlShutdown()
        return None, None

    def start(self):
        try:
            self.nvml, self.handle = self._nvml_handle()
        except Exception:       # no NVML library or no matching device
            self.nvml, self.handle = None, None
        if self.handle is not None:
            self.source = "nvml"
            self.mx.append(float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                     self.nvml.NVML_CLOCK_SM)))
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
        else:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, ValueError):
                self.proc = None
                return
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()
        self.first.wait(timeout=3.0)

    def _poll_nvml(self):
        nv, h = self.nvml, self.handle
        while not self.stop_flag.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                break
            for n, bit in self.REASON_BITS.items():
                if mask & bit:
                    self.reasons.add(n)
            self.first.set()
            time.sleep(0.0005)

    def _read_smi(self):
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.proc.stdout:
            parts = [p.strip() for p in ln.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            if self.stop_flag.is_set():
                continue
            self.sm.append(sm)
            self.mx.append(mx)
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    self.reasons.add(n)
            self.first.set()

    def stop(self) -> dict:
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0,
                    "reasons": ["no clock source (NVML and nvidia-smi unavailable)"]}
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.thread.join(timeout=5)
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        sm = list(self.sm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": max(self.mx) if self.mx else None,
                "samples": len(sm), "source": self.source,
                "reasons": sorted(self.reasons)}


# ---------------------------------------------------------- distributed ---
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str, world: int):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(value: float, device) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(world: int, flops_per_step: float, steps: int, max_ms: float) -> dict:
    """Whole-job throughput of `world` replicas that each ran `steps` steps,
    timed as the max over ranks."""
    total = world * flops_per_step * steps
    return {"value": total / (max_ms * 1e-3) / 1e12, "ms_per_step": max_ms / steps}


# ------------------------------------------------------------ CPU oracle ---
def cpu_sample_work(w, inp, n_heads: int, blocks_per_head: int, seed: int = 0):
    """Runs the oracle on a bounded sample of the layer; returns (flops, seconds).

    The sample: the gate over all of X, then for `n_heads` heads the block
    selection (all query blocks), the linear state, and for `blocks_per_head`
    query blocks the sparse attention plus the linear term of their rows.
    Counted flops follow the metric's rule restricted to the sample."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    B, H, N, d, bs = w.B, w.H, w.N, w.d, w.block
    heads = [(int(rng.integers(B)), int(h)) for h in rng.choice(H, size=min(n_heads, H), replace=False)]
    t0 = time.perf_counter()
    s = oracle.gate(inp["x"], inp["w_gate"], inp["bias"])
    flops = 0.0
    for b, h in heads:
        q, k, v = (oracle.as64(inp[n][b, h]) for n in ("q", "k", "v"))
        Hst, Z = oracle.linear_state(k, v)
        flops += 2.0 * N * d * d + N * d
        blocks = rng.choice(w.nb, size=min(blocks_per_head, w.nb), replace=False)
        if w.mode == "topk":
            idx = oracle.select_topk(oracle.block_scores(q, k, bs), w.topk)
            res = oracle.topk_attention_rows(q, k, v, idx, bs, blocks)
            kept = w.topk
        else:
            res = {}
            for i in blocks:
                rows = np.arange(i * bs, min(N, (i + 1) * bs))
                res[i] = (oracle.swa_attention_rows(q, k, v, w.window, rows) if w.mode == "swa"
                          else oracle.dense_attention(q[rows], k, v))
            kept = min(w.nb, (2 * w.window) // bs + 1) if w.mode == "swa" else w.nb
        for i in blocks:
            rows = np.arange(i * bs, min(N, (i + 1) * bs))
            o_l = oracle.linear_apply(q[rows], Hst, Z, w.eps)
            oracle.combine(res[i], o_l, oracle.as64(inp["w_lin"][h]), s[b])
            flops += 4.0 * d * bs * bs * kept + len(rows) * (4.0 * d * d + 4.0 * d)
    return flops, time.perf_counter() - t0


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------- sweep ---
# "name+regroup_in_load": the workload with its ST-SWA heads regrouped inside
# the attention's loads instead of copied (the library's non-default form).
SWEEP = ("swa480", "swa480+regroup_in_load", "topk720", "cfg_b2h40_s80", "cfg_b2h40_s90",
         "cfg_b2h40_s95", "cfg_b2h40_all")


def run_sweep(names, device, stream, peaks, steps: int = 5, warmup: int = 2) -> dict:
    """The other workloads of the method's video shapes, each timed like the
    headline (one salad_forward per step, CUDA events on the launch stream)
    next to the same library's dense attention on the same Q, K, V.  Inputs
    are drawn on the device with the synthetic recipe (``generate_device``:
    same distributions and frame structure, not the host generator's bytes,
    whose draws take minutes at these sizes)."""
    import torch
    import sparse_linear_hybrid_top_b200 as salad
    from synth import WORKLOADS, generate_device
    out = {}
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained") or burst)
    for name in names:
        base, _, option = name.partition("+")
        w = WORKLOADS[base]
        dev = generate_device(w, device, seed=w.seeds[0])
        extra = {}
        if w.mode == "swa":
            extra = dict(window=w.window, space_major_heads=w.space_major_heads, F=w.F,
                         Hh=w.Hh, Wh=w.Wh)
        if option == "regroup_in_load":
            extra["regroup_in_load"] = True
        plan = salad.ForwardPlan(dev["q"], dev["k"], dev["v"], dev["x"], dev["w_gate"],
                                 dev["w_lin"], mode=w.mode, topk=w.topk, bias=w.bias, eps=w.eps,
                                 **extra)
        for _ in range(warmup):
            plan.run(stream)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for e5 in ev:
            for e in e5:
                e.record(stream)
        torch.cuda.synchronize(device)
        t0.record(stream)
        for i in range(steps):
            plan.set_phase_events(ev[i])
            plan.run(stream)
        t1.record(stream)
        torch.cuda.synchronize(device)
        plan.set_phase_events(None)
        salad.check_error(stream)
        ms = t0.elapsed_time(t1) / steps
        attn = statistics.fmean(e5[3].elapsed_time(e5[4]) for e5 in ev)
        pre = statistics.fmean(e5[0].elapsed_time(e5[3]) for e5 in ev)
        salad.dense_attn(dev["q"], dev["k"], dev["v"], stream=stream)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nd = 2
        d0.record(stream)
        for _ in range(nd):
            salad.dense_attn(dev["q"], dev["k"], dev["v"], stream=stream)
        d1.record(stream)
        torch.cuda.synchronize(device)
        dense_ms = d0.elapsed_time(d1) / nd
        fl = step_flops(w)
        ach = fl["attn_kernel"] / (attn * 1e-3) / 1e12
        out[name] = {
            "B": w.B, "H": w.H, "N": w.N, "mode": w.mode, "topk": w.topk, "window": w.window,
            "sparsity": round(1 - fl["sparse"] / fl["dense"], 4),
            "ms_per_layer": round(ms, 4),
            "value": round(fl["total"] / (ms * 1e-3) / 1e12, 2),
            "phases_ms": {"pre_attention": round(pre, 4), "attention": round(attn, 4)},
            "attention_tflops": round(ach, 1),
            "attention_frac_of_burst": round(ach / burst, 4),
            "attention_frac_of_sustained": round(ach / sustained, 4),
            "dense_ms": round(dense_ms, 3),
            "dense_tflops": round(fl["dense"] / (dense_ms * 1e-3) / 1e12, 1),
            "speedup_vs_dense": round(dense_ms / ms, 3),
            "attention_speedup_vs_dense": round(dense_ms / attn, 3),
        }
        del plan, dev
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ runs ---
def run_ours(args, w) -> int:
    import torch
    world, rank, local = dist_env()
    if world != args.gpus:
        print(json.dumps({"error": f"WORLD_SIZE={world} but --gpus {args.gpus}"}), flush=True)
        return 2
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist("nccl", world)
    import sparse_linear_hybrid_top_b200 as salad
    from synth import generate, generate_projections

    host = generate(w)
    dev = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
    extra = {}
    if w.mode == "swa":
        extra = dict(window=w.window, space_major_heads=w.space_major_heads, F=w.F, Hh=w.Hh,
                     Wh=w.Wh)
    plan = salad.ForwardPlan(dev["q"], dev["k"], dev["v"], dev["x"], dev["w_gate"], dev["w_lin"],
                             mode=w.mode, topk=w.topk, bias=w.bias, eps=w.eps, **extra)
    stream = torch.cuda.current_stream(device)
    fl = step_flops(w)

    for _ in range(args.warmup):
        plan.run(stream)
    salad.check_error(stream)

    # Phase events: 5 per step, recorded by the library on the launch stream.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device())
    for e5 in ev:                 # create the handles before the timed region
        for e in e5:
            e.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    clocks.start()
    start.record(stream)
    for i in range(args.steps):
        plan.set_phase_events(ev[i])
        plan.run(stream)
    end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    plan.set_phase_events(None)
    salad.check_error(stream)
    local_ms = start.elapsed_time(end)
    max_ms = reduce_max(local_ms, device)
    agg = aggregate(world, fl["total"], args.steps, max_ms)

    def phase(a, b):
        return statistics.fmean(e5[a].elapsed_time(e5[b]) for e5 in ev)
    # The gate and the linear branch run on side streams beside the sparse
    # pattern: the first three figures are times from the start of the step.
    phases = {"gate_done": phase(0, 1), "pattern_done": phase(0, 2),
              "pre_attention": phase(0, 3), "attention": phase(3, 4)}
    attn_ms = phases["attention"]

    # Dense comparator on the same Q, K, V (same library).
    for _ in range(2):
        salad.dense_attn(dev["q"], dev["k"], dev["v"], stream=stream)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nd = max(2, min(10, args.steps))
    d0.record(stream)
    for _ in range(nd):
        salad.dense_attn(dev["q"], dev["k"], dev["v"], stream=stream)
    d1.record(stream)
    torch.cuda.synchronize(device)
    dense_ms = d0.elapsed_time(d1) / nd

    # The optional parts of the layer, timed the same way (diagnostics; the
    # headline above is the default layer): the 3-D rotary encoding in the
    # linear branch, and post-training branch dropping with every sample
    # below the threshold (the sparse branch alone plus the gate).
    def time_plan(p, n):
        for _ in range(3):
            p.run(stream)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n):
            p.run(stream)
        t1.record(stream)
        torch.cuda.synchronize(device)
        salad.check_error(stream)
        return reduce_max(t0.elapsed_time(t1) / n, device)
    nv = max(3, min(args.steps, 100))
    grid = {} if w.mode == "swa" else dict(F=w.F, Hh=w.Hh, Wh=w.Wh)
    variants = {
        "rope3d": time_plan(salad.ForwardPlan(
            dev["q"], dev["k"], dev["v"], dev["x"], dev["w_gate"], dev["w_lin"], mode=w.mode,
            topk=w.topk, bias=w.bias, eps=w.eps, rope3d=True, **extra, **grid), nv),
        "branch_dropped": time_plan(salad.ForwardPlan(
            dev["q"], dev["k"], dev["v"], dev["x"], dev["w_gate"], dev["w_lin"], mode=w.mode,
            topk=w.topk, bias=w.bias, eps=w.eps, drop_threshold=1.0, **extra), nv),
    }
    # Full-width projections: the linear branch's W_lin over all heads
    # (H*d x H*d) and the output projection W_out (H*d x H*d), two tcgen05
    # GEMMs after the attention.  The GEMM alone is timed too, against the
    # burst bf16 peak (it runs by itself here).
    proj = {n: t.to(device) for n, t in generate_projections(w).items()}
    variants["full_width_proj"] = time_plan(salad.ForwardPlan(
        dev["q"], dev["k"], dev["v"], dev["x"], dev["w_gate"], None, mode=w.mode,
        topk=w.topk, bias=w.bias, eps=w.eps, w_lin_full=proj["w_lin_full"],
        w_out=proj["w_out"], **extra), nv)
    K = w.H * w.d
    g_out = torch.empty_like(dev["q"])
    g_s = torch.full((w.B,), 0.5, dtype=torch.float32, device=device)
    for _ in range(3):
        salad.project(dev["q"], proj["w_lin_full"], out_per_head=True, resid=dev["v"], s=g_s,
                      out=g_out, stream=stream)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(nv):
        salad.project(dev["q"], proj["w_lin_full"], out_per_head=True, resid=dev["v"], s=g_s,
                      out=g_out, stream=stream)
    g1.record(stream)
    torch.cuda.synchronize(device)
    salad.check_error(stream)
    gemm_ms = g0.elapsed_time(g1) / nv
    gemm_flops = 2.0 * w.B * w.N * K * K
    del g_out

    # End to end through the public API: pinned host inputs -> device ->
    # salad_forward -> result back to the host, every step.
    names = ("q", "k", "v", "x", "w_gate", "w_lin")
    pinned = {n: host[n].pin_memory() for n in names}
    h2d = sum(pinned[n].numel() * pinned[n].element_size() for n in names)
    d2h = plan.o.numel() * plan.o.element_size()
    e2e_steps = max(3, min(args.steps, 50))

    def timed(run_steps) -> float:
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run_steps(e0)
        e1.record(stream)
        torch.cuda.synchronize(device)
        return reduce_max(e0.elapsed_time(e1), device)

    # (a) One stream, one step after the other: copy in, compute, copy out.
    out_host = torch.empty(plan.o.shape, dtype=plan.o.dtype).pin_memory()

    def serial(_t0=None, n_steps=e2e_steps):
        for _ in range(n_steps):
            for n in names:
                dev[n].copy_(pinned[n], non_blocking=True)
            plan.run(stream)
            out_host.copy_(plan.o, non_blocking=True)
    serial(n_steps=2)
    serial_ms = timed(serial)

    # (b) Pipelined, as a serving loop drives the library: two input sets and
    # two plans; step i's inputs cross PCIe on a copy stream while step i-1
    # computes, and step i-1's result returns on a third stream (PCIe is
    # full duplex).  Each step still copies all its inputs in and its output
    # back inside the timed region.
    sets = [dev, {n: torch.empty_like(dev[n]) for n in names}]
    plans = [plan, salad.ForwardPlan(sets[1]["q"], sets[1]["k"], sets[1]["v"], sets[1]["x"],
                                     sets[1]["w_gate"], sets[1]["w_lin"], mode=w.mode,
                                     topk=w.topk, bias=w.bias, eps=w.eps, **extra)]
    outs = [torch.empty(plan.o.shape, dtype=plan.o.dtype).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipelined(t0=None, n_steps=e2e_steps):
        if t0 is not None:
            s_in.wait_event(t0)
        for i in range(n_steps):
            k = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_run[k])      # plan k has read set k
                for n in names:
                    sets[k][n].copy_(pinned[n], non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_out[k])        # plan k's output has left
            plans[k].run(stream)
            ev_run[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_run[k])
                outs[k].copy_(plans[k].o, non_blocking=True)
                ev_out[k].record(s_out)
        for k in range(min(2, n_steps)):
            stream.wait_event(ev_out[k])
    pipelined(n_steps=2)
    pipe_ms = timed(pipelined)
    salad.check_error(stream)
    e2e = aggregate(world, fl["total"], e2e_steps, pipe_ms)
    e2e_serial = aggregate(world, fl["total"], e2e_steps, serial_ms)
    del sets, plans, outs

    peaks, peaks_src = load_peaks()
    peak, peak_kind = choose_peak(peaks, local_ms, clk)
    achieved = fl["attn_kernel"] / (attn_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": round(agg["value"], 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(agg["ms_per_step"], 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(w, world),
        "ms_per_layer": round(agg["ms_per_step"], 5),
        "phases_ms": {k: round(v, 5) for k, v in phases.items()},
        "dense_ms": round(dense_ms, 4), "speedup_vs_dense": round(dense_ms / agg["ms_per_step"], 3),
        "variants_ms_per_layer": {k: round(v, 5) for k, v in variants.items()},
        "proj_gemm": {"kernel": "proj_pair_kernel (cta_group::2, 256 x 256 pair tiles)", "shape": [w.B * w.N, K, K],
                      "ms": round(gemm_ms, 5),
                      "tflops": round(gemm_flops / (gemm_ms * 1e-3) / 1e12, 2),
                      "frac": round(gemm_flops / (gemm_ms * 1e-3) / 1e12 / float(peaks["bf16_tflops"]), 4),
                      "peak_source": f"bf16 burst, {peaks_src}"},
        "flops_per_step": fl["total"],
        "roofline": {"bound": "tensor", "kernel": "attn_kernel<128,hybrid>",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_kind}, {peaks_src} (timed region {local_ms:.1f} ms, "
                                    f"median SM clock {clk.get('sm_mhz')} of {clk.get('sm_max_mhz')} MHz)",
                     "frac_of_burst": round(achieved / float(peaks["bf16_tflops"]), 4),
                     "frac_of_sustained": round(
                         achieved / float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]), 4),
                     "traffic": committed_traffic(w.name),
                     "algorithmic_flops_per_launch": fl["attn_kernel"]},
        "e2e": {"value": round(e2e["value"], 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": round(e2e["ms_per_step"], 4),
                "mode": "pipelined: step i+1's inputs cross PCIe while step i computes",
                "serial": {"value": round(e2e_serial["value"], 3),
                           "ms_per_step": round(e2e_serial["ms_per_step"], 4)}},
        "gpu_launches": launches_per_step(w) * args.steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_sweep:
        # Timed after the headline line's numbers were taken.
        line["workloads"] = run_sweep([n for n in SWEEP if n.partition("+")[0] != w.name],
                                      device, stream, peaks)
        line["workloads_inputs"] = "device-drawn with the synthetic recipe (synth.generate_device)"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        del dev
        flops, secs = cpu_sample_work(w, host, n_heads=args.cpu_heads, blocks_per_head=args.cpu_blocks)
        line["cpu_baseline"] = {"value": round(flops / secs / 1e12, 6), "unit": UNIT,
                                "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"gate over all X; {args.cpu_heads} heads: selection, linear state, "
                                          f"{args.cpu_blocks} query blocks each (attention + "
                                          f"linear term); {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        barrier(device)
        dist.destroy_process_group()
    return 0


def run_reference(args, w) -> int:
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    from synth import generate
    host = generate(w)
    for _ in range(args.warmup):
        cpu_sample_work(w, host, n_heads=1, blocks_per_head=args.ref_blocks, seed=1000)
    t_flops, t_secs = 0.0, 0.0
    for i in range(args.steps):
        f, s = cpu_sample_work(w, host, n_heads=1, blocks_per_head=args.ref_blocks, seed=i)
        t_flops += f
        t_secs += s
    value = t_flops / t_secs / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t_secs * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cpu_threads(),
                         "kind": "oracle",
                         "sample": f"per step: gate over all X; 1 head: selection, linear "
                                   f"state, {args.ref_blocks} query blocks"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="topk480")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-heads", type=int, default=6, help="heads in the cpu_baseline sample")
    ap.add_argument("--cpu-blocks", type=int, default=488, help="query blocks per head in cpu_baseline")
    ap.add_argument("--ref-blocks", type=int, default=16, help="query blocks per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the other workloads (ST-SWA 480p, 720p, B=2 H=40 sparsity sweep)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    from synth import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
