#!/usr/bin/env python
"""Benchmark of the GLQ compressed-weight linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl glq|reference]

A step is one pass of the decode hot path (input RHT -> codebook GEMV ->
output RHT) over the five projections of the SmolLM3-3B-shaped workload
(q, o 2048x2048; gate, up 11008x2048; down 2048x11008; 4 bpw = uint16 E8
index + uint16 E8 residual, residual scale 1/8) for one token (B = 1), bf16
activations.  Indices are HBM-resident: 8 copies of the five layers rotate
(310 MB > the 126 MB L2).  Steps are CUDA-graph replays.

value = algorithmic bytes per step (index bytes + activations in/out +
bit-packed signs) / step time, in GB/s, summed over replicas.  Extra keys
report the per-layer times, the 24B-class decode sweep, prefill TFLOP/s, the
kernel roofline, the end-to-end number through host buffers, the fp64
oracle on the host cores and the SM clocks seen while timing.

Multi-GPU: the layer does not shard (one GPU per layer); --gpus N runs N
independent replicas under torchrun, one per rank (weak scaling, no
collective on the data path), and reports the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import glq_inputs as gi  # noqa: E402

METRIC = "glq_linear achieved HBM GB/s + µs/layer at B=1; prefill TFLOP/s; % roofline"
MAIN_WORKLOAD = "smollm3-3b-4bpw"
NCOPY = 8
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def layer_bytes(m: int, n: int, bpw: int, B: int, out_bytes: int = 2) -> int:
    """Algorithmic HBM bytes of one layer call: indices + x + y + signs."""
    return m * n * bpw // 8 + 2 * B * n + out_bytes * B * m + (m + 7) // 8 + (n + 7) // 8


def gemv_bytes(m: int, n: int, bpw: int, B: int) -> int:
    """Algorithmic bytes of the GEMV kernel alone: indices + fp16 xr + fp32 z."""
    return m * n * bpw // 8 + 2 * B * n + 4 * B * m


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get(
            "bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples (200 ms period) with wall times."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.samples = []
        self.proc = None
        self.thread = None
        self.gpu_index = gpu_index
        self.period_ms = period_ms

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", f"-lms={self.period_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._reader, daemon=True)
        self.thread.start()

    def _reader(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        inside = [p for (t, p) in self.samples if t0 <= t <= t1]
        note = "samples inside the timed region"
        if not inside:
            inside = [p for (t, p) in self.samples if t0 - 2.0 <= t <= t1 + 0.5]
            note = ("timed region shorter than the sampling period: samples from the identical "
                    "replays around it")
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "no samples"}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None

        sm = [num(p[1]) for p in inside if num(p[1]) is not None]
        smax = [num(p[2]) for p in inside if num(p[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in inside:
            for name, v in zip(names, p[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(inside), "note": note}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (the job time is the slowest rank's)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# the GLQ arm
# ---------------------------------------------------------------------------

class WorkloadSet:
    """ncopy device copies of the layers of a workload, with their x / y."""

    def __init__(self, glq, torch, key: str, B: int, ncopy: int, out_dtype=None):
        self.wl = gi.WORKLOADS[key]
        self.B = B
        self.torch = torch
        self.e8 = glq.Codebook.e8()
        xdt = torch.bfloat16 if self.wl.x_dtype == "bf16" else torch.float16
        self.out_dtype = out_dtype or xdt
        self.host = [gi.workload_layer(self.wl, i) for i in range(len(self.wl.layers))]
        self.xbits = [gi.workload_x(self.wl, i, B) for i in range(len(self.wl.layers))]
        self.copies = []
        for c in range(ncopy):
            layers = []
            for i, L in enumerate(self.host):
                res = None
                if L.bpw == 3:
                    res = glq.Codebook(L.cb2_f16.reshape(256, 8))
                elif L.bpw == 4:
                    res = self.e8
                lay = glq.GlqLinear(L.m, L.n, L.bpw, L.idx1, L.idx2, self.e8, res,
                                    L.weight_scale, L.resid_scale, L.s_in, L.s_out)
                lay.reserve(min(B, 16))
                x = torch.from_numpy(self.xbits[i].view(np.int16).copy()).cuda().view(xdt)
                y = torch.empty((B, L.m), dtype=self.out_dtype, device="cuda")
                layers.append((lay, x, y))
            self.copies.append(layers)

    def step(self, c: int, stream=None, B=None):
        B = self.B if B is None else B
        for lay, x, y in self.copies[c]:
            lay(x[:B], out=y[:B], stream=stream)

    def step_bytes(self, B=None) -> int:
        B = self.B if B is None else B
        ob = 4 if self.out_dtype == self.torch.float32 else 2
        return sum(layer_bytes(L.m, L.n, L.bpw, B, ob) for L in self.host)

    def step_flops(self, B=None) -> int:
        B = self.B if B is None else B
        return sum(2 * B * L.m * L.n for L in self.host)


def launches_per_step(ws: "WorkloadSet", B: int) -> int:
    """Kernels one decode step launches: per layer the GEMV, plus the input
    transform unless it is fused into the GEMV, plus the output transform
    (glq_decode_plan reports the plan the library takes)."""
    n = 0
    for lay, _, _ in ws.copies[0]:
        plan = lay.decode_plan(B)
        n += 2 + (0 if plan["fused_input"] else 1)
    return n


def capture_graphs(torch, fn_per_copy, ncopy):
    graphs = []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c in range(ncopy):  # warm the launch paths outside capture
            fn_per_copy(c)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for c in range(ncopy):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn_per_copy(c)
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs


def time_replays(torch, graphs, reps: int, warm: int = 3) -> float:
    """Mean ms per replay over `reps` replays rotating the graphs."""
    for i in range(warm):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        graphs[i % len(graphs)].replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def per_layer_times(torch, ws: WorkloadSet, reps: int, B=None, per_graph: int = 20):
    """Per layer: CUDA graphs of `per_graph` back-to-back glq_linear calls of
    that layer (rotating the weight copies), mean over the replays; and the
    eager latency of one call (events around it, median of 21)."""
    B = ws.B if B is None else B
    out = {}
    nc = len(ws.copies)
    for i, spec in enumerate(ws.wl.layers):
        def fn(c, i=i):
            for k in range(per_graph):
                lay, x, y = ws.copies[(c + k) % nc][i]
                lay(x[:B], out=y[:B])
        graphs = capture_graphs(torch, fn, nc)
        ms = time_replays(torch, graphs, max(1, reps // per_graph)) / per_graph
        del graphs
        eager = []
        for k in range(21):
            lay, x, y = ws.copies[k % nc][i]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            lay(x[:B], out=y[:B])
            e1.record()
            torch.cuda.synchronize()
            eager.append(e0.elapsed_time(e1))
        L = ws.host[i]
        b = layer_bytes(L.m, L.n, L.bpw, B, 2)
        out[f"{spec.name} {L.m}x{L.n}"] = {"us": round(ms * 1e3, 3), "GBps": round(b / (ms * 1e-3) / 1e9, 1),
                                           "eager_us": round(sorted(eager)[10] * 1e3, 2)}
    return out


def dense_reference_section(glq, torch, hbm_peak, tc_peak) -> dict:
    """Context, not the product: the same shapes as a dense bf16 linear on
    cuBLAS (torch.nn.functional.linear), W materialised by
    glq_dequant_reference (16 bits per weight instead of 2-4).  Decode: the
    3B-shaped layers at B = 1 (4 rotating copies, 600 MB, above L2); prefill:
    the 8B MLP shapes at 8192 tokens, GEMM alone and dequantise + GEMM."""
    import torch.nn.functional as F
    res = {"decode_b1": {}, "prefill_b8192": {}}
    ws = WorkloadSet(glq, torch, MAIN_WORKLOAD, 1, 1)
    for i, spec in enumerate(ws.wl.layers):
        lay, x, _ = ws.copies[0][i]
        L = ws.host[i]
        Ws = [lay.dequant().to(torch.bfloat16) for _ in range(4)]
        xs = x[:1].to(torch.bfloat16)
        def fn(c):
            for k in range(20):
                F.linear(xs, Ws[(c + k) % 4])
        graphs = capture_graphs(torch, fn, 4)
        ms = time_replays(torch, graphs, 10) / 20
        del graphs
        b = 2 * L.m * L.n + 2 * L.n + 2 * L.m
        res["decode_b1"][f"{spec.name} {L.m}x{L.n}"] = {
            "us": round(ms * 1e3, 2), "GBps": round(b / (ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(b / (ms * 1e-3) / 1e9 / hbm_peak, 3)}
        del Ws
    del ws
    torch.cuda.empty_cache()
    wp = WorkloadSet(glq, torch, "prefill-8b-mlp-4bpw", 8192, 1)
    for i, (lay, x, _) in enumerate(wp.copies[0]):
        L = wp.host[i]
        W = lay.dequant().to(torch.bfloat16)
        xb = x.to(torch.bfloat16)
        F.linear(xb, W)
        torch.cuda.synchronize()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        for _ in range(5):
            F.linear(xb, W)
        e1.record()
        for _ in range(5):
            F.linear(xb, lay.dequant().to(torch.bfloat16))
        e2.record()
        torch.cuda.synchronize()
        g_ms, dg_ms = e0.elapsed_time(e1) / 5, e1.elapsed_time(e2) / 5
        fl = 2.0 * 8192 * L.m * L.n
        res["prefill_b8192"][f"{L.m}x{L.n}"] = {
            "gemm_us": round(g_ms * 1e3, 1), "gemm_TFLOPs": round(fl / (g_ms * 1e-3) / 1e12, 1),
            "dequant_gemm_us": round(dg_ms * 1e3, 1),
            "dequant_gemm_TFLOPs": round(fl / (dg_ms * 1e-3) / 1e12, 1)}
        del W
    del wp
    torch.cuda.empty_cache()
    res["note"] = "cuBLAS bf16 via torch; W materialised at 16 bits per weight; not the product path"
    return res


def gemv_kernel_time(torch, ws: WorkloadSet, layer_index: int, reps: int, B=None) -> float:
    """Mean ms of the GEMV kernel alone: CUDA graphs of 20 back-to-back
    launches (no host launch cost between them), rotating the weight copies,
    timed with events on the stream the kernels run on."""
    B = min(ws.B if B is None else B, 16)
    for c in range(len(ws.copies)):
        lay, x, y = ws.copies[c][layer_index]
        lay(x[:B], out=y[:B])
    torch.cuda.synchronize()
    per_graph = 20

    def fn(c):
        for i in range(per_graph):
            ws.copies[(c + i) % len(ws.copies)][layer_index][0].gemv_replay(B)

    graphs = capture_graphs(torch, fn, len(ws.copies))
    n = max(1, reps // per_graph)
    ms = time_replays(torch, graphs, n)
    del graphs
    return ms / per_graph


def profiled_traffic(profile: str, source: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    recorded in a committed ncu summary under profiles/, or None when the
    kernel source has changed since that capture (its sha256 differs)."""
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    try:
        text = open(os.path.join(root, "profiles", profile)).read()
        src = open(os.path.join(root, "e8_lattice_codebook_b200", "csrc", source), "rb").read()
    except OSError:
        return None
    if hashlib.sha256(src).hexdigest() not in text:
        return None
    for line in text.splitlines():
        if line.startswith("traffic_bytes_per_launch"):
            return int(line.split(":")[1].split()[0])
    return None


def prefill_section(glq, torch, tc_peak, peak_src, batches=(512, 2048, 8192), reps=5) -> dict:
    """8B-class MLP prefill (14336x4096 and 4096x14336 at 4 bpw): the whole
    glq_linear step (input RHT, tensor-core GEMM, output RHT) per batch, and
    the GEMM kernel alone (glq_prefill_replay) per layer, timed with events
    on the stream the kernels run on.  The inputs (x 8192 x 14336 bf16 is
    235 MB) exceed L2."""
    pre = {}
    wp = WorkloadSet(glq, torch, "prefill-8b-mlp-4bpw", max(batches), 1)
    for Bp in batches:
        wp.step(0, B=Bp)
        torch.cuda.synchronize()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        for _ in range(reps):
            wp.step(0, B=Bp)
        p1.record()
        torch.cuda.synchronize()
        msp = p0.elapsed_time(p1) / reps
        tf = wp.step_flops(Bp) / (msp * 1e-3) / 1e12
        entry = {"ms_per_step": round(msp, 3), "TFLOPs": round(tf, 2),
                 "frac_bf16_peak": round(tf / tc_peak, 4)}
        gemm = {}
        for li, (lay, x, y) in enumerate(wp.copies[0]):
            L = wp.host[li]
            lay(x[:Bp], out=y[:Bp])  # leaves this batch's activations in the workspace
            torch.cuda.synchronize()
            lay.prefill_replay(Bp)
            k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            k0.record()
            for _ in range(reps):
                lay.prefill_replay(Bp)
            k1.record()
            torch.cuda.synchronize()
            mk = k0.elapsed_time(k1) / reps
            tk = 2.0 * Bp * L.m * L.n / (mk * 1e-3) / 1e12
            gemm[f"{L.m}x{L.n}"] = {"kernel_us": round(mk * 1e3, 1), "TFLOPs": round(tk, 1),
                                    "frac": round(tk / tc_peak, 4)}
        entry["gemm_kernel"] = gemm
        pre[f"B={Bp}"] = entry
    pre["peak"] = {"TFLOPs": tc_peak, "source": peak_src,
                   "note": "fp16 operands: measured cuBLAS bf16 peak (same nominal rate)"}
    del wp
    torch.cuda.empty_cache()
    return pre


def decode24_section(glq, torch, hbm_peak, batches=(1, 2, 4, 8, 16), reps=100) -> dict:
    """24B-class decode (q 4096x5120, o 5120x4096, gate/up 32768x5120, down
    5120x32768 at 4 bpw, bf16): per batch the five-layer step as CUDA-graph
    replays over two weight copies (544 MB > L2); at B = 1 also the per-layer
    times and the GEMV kernel alone on the gate layer."""
    sweep = {}
    w24 = WorkloadSet(glq, torch, "24b-decode-4bpw", max(batches), 2)
    for Bd in batches:
        g24 = capture_graphs(torch, lambda c, Bd=Bd: w24.step(c, B=Bd), 2)
        ms24 = time_replays(torch, g24, reps=reps)
        b24 = w24.step_bytes(Bd)
        entry = {"ms_per_step": round(ms24, 4), "GBps": round(b24 / (ms24 * 1e-3) / 1e9, 1),
                 "frac_hbm": round(b24 / (ms24 * 1e-3) / 1e9 / hbm_peak, 4)}
        if Bd == 1:
            entry["layers_us"] = per_layer_times(torch, w24, reps=reps, B=1)
            mk = gemv_kernel_time(torch, w24, 2, reps=reps, B=1)
            Lg = w24.host[2]
            ach = gemv_bytes(Lg.m, Lg.n, Lg.bpw, 1) / (mk * 1e-3) / 1e9
            entry["gemv_gate_us"] = round(mk * 1e3, 3)
            entry["gemv_gate_frac_hbm"] = round(ach / hbm_peak, 4)
        sweep[f"B={Bd}"] = entry
        del g24
    del w24
    torch.cuda.empty_cache()
    return sweep


def oracle_step_seconds(ws_host, xbits, bpw, x_bf16) -> float:
    from oracle import glq_oracle as orc
    t0 = time.perf_counter()
    for L, xb in zip(ws_host, xbits):
        orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in,
                   L.s_out, xb[:1], x_bf16, cb2=L.cb2_f16)
    return time.perf_counter() - t0


def run_glq(args):
    import torch
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import e8_lattice_codebook_b200 as glq

    hbm_peak, tc_peak, tc_peak_sus, peak_src = read_peaks()
    B = 1
    ws = WorkloadSet(glq, torch, MAIN_WORKLOAD, B, NCOPY)
    graphs = capture_graphs(torch, ws.step, NCOPY)
    bytes_step = ws.step_bytes()

    # clocks: the sampler runs through warm-up and the timed steps
    sampler = ClockSampler(local)
    sampler.start()
    soak_end = time.time() + 1.0
    i = 0
    while time.time() < soak_end:  # ~1 s of identical replays for the clock sampler
        graphs[i % NCOPY].replay()
        i += 1
        if i % 256 == 0:
            torch.cuda.synchronize()
    for i in range(args.warmup):
        graphs[i % NCOPY].replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    torch.cuda.nvtx.range_push("timed")
    e0.record()
    for i in range(args.steps):
        graphs[i % NCOPY].replay()
    e1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    time.sleep(0.25)
    sampler.stop()
    ms_total = e0.elapsed_time(e1)
    ms_total = max_over_ranks(ms_total, world, device=torch.device("cuda", local))
    ms_step = ms_total / args.steps
    value = world * bytes_step / (ms_step * 1e-3) / 1e9
    clocks = sampler.summary(t_wall0, t_wall1)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 MMA operands, fp32 accumulate (bf16 activations in/out)",
        "data": "synthetic (seeded uniform indices, Rademacher signs, N(0,1) activations)",
        "config": {
            "workload": ("smollm3-3b-4bpw decode: q,o 2048x2048, gate,up 11008x2048, "
                         "down 2048x11008 @ 4 bpw (u16 E8 + u16 E8 residual, rs 1/8), B=1, bf16"),
            "global_batch": B * world, "parallelism": f"replicas x{world}",
            "l2": f"{NCOPY} rotating copies of the layer set "
                  f"({NCOPY * sum(L.m * L.n // 2 for L in ws.host) / 1e6:.0f} MB > 126 MB L2)",
            "timing": "CUDA-graph replay, CUDA events, max over ranks",
        },
        "gpu_launches": launches_per_step(ws, B) * args.steps,
        "clocks": clocks,
    }
    if rank != 0:
        return None

    # ---- extra measurements (rank 0) -------------------------------------
    result["layers_us"] = per_layer_times(torch, ws, reps=400)

    # roofline of the GEMV (the largest layer of the step: gate 11008x2048)
    li = 2
    L = ws.host[li]
    ms_k = gemv_kernel_time(torch, ws, li, reps=400)
    achieved = gemv_bytes(L.m, L.n, L.bpw, B) / (ms_k * 1e-3) / 1e9
    result["roofline"] = {
        "kernel": f"gemv_kernel<4,1> gate {L.m}x{L.n} B=1",
        "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
        "frac": round(achieved / hbm_peak, 4), "peak_source": f"{peak_src} hbm_gbs (burst)",
        "traffic": profiled_traffic("gemv_smollm3-3b-gate-up-down_4bpw_b1.md", "glq_gemv.cu"),
        "kernel_us": round(ms_k * 1e3, 3),
        "algorithmic_bytes": gemv_bytes(L.m, L.n, L.bpw, B),
    }

    # e2e through the public API with host buffers: per step, the step's
    # inputs (the five layers' x, contiguous in pinned host memory) go to the
    # device in one copy and its result (the five y) comes back in one copy
    xdt = torch.bfloat16
    xs_host = np.concatenate([xb.view(np.int16).reshape(-1) for xb in ws.xbits])
    hx = torch.from_numpy(xs_host.copy()).view(xdt).pin_memory()
    dx = torch.empty_like(hx, device="cuda")
    ysz = [B * Lh.m for Lh in ws.host]
    hy = torch.empty(sum(ysz), dtype=xdt).pin_memory()
    dy = torch.empty(sum(ysz), dtype=xdt, device="cuda")
    xoff = np.cumsum([0] + [xb.size for xb in ws.xbits]).tolist()
    yoff = np.cumsum([0] + ysz).tolist()
    xv = [dx[xoff[i]:xoff[i + 1]].view(B, ws.host[i].n) for i in range(len(ws.host))]
    yv = [dy[yoff[i]:yoff[i + 1]].view(B, ws.host[i].m) for i in range(len(ws.host))]
    h2d = hx.numel() * 2
    d2h = hy.numel() * 2

    def e2e_step(c):
        dx.copy_(hx, non_blocking=True)
        for (lay, _, _), x, y in zip(ws.copies[c], xv, yv):
            lay(x, out=y)
        hy.copy_(dy, non_blocking=True)

    for c in range(NCOPY):
        e2e_step(c)
    torch.cuda.synchronize()
    reps = max(50, min(args.steps, 2000))
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for i in range(reps):
        e2e_step(i % NCOPY)
    f1.record()
    torch.cuda.synchronize()
    ms_eager = f0.elapsed_time(f1) / reps
    # the same step captured once per weight copy in a CUDA graph (the
    # deployment form of a decode step: glq_linear is capturable), replayed:
    # every replay still copies x from pinned host memory and y back to it
    e2e_graphs = capture_graphs(torch, e2e_step, NCOPY)
    ms_e2e = time_replays(torch, e2e_graphs, reps)
    del e2e_graphs
    result["e2e"] = {"value": round(bytes_step / (ms_e2e * 1e-3) / 1e9, 2), "unit": "GB/s",
                     "ms_per_step": round(ms_e2e, 6), "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h,
                     "how": ("one pinned H2D copy of the step's x, glq_linear per layer, one D2H copy "
                             "of the step's y; the step captured in a CUDA graph and replayed, events"),
                     "eager": {"value": round(bytes_step / (ms_eager * 1e-3) / 1e9, 2),
                               "ms_per_step": round(ms_eager, 6),
                               "how": "the same calls issued eagerly from Python"}}

    # 24B-class decode sweep
    if not args.quick:
        result["decode_24b"] = decode24_section(glq, torch, hbm_peak)

        result["prefill"] = prefill_section(glq, torch, tc_peak, peak_src)
        result["dense_bf16_reference"] = dense_reference_section(glq, torch, hbm_peak, tc_peak)

    # fp64 oracle on the host cores (one decode step, 1 token, 5 layers)
    if world == 1 and not args.no_cpu:
        secs = oracle_step_seconds(ws.host, ws.xbits, 4, True)
        result["cpu_baseline"] = {
            "value": round(bytes_step / secs / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "seconds": round(secs, 3),
            "sample": "one full step: 1 token through q,o,gate,up,down (fp64, single thread)"}
    return result


# ---------------------------------------------------------------------------
# the reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    world, rank, local = dist_setup()
    if world > 1 and rank != 0:
        return None
    wl = gi.WORKLOADS[MAIN_WORKLOAD]
    host = [gi.workload_layer(wl, i) for i in range(len(wl.layers))]
    xbits = [gi.workload_x(wl, i, 1) for i in range(len(wl.layers))]
    bytes_step = sum(layer_bytes(L.m, L.n, L.bpw, 1, 2) for L in host)
    for _ in range(args.warmup if args.warmup <= 1 else 1):
        oracle_step_seconds(host, xbits, 4, True)
    budget = 150.0
    t_step = None
    times = []
    t_start = time.perf_counter()
    for i in range(args.steps):
        times.append(oracle_step_seconds(host, xbits, 4, True))
        if time.perf_counter() - t_start > budget:
            break
    t_step = sum(times) / len(times)
    value = bytes_step / t_step / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": len(times), "warmup": args.warmup,
        "ms_per_step": round(t_step * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": ("smollm3-3b-4bpw decode: q,o 2048x2048, gate,up 11008x2048, "
                                "down 2048x11008 @ 4 bpw, B=1, bf16"),
                   "global_batch": 1, "parallelism": "single host thread"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{len(times)} full steps (1 token, 5 layers) of the fp64 oracle"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_prefill_only(args):
    """The prefill timings alone, one JSON object (not the bench line)."""
    import torch
    import e8_lattice_codebook_b200 as glq
    torch.cuda.set_device(0)
    _, tc_peak, _, peak_src = read_peaks()
    batches = (args.prefill_batch,) if args.prefill_batch else (512, 2048, 8192)
    return {"section": "prefill", "prefill": prefill_section(glq, torch, tc_peak, peak_src, batches,
                                                            reps=max(1, min(args.steps, 20)))}


def run_decode24_only(args):
    """The 24B-class decode timings alone, one JSON object (not the bench line)."""
    import torch
    import e8_lattice_codebook_b200 as glq
    torch.cuda.set_device(0)
    hbm_peak = read_peaks()[0]
    batches = (args.decode_batch,) if args.decode_batch else (1, 2, 4, 8, 16)
    return {"section": "decode24", "decode_24b": decode24_section(glq, torch, hbm_peak, batches,
                                                                  reps=max(20, min(args.steps, 400)))}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["glq", "reference"], default="glq")
    ap.add_argument("--quick", action="store_true", help="skip the 24B sweep and prefill")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle baseline")
    ap.add_argument("--section", choices=["all", "prefill", "decode24"], default="all",
                    help="prefill / decode24: time only that workload (profiling runs)")
    ap.add_argument("--prefill-batch", type=int, default=0,
                    help="with --section prefill: one batch instead of 512, 2048, 8192")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="with --section decode24: one batch instead of 1, 2, 4, 8, 16")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.section == "prefill":
        res = run_prefill_only(args)
    elif args.section == "decode24":
        res = run_decode24_only(args)
    else:
        res = run_reference(args) if args.impl == "reference" else run_glq(args)
    if res is not None:
        print(json.dumps(res), flush=True)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and args.impl == "glq":
        import torch.distributed as dist
        if dist.is_initialized():
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
