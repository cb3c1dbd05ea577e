#!/usr/bin/env python
"""Benchmark of the GLQ compressed-weight linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl glq|reference]

A step is one pass of the decode hot path (input RHT -> codebook GEMV ->
output RHT) over the five projections of the 24B-class workload (q
4096x5120, o 5120x4096, gate / up 32768x5120, down 5120x32768; 4 bpw =
uint16 E8 index + uint16 E8 residual, residual scale 1/8) for one token
(B = 1), bf16 activations.  Indices are HBM-resident: enough copies of each
layer rotate that every layer's copies exceed twice the 126 MB L2.  Steps are
CUDA-graph replays.

value = algorithmic bytes per step (index bytes + activations in/out +
bit-packed signs) / step time, in GB/s, summed over replicas.  Extra keys
report every decode configuration at every batch it names (per-layer
us, GB/s and fraction of the measured HBM bandwidth), prefill TFLOP/s, the
GEMV kernel's roofline, the end-to-end number through host buffers, the
fp64 oracle on the host cores and the SM clocks seen while timing.

Multi-GPU: one layer runs on one GPU; --gpus N runs N independent replicas
under torchrun, one per rank (weak scaling, no collective on the data path),
and reports the max-over-ranks time.
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
MAIN_WORKLOAD = "24b-decode-4bpw"
L2_BYTES = 126 * 1024 * 1024
DECODE_DTYPE = ("u8 x s8/u8 integer MMA on int16-quantised rotated activations (exact int32 sums, "
                "fp64 across K splits); bf16 activations in and out")
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the
# GEMV on the 24B-class gate layer at one token, from the ncu capture whose
# summary is profiles/gemv_24b-gate-32768x5120_4bpw_b1.md, keyed by the
# sha256 of the GEMV source it was taken at: a changed kernel reports null.
PROFILED_GEMV_TRAFFIC = {
    "8ba979ed5d9f9b06b4f37ef8298de07a9693d969ba3a03536565df023ef772d1": 84113664 + 3624960,
}
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

def copies_for(index_bytes: int, cap: int = 1024) -> int:
    """Copies of a layer whose indices together exceed twice the L2."""
    return max(2, min(cap, -(-2 * L2_BYTES // max(1, index_bytes))))


class WorkloadSet:
    """Device copies of the layers of a workload, with their x / y.  Layer i
    has ncopy_i copies, enough that they exceed twice the L2 (so a rotation
    over them reads the indices from HBM); step copy c uses copy c mod
    ncopy_i of every layer."""

    def __init__(self, glq, torch, key: str, B: int, ncopy=None, out_dtype=None, max_copies: int = 1024):
        self.wl = gi.WORKLOADS[key]
        self.B = B
        self.torch = torch
        self.e8 = glq.Codebook.e8()
        xdt = torch.bfloat16 if self.wl.x_dtype == "bf16" else torch.float16
        self.xdt = xdt
        self.out_dtype = out_dtype or xdt
        self.host = [gi.workload_layer(self.wl, i) for i in range(len(self.wl.layers))]
        self.xbits = [gi.workload_x(self.wl, i, B) for i in range(len(self.wl.layers))]
        self.ncopies = [ncopy or copies_for(L.m * L.n * L.bpw // 8, max_copies) for L in self.host]
        self.layers = []  # [layer][copy] = (GlqLinear, x, y)
        for i, L in enumerate(self.host):
            res = None
            if L.bpw % 2:
                res = glq.Codebook(L.cb2_f16.reshape(256, 8))
            elif L.bpw == 4:
                res = self.e8
            x = torch.from_numpy(self.xbits[i].view(np.int16).copy()).cuda().view(xdt)
            row = []
            for c in range(self.ncopies[i]):
                lay = glq.GlqLinear(L.m, L.n, L.bpw, L.idx1, L.idx2, self.e8, res,
                                    L.weight_scale, L.resid_scale, L.s_in, L.s_out)
                lay.reserve(min(B, 16))
                y = torch.empty((B, L.m), dtype=self.out_dtype, device="cuda")
                row.append((lay, x, y))
            self.layers.append(row)
        self.ncopy = max(self.ncopies)

    def copy(self, c: int):
        return [row[c % len(row)] for row in self.layers]

    def step(self, c: int, stream=None, B=None):
        B = self.B if B is None else B
        for lay, x, y in self.copy(c):
            lay(x[:B], out=y[:B], stream=stream)

    def step_bytes(self, B=None) -> int:
        B = self.B if B is None else B
        ob = 4 if self.out_dtype == self.torch.float32 else 2
        return sum(layer_bytes(L.m, L.n, L.bpw, B, ob) for L in self.host)

    def step_flops(self, B=None) -> int:
        B = self.B if B is None else B
        return sum(2 * B * L.m * L.n for L in self.host)

    def index_bytes(self) -> int:
        return sum(n * L.m * L.n * L.bpw // 8 for n, L in zip(self.ncopies, self.host))


def launches_per_step(ws: "WorkloadSet", B: int) -> int:
    """Kernels one decode step launches: per layer the GEMV, plus the input
    transform unless it is fused into the GEMV, plus the output transform
    (glq_decode_plan reports the plan the library takes)."""
    n = 0
    for lay, _, _ in ws.copy(0):
        plan = lay.decode_plan(min(B, 16))
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
    """Mean ms per replay over max(reps, len(graphs)) replays rotating the
    graphs, starting after the warm-up ones (so every timed replay meets
    weight copies that were last touched a full rotation earlier)."""
    n = len(graphs)
    for i in range(warm):
        graphs[i % n].replay()
    torch.cuda.synchronize()
    reps = max(reps, n)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        graphs[(warm + i) % n].replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def per_layer_times(torch, ws: WorkloadSet, reps: int, hbm_peak: float, B=None, per_graph: int = 20):
    """Per layer: CUDA graphs of `per_graph` back-to-back glq_linear calls of
    that layer (rotating its copies, which exceed twice the L2), mean over
    the replays; and the eager latency of one call (events around it,
    median of 21)."""
    B = ws.B if B is None else B
    out = {}
    total_us = 0.0
    for i, spec in enumerate(ws.wl.layers):
        row = ws.layers[i]
        nc = len(row)

        def fn(c, row=row, nc=nc):
            for k in range(per_graph):
                lay, x, y = row[(c * per_graph + k) % nc]
                lay(x[:B], out=y[:B])
        ngraph = -(-nc // per_graph)  # every copy once per round of graphs
        graphs = capture_graphs(torch, fn, ngraph)
        ms = time_replays(torch, graphs, max(1, reps // per_graph)) / per_graph
        del graphs
        eager = []
        for k in range(21):
            lay, x, y = row[k % nc]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            lay(x[:B], out=y[:B])
            e1.record()
            torch.cuda.synchronize()
            eager.append(e0.elapsed_time(e1))
        L = ws.host[i]
        b = layer_bytes(L.m, L.n, L.bpw, B, 2)
        gbs = b / (ms * 1e-3) / 1e9
        total_us += ms * 1e3
        out[f"{spec.name} {L.m}x{L.n}"] = {"us": round(ms * 1e3, 3), "GBps": round(gbs, 1),
                                           "frac_hbm": round(gbs / hbm_peak, 4),
                                           "eager_us": round(sorted(eager)[10] * 1e3, 2),
                                           "copies": nc}
    out["sum_us"] = round(total_us, 3)
    return out


def decode_config_section(glq, torch, key: str, hbm_peak: float, batches=None, reps: int = 200,
                          gemv_layer=None) -> dict:
    """One decode configuration at every batch it names: the whole step
    (its layers back to back) as CUDA-graph replays rotating the copies, and
    the per-layer times; optionally the GEMV kernel alone on one layer."""
    wl = gi.WORKLOADS[key]
    batches = batches or wl.batches
    res = {}
    ws = WorkloadSet(glq, torch, key, max(batches))
    for Bd in batches:
        graphs = capture_graphs(torch, lambda c, Bd=Bd: ws.step(c, B=Bd), ws.ncopy)
        ms = time_replays(torch, graphs, reps=reps)
        del graphs
        b = ws.step_bytes(Bd)
        entry = {"ms_per_step": round(ms, 5), "GBps": round(b / (ms * 1e-3) / 1e9, 1),
                 "frac_hbm": round(b / (ms * 1e-3) / 1e9 / hbm_peak, 4),
                 "layers_us": per_layer_times(torch, ws, reps=reps, hbm_peak=hbm_peak, B=Bd)}
        if gemv_layer is not None and Bd == batches[0]:
            mk = gemv_kernel_time(torch, ws, gemv_layer, reps=reps, B=Bd)
            Lg = ws.host[gemv_layer]
            ach = gemv_bytes(Lg.m, Lg.n, Lg.bpw, Bd) / (mk * 1e-3) / 1e9
            entry["gemv_alone"] = {"layer": f"{wl.layers[gemv_layer].name} {Lg.m}x{Lg.n}",
                                   "us": round(mk * 1e3, 3), "GBps": round(ach, 1),
                                   "frac_hbm": round(ach / hbm_peak, 4)}
        res[f"B={Bd}"] = entry
    res["workload"] = wl.description
    res["index_bytes_on_device"] = ws.index_bytes()
    del ws
    torch.cuda.empty_cache()
    return res


def dense_reference_section(glq, torch, hbm_peak, tc_peak) -> dict:
    """Context, not the product: the same shapes as a dense bf16 linear on
    cuBLAS (torch.nn.functional.linear), W materialised by
    glq_dequant_reference (16 bits per weight instead of 2-4).  Decode: the
    24B-class layers at B = 1 (two rotating copies, 2.2 GB, above L2);
    prefill: the 8B MLP shapes at 8192 tokens, GEMM alone and dequantise +
    GEMM."""
    import torch.nn.functional as F
    res = {"decode_b1": {}, "prefill_b8192": {}}
    ws = WorkloadSet(glq, torch, MAIN_WORKLOAD, 1, ncopy=1)
    total = 0.0
    for i, spec in enumerate(ws.wl.layers):
        lay, x, _ = ws.layers[i][0]
        L = ws.host[i]
        Ws = [lay.dequant().to(torch.bfloat16) for _ in range(2)]
        xs = x[:1].to(torch.bfloat16)

        def fn(c):
            for k in range(20):
                F.linear(xs, Ws[(c + k) % 2])
        graphs = capture_graphs(torch, fn, 2)
        ms = time_replays(torch, graphs, 10) / 20
        del graphs
        b = 2 * L.m * L.n + 2 * L.n + 2 * L.m
        total += ms * 1e3
        res["decode_b1"][f"{spec.name} {L.m}x{L.n}"] = {
            "us": round(ms * 1e3, 2), "GBps": round(b / (ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(b / (ms * 1e-3) / 1e9 / hbm_peak, 3)}
        del Ws
    res["decode_b1"]["sum_us"] = round(total, 2)
    del ws
    torch.cuda.empty_cache()
    wp = WorkloadSet(glq, torch, "prefill-8b-mlp-4bpw", 8192, ncopy=1)
    for i in range(len(wp.host)):
        lay, x, _ = wp.layers[i][0]
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
    launches (no host launch cost between them), rotating the layer's
    copies, timed with events on the stream the kernels run on."""
    B = min(ws.B if B is None else B, 16)
    row = ws.layers[layer_index]
    for lay, x, y in row:
        lay(x[:B], out=y[:B])
    torch.cuda.synchronize()
    per_graph = 20

    def fn(c):
        for i in range(per_graph):
            row[(c * per_graph + i) % len(row)][0].gemv_replay(B)

    graphs = capture_graphs(torch, fn, -(-len(row) // per_graph))
    n = max(1, reps // per_graph)
    ms = time_replays(torch, graphs, n)
    del graphs
    return ms / per_graph


def gemv_source_sha256() -> str:
    import hashlib
    path = os.path.join(ROOT, "e8_lattice_codebook_b200", "csrc", "glq_gemv.cu")
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def prefill_section(glq, torch, tc_peak, peak_src, batches=(512, 2048, 8192), reps=5, hbm_peak=None) -> dict:
    """8B-class MLP prefill (14336x4096 and 4096x14336 at 4 bpw): the whole
    glq_linear step (input RHT, tensor-core GEMM, output RHT) per batch, and
    the GEMM kernel alone (glq_prefill_replay) per layer, and the input
    transform alone with either kernel, timed with events on the stream the
    kernels run on.  The inputs (x 8192 x 14336 bf16 is 235 MB) exceed L2."""
    pre = {}
    wp = WorkloadSet(glq, torch, "prefill-8b-mlp-4bpw", max(batches), ncopy=1)
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
        for li in range(len(wp.host)):
            lay, x, y = wp.layers[li][0]
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
        if hbm_peak:
            entry["input_transform"] = input_transform_times(glq, torch, wp, Bp, hbm_peak, reps=reps)
        pre[f"B={Bp}"] = entry
    pre["peak"] = {"TFLOPs": tc_peak, "source": peak_src,
                   "note": "fp16 operands: measured cuBLAS bf16 peak (same nominal rate)"}
    del wp
    torch.cuda.empty_cache()
    return pre


def input_transform_times(glq, torch, wp, Bp: int, hbm_peak: float, reps: int = 5) -> dict:
    """The input transform of each prefill layer alone (glq_rht_input_operand),
    the CUDA-core butterfly kernel (1) against the warp tensor-core kernel (2),
    on row windows of the layer's activations that rotate through more than
    L2 (the largest batch's rows).  Per layer, longest rows first: three
    warm-up pairs (butterfly, tensor core) launched eagerly, then per kernel
    a CUDA graph of `reps` launches, replayed three times between events.
    Algorithmic bytes: B n (2 B in + 2 B out)."""
    out = {}
    for li in sorted(range(len(wp.host)), key=lambda i: -wp.host[i].n):
        lay, x, _ = wp.layers[li][0]
        L = wp.host[li]
        nwin = max(1, x.shape[0] // Bp)
        n_pad = (L.n + 127) // 128 * 128
        xh = torch.empty((nwin * Bp, n_pad), dtype=torch.float16, device="cuda")
        info = torch.empty((nwin * Bp, 4), dtype=torch.float32, device="cuda")

        def launch(kern, w, stream):
            glq.glq_rht_input_operand(lay.handle, x[w * Bp].data_ptr(), glq.dtype_code(x.dtype),
                                      xh[w * Bp].data_ptr(), info[w * Bp].data_ptr(), Bp, kern,
                                      stream.cuda_stream)
        cur = torch.cuda.current_stream()
        for w in range(3):
            launch(1, w % nwin, cur)
            launch(2, w % nwin, cur)
        torch.cuda.synchronize()
        alg = Bp * L.n * 4
        entry = {"algorithmic_bytes": alg, "hbm_us": round(alg / (hbm_peak * 1e9) * 1e6, 2)}
        for kern, name in ((1, "butterfly"), (2, "tensor_core")):
            g = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    for r in range(reps):
                        launch(kern, r % nwin, s)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(3):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / (3 * reps)
            gbs = alg / (us * 1e-6) / 1e9
            entry[name] = {"us": round(us, 2), "GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4)}
            del g
        out[f"n={L.n}"] = entry
        del xh, info
    return out


def oracle_step_seconds(ws_host, xbits, x_bf16, threads: int = 1) -> float:
    """Seconds of the fp64 oracle for one decode step (the first token of
    every layer); threads: rows of each layer split over that many threads."""
    from oracle import glq_oracle as orc
    t0 = time.perf_counter()
    for L, xb in zip(ws_host, xbits):
        orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in,
                   L.s_out, xb[:1], x_bf16, cb2=L.cb2_f16, threads=threads)
    return time.perf_counter() - t0


def oracle_prefill_sample(threads: int, tokens: int = 64) -> dict:
    """The fp64 oracle on a seeded sample of `tokens` token rows of the 8B MLP
    prefill workload (both layers, all outputs): per-token seconds and the
    TFLOP/s that extrapolates to each batch (labelled extrapolated)."""
    from oracle import glq_oracle as orc
    wl = gi.WORKLOADS["prefill-8b-mlp-4bpw"]
    secs = 0.0
    flops_tok = 0
    for li in range(len(wl.layers)):
        L = gi.workload_layer(wl, li)
        xb = gi.workload_x(wl, li, max(wl.batches))
        rng = np.random.default_rng(7 + li)
        rows = np.sort(rng.choice(xb.shape[0], size=tokens, replace=False))
        t0 = time.perf_counter()
        orc.linear(L.m, L.n, L.bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out,
                   xb[rows], True, threads=threads)
        secs += time.perf_counter() - t0
        flops_tok += 2 * L.m * L.n
    per_tok = secs / tokens
    return {"tokens": tokens, "threads": threads, "seconds": round(secs, 3),
            "per_token_s": round(per_tok, 5),
            "TFLOPs_extrapolated": {f"B={B}": round(flops_tok * B / (per_tok * B) / 1e12, 6)
                                    for B in wl.batches},
            "label": "extrapolated: per-token time of the sample x B (the layer is linear in the tokens)"}


def bench_config(world: int) -> dict:
    """The `config` object both arms print (identical by construction)."""
    return {"workload": ("24b-decode-4bpw: q 4096x5120, o 5120x4096, gate/up 32768x5120, "
                         "down 5120x32768 @ 4 bpw (u16 E8 + u16 E8 residual, rs 1/8), B=1, bf16 x/y; "
                         "synthetic seeded inputs"),
            "global_batch": world, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2: every layer's rotating copies exceed 2 x 126 MB"}


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
    ws = WorkloadSet(glq, torch, MAIN_WORKLOAD, B)
    NG = ws.ncopy
    graphs = capture_graphs(torch, ws.step, NG)
    bytes_step = ws.step_bytes()

    # clocks: the sampler runs through warm-up and the timed steps
    sampler = ClockSampler(local)
    sampler.start()
    soak_end = time.time() + 1.0
    i = 0
    while time.time() < soak_end:  # ~1 s of identical replays for the clock sampler
        graphs[i % NG].replay()
        i += 1
        if i % 256 == 0:
            torch.cuda.synchronize()
    for i in range(args.warmup):
        graphs[i % NG].replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record()
    for i in range(args.steps):
        graphs[i % NG].replay()
    e1.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    time.sleep(0.25)
    sampler.stop()
    del graphs
    ms_total = e0.elapsed_time(e1)
    ms_total = max_over_ranks(ms_total, world, device=torch.device("cuda", local))
    ms_step = ms_total / args.steps
    value = world * bytes_step / (ms_step * 1e-3) / 1e9
    clocks = sampler.summary(t_wall0, t_wall1)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DECODE_DTYPE,
        "data": "synthetic (seeded uniform indices, Rademacher signs, N(0,1) activations)",
        "config": bench_config(world),
        "frac_hbm": round(value / world / hbm_peak, 4),
        "timing": (f"CUDA-graph replays of the step over {NG} weight copies "
                   f"({ws.index_bytes() / 1e6:.0f} MB of indices), CUDA events, max over ranks"),
        "gpu_launches": launches_per_step(ws, B) * args.steps,
        "clocks": clocks,
    }
    if rank != 0:
        return None

    # ---- extra measurements (rank 0) -------------------------------------
    result["layers_us"] = per_layer_times(torch, ws, reps=400, hbm_peak=hbm_peak)

    # roofline of the GEMV (the largest layer of the step: gate 32768x5120)
    li = 2
    L = ws.host[li]
    ms_k = gemv_kernel_time(torch, ws, li, reps=400)
    achieved = gemv_bytes(L.m, L.n, L.bpw, B) / (ms_k * 1e-3) / 1e9
    plan = ws.layers[li][0][0].decode_plan(B)
    sha = gemv_source_sha256()
    traffic = PROFILED_GEMV_TRAFFIC.get(sha)
    prof = "profiles/gemv_24b-gate-32768x5120_4bpw_b1.md"
    result["roofline"] = {
        "kernel": (f"gemv_kernel<4,1,{plan['fused_input']},{plan['warps']}> gate {L.m}x{L.n} B=1 "
                   f"({plan['bands']} bands x {plan['splits']} splits)"),
        "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
        "frac": round(achieved / hbm_peak, 4), "peak_source": f"{peak_src} hbm_gbs (burst)",
        "traffic": traffic,
        "traffic_source": (f"{prof}: ncu capture of this kernel source (glq_gemv.cu sha256 {sha[:12]}...)"
                           if traffic is not None else
                           f"null: glq_gemv.cu changed since the capture in {prof}"),
        "kernel_us": round(ms_k * 1e3, 3),
        "algorithmic_bytes": gemv_bytes(L.m, L.n, L.bpw, B),
    }

    # e2e through the public API with host buffers: per step, the step's
    # inputs (the five layers' x, contiguous in pinned host memory) go to the
    # device in one copy and its result (the five y) comes back in one copy
    xdt = ws.xdt
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
        for (lay, _, _), x, y in zip(ws.copy(c), xv, yv):
            lay(x, out=y)
        hy.copy_(dy, non_blocking=True)

    for c in range(NG):
        e2e_step(c)
    torch.cuda.synchronize()
    reps = max(50, min(args.steps, 2000))
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for i in range(reps):
        e2e_step(i % NG)
    f1.record()
    torch.cuda.synchronize()
    ms_eager = f0.elapsed_time(f1) / reps
    # the same step captured once per weight copy in a CUDA graph (the
    # deployment form of a decode step: glq_linear is capturable), replayed:
    # every replay still copies x from pinned host memory and y back to it
    e2e_graphs = capture_graphs(torch, e2e_step, NG)
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
    del ws
    torch.cuda.empty_cache()

    if not args.quick:
        # every decode configuration at every batch it names
        result["decode"] = {
            "24b-decode-4bpw": decode_config_section(glq, torch, "24b-decode-4bpw", hbm_peak,
                                                     batches=(2, 4, 8, 16), reps=100),
            "smollm3-3b-4bpw": decode_config_section(glq, torch, "smollm3-3b-4bpw", hbm_peak,
                                                     gemv_layer=2),
            "smollm2-360m-3bpw": decode_config_section(glq, torch, "smollm2-360m-3bpw", hbm_peak),
            "single-1024-2bpw": decode_config_section(glq, torch, "single-1024-2bpw", hbm_peak),
            # 5-8 bpw residual stages and a mixed-precision model
            "24b-decode-5bpw": decode_config_section(glq, torch, "24b-decode-5bpw", hbm_peak, gemv_layer=2),
            "24b-decode-6bpw": decode_config_section(glq, torch, "24b-decode-6bpw", hbm_peak, gemv_layer=2),
            "smollm3-3b-mixed": decode_config_section(glq, torch, "smollm3-3b-mixed", hbm_peak),
        }
        result["prefill"] = prefill_section(glq, torch, tc_peak, peak_src, hbm_peak=hbm_peak)
        # the batches between the decode path and the 512-token tiles
        result["prefill_mid"] = prefill_section(glq, torch, tc_peak, peak_src, batches=(32, 64, 128), reps=20)
        result["dense_bf16_reference"] = dense_reference_section(glq, torch, hbm_peak, tc_peak)

    # fp64 oracle on the host cores: one decode step (1 token, 5 layers) on
    # one thread and on every host core, and a 64-token prefill sample
    if world == 1 and not args.no_cpu:
        from oracle import glq_oracle as orc
        host = [gi.workload_layer(gi.WORKLOADS[MAIN_WORKLOAD], i) for i in range(5)]
        xb1 = [gi.workload_x(gi.WORKLOADS[MAIN_WORKLOAD], i, 1) for i in range(5)]
        nthr = orc.default_threads()
        secs_all = oracle_step_seconds(host, xb1, True, threads=nthr)
        secs_one = oracle_step_seconds(host, xb1, True, threads=1)
        result["cpu_baseline"] = {
            "value": round(bytes_step / secs_all / 1e9, 4), "unit": "GB/s", "cores": nthr,
            "kind": "oracle", "seconds": round(secs_all, 3),
            "sample": (f"one full step: 1 token through q, o, gate, up, down of the 24B-class workload "
                       f"(fp64), rows of each layer split over {nthr} threads"),
            "single_core": {"value": round(bytes_step / secs_one / 1e9, 4), "unit": "GB/s", "cores": 1,
                            "seconds": round(secs_one, 3)},
            "prefill_sample": oracle_prefill_sample(nthr),
        }
    return result


# ---------------------------------------------------------------------------
# the reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    world, rank, local = dist_setup()
    if world > 1 and rank != 0:
        return None
    from oracle import glq_oracle as orc
    wl = gi.WORKLOADS[MAIN_WORKLOAD]
    host = [gi.workload_layer(wl, i) for i in range(len(wl.layers))]
    xbits = [gi.workload_x(wl, i, 1) for i in range(len(wl.layers))]
    bytes_step = sum(layer_bytes(L.m, L.n, L.bpw, 1, 2) for L in host)
    nthr = orc.default_threads()
    oracle_step_seconds(host, xbits, True, threads=nthr)  # one untimed step
    budget = 120.0
    times = []
    t_start = time.perf_counter()
    for i in range(args.steps):
        times.append(oracle_step_seconds(host, xbits, True, threads=nthr))
        if time.perf_counter() - t_start > budget:
            break
    t_step = sum(times) / len(times)
    value = bytes_step / t_step / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": len(times), "warmup": args.warmup,
        "ms_per_step": round(t_step * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(world),
        "timing": f"wall clock per step on the host, {nthr} threads; stops after {budget:.0f} s",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthr, "kind": "oracle",
                         "sample": (f"{len(times)} full steps (1 token, 5 layers of the 24B-class workload) of "
                                    f"the fp64 oracle, rows split over {nthr} threads")},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_prefill_only(args):
    """The prefill timings alone, one JSON object (not the bench line)."""
    import torch
    import e8_lattice_codebook_b200 as glq
    torch.cuda.set_device(0)
    hbm_peak, tc_peak, _, peak_src = read_peaks()
    batches = (args.prefill_batch,) if args.prefill_batch else (512, 2048, 8192)
    return {"section": "prefill", "prefill": prefill_section(glq, torch, tc_peak, peak_src, batches,
                                                            reps=max(1, min(args.steps, 20)),
                                                            hbm_peak=hbm_peak)}


def run_transforms_only(args):
    """The prefill layers' input transforms alone, both kernels, one JSON
    object (not the bench line; profiling runs: the launch order is that of
    input_transform_times)."""
    import torch
    import e8_lattice_codebook_b200 as glq
    torch.cuda.set_device(0)
    hbm_peak = read_peaks()[0]
    B = args.prefill_batch or 2048
    wp = WorkloadSet(glq, torch, "prefill-8b-mlp-4bpw", 8192, ncopy=1)
    return {"section": "transforms", "B": B,
            "input_transform": input_transform_times(glq, torch, wp, B, hbm_peak,
                                                     reps=max(1, min(args.steps, 50)))}


def run_decode_only(args):
    """One decode configuration's timings alone, one JSON object (not the
    bench line; profiling runs)."""
    import torch
    import e8_lattice_codebook_b200 as glq
    torch.cuda.set_device(0)
    hbm_peak = read_peaks()[0]
    key = args.workload or MAIN_WORKLOAD
    batches = (args.decode_batch,) if args.decode_batch else None
    gl = 2 if key in ("24b-decode-4bpw", "smollm3-3b-4bpw") else None
    return {"section": "decode", "workload": key,
            "decode": decode_config_section(glq, torch, key, hbm_peak, batches,
                                            reps=max(20, min(args.steps, 400)), gemv_layer=gl)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["glq", "reference"], default="glq")
    ap.add_argument("--quick", action="store_true", help="skip the 24B sweep and prefill")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle baseline")
    ap.add_argument("--section", choices=["all", "prefill", "decode", "transforms"], default="all",
                    help="prefill / decode: time only that workload (profiling runs)")
    ap.add_argument("--workload", default="", help="with --section decode: the workload key")
    ap.add_argument("--prefill-batch", type=int, default=0,
                    help="with --section prefill: one batch instead of 512, 2048, 8192")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="with --section decode: one batch instead of the workload's batches")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.section == "prefill":
        res = run_prefill_only(args)
    elif args.section == "transforms":
        res = run_transforms_only(args)
    elif args.section == "decode":
        res = run_decode_only(args)
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
