"""Seeded synthetic inputs for the GLQ compressed-weight linear layer.

This module only draws random numbers; it holds none of the layer's
arithmetic.  Both the CUDA path (through the package's Python binding) and
the fp64 oracle consume the same host arrays it produces.

Recipe (numpy PCG64, ``numpy.random.default_rng``):
  * per layer, ``rng = default_rng([seed, layer_id])`` draws, in order:
    idx1 (uint16, uniform [0, 65536)); the residual stages of the bit width
    in stage order (a 16-bit E8 stage: uint16 uniform; the 8-bit stage of an
    odd bpw: uint8 uniform [0, 256)); for an odd bpw the 256-entry residual
    codebook (256 x 8 normal draws of standard deviation 0.5, rounded to
    fp16); S_in and S_out (Rademacher +-1, int8).  Residual stage s (s = 1,
    2, ...) has the scale 8^-s;
  * per (layer, batch), ``rng = default_rng([seed, layer_id, 1_000_000 + B])``
    draws x ~ N(0, 1) of shape [B][n] (float64), then -- when the workload
    has outliers -- floor(0.01 n) distinct columns, which are multiplied by
    20 for every token; x is then rounded to fp16 or bf16 (nearest even).

The workloads mirror the shapes of the models the GLQ project pages serve
(SmolLM2-360M, SmolLM3-3B, a 24B-class model, an 8B-class MLP prefill), plus
the 24B-class shapes at 5 and 6 bpw and a mixed-precision SmolLM3-3B-shaped
set (the pages' 3.5 / 4.5 bpw "mixed" checkpoints are layers of different
bit widths).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

CODEBOOK_ENTRIES = 65536
RESIDUAL8_ENTRIES = 256


@dataclass(frozen=True)
class LayerSpec:
    name: str
    m: int  # output features
    n: int  # input features


@dataclass(frozen=True)
class Workload:
    key: str
    description: str
    seed: int
    bpw: int
    x_dtype: str  # "f16" | "bf16"
    layers: tuple
    batches: tuple
    weight_scale: float = 0.05
    resid_scale: float = 0.125
    outliers: bool = False
    extra: dict = field(default_factory=dict)
    layer_bpw: tuple = ()  # per-layer bit widths of a mixed-precision model (overrides bpw)

    def bpw_of(self, layer_id: int) -> int:
        return self.layer_bpw[layer_id] if self.layer_bpw else self.bpw


WORKLOADS = {
    "single-1024-2bpw": Workload(
        "single-1024-2bpw",
        "single GLQ linear 1024x1024 at 2 bpw (one uint16 index per 8 weights), fp16 x",
        seed=0, bpw=2, x_dtype="f16",
        layers=(LayerSpec("linear", 1024, 1024),), batches=(1,)),
    "smollm3-3b-4bpw": Workload(
        "smollm3-3b-4bpw",
        "SmolLM3-3B-shaped projections at 4 bpw (uint16 + uint16 E8 residual, rs 1/8), bf16 x",
        seed=1, bpw=4, x_dtype="bf16",
        layers=(LayerSpec("q", 2048, 2048), LayerSpec("o", 2048, 2048),
                LayerSpec("gate", 11008, 2048), LayerSpec("up", 11008, 2048),
                LayerSpec("down", 2048, 11008)),
        batches=(1, 4)),
    "smollm2-360m-3bpw": Workload(
        "smollm2-360m-3bpw",
        "SmolLM2-360M-shaped non-power-of-two layers at 3 bpw (uint16 + uint8 residual, rs 1/8), fp16 x",
        seed=2, bpw=3, x_dtype="f16",
        layers=(LayerSpec("attn", 960, 960), LayerSpec("gate_up", 2560, 960),
                LayerSpec("down", 960, 2560)),
        batches=(1, 2, 8)),
    "24b-decode-4bpw": Workload(
        "24b-decode-4bpw",
        "24B-class decode sweep at 4 bpw (hidden 5120, MLP 32768), bf16 x",
        seed=3, bpw=4, x_dtype="bf16",
        layers=(LayerSpec("q", 4096, 5120), LayerSpec("o", 5120, 4096),
                LayerSpec("gate", 32768, 5120), LayerSpec("up", 32768, 5120),
                LayerSpec("down", 5120, 32768)),
        batches=(1, 2, 4, 8, 16)),
    "24b-decode-5bpw": Workload(
        "24b-decode-5bpw",
        "24B-class decode at 5 bpw (uint16 + uint16 E8 + uint8 residual stages, scales 1/8, 1/64), bf16 x",
        seed=13, bpw=5, x_dtype="bf16",
        layers=(LayerSpec("q", 4096, 5120), LayerSpec("o", 5120, 4096),
                LayerSpec("gate", 32768, 5120), LayerSpec("up", 32768, 5120),
                LayerSpec("down", 5120, 32768)),
        batches=(1, 16)),
    "24b-decode-6bpw": Workload(
        "24b-decode-6bpw",
        "24B-class decode at 6 bpw (uint16 + two uint16 E8 residual stages, scales 1/8, 1/64), bf16 x",
        seed=14, bpw=6, x_dtype="bf16",
        layers=(LayerSpec("q", 4096, 5120), LayerSpec("o", 5120, 4096),
                LayerSpec("gate", 32768, 5120), LayerSpec("up", 32768, 5120),
                LayerSpec("down", 5120, 32768)),
        batches=(1, 16)),
    "smollm3-3b-mixed": Workload(
        "smollm3-3b-mixed",
        "SmolLM3-3B-shaped projections, mixed precision: q, o at 4 bpw; gate, up, down at 5 bpw "
        "(4.64 bpw by weight), bf16 x",
        seed=15, bpw=5, x_dtype="bf16",
        layers=(LayerSpec("q", 2048, 2048), LayerSpec("o", 2048, 2048),
                LayerSpec("gate", 11008, 2048), LayerSpec("up", 11008, 2048),
                LayerSpec("down", 2048, 11008)),
        batches=(1, 4), layer_bpw=(4, 4, 5, 5, 5)),
    "prefill-8b-mlp-4bpw": Workload(
        "prefill-8b-mlp-4bpw",
        "prefill GEMM at 4 bpw, 14336x4096 and 4096x14336, bf16 x with 1% outlier columns x20",
        seed=5, bpw=4, x_dtype="bf16", outliers=True,
        layers=(LayerSpec("up", 14336, 4096), LayerSpec("down", 4096, 14336)),
        batches=(512, 2048, 8192)),
}


def stage_bits(bpw: int) -> list:
    """Index widths of the residual stages of a bit width (after the 16-bit
    primary): 16-bit E8 stages, then one 8-bit stage for an odd bpw."""
    if not 2 <= bpw <= 8:
        raise ValueError("bpw must be in 2..8")
    return [16] * ((bpw - 2) // 2) + ([8] if bpw % 2 else [])


@dataclass
class LayerInputs:
    m: int
    n: int
    bpw: int
    idx1: np.ndarray          # uint16 [m][n/8]
    # residual indices: None (2 bpw); one array (3 bpw: uint8, 4 bpw: uint16);
    # from 5 bpw a list with one array per stage (stage order)
    idx2: object
    cb2_f16: np.ndarray | None  # uint16 fp16 bits [256][8] for an odd bpw
    s_in: np.ndarray          # int8 [n], +-1
    s_out: np.ndarray         # int8 [m], +-1
    weight_scale: float
    resid_scale: object       # float (2-4 bpw) or a list of one scale per stage

    def stages(self):
        """(list of residual index arrays, list of their scales)."""
        if self.bpw == 2:
            return [], []
        if self.bpw <= 4:
            return [self.idx2], [self.resid_scale]
        return list(self.idx2), list(self.resid_scale)


def _rademacher(rng, k):
    return (rng.integers(0, 2, size=k, dtype=np.int8) * 2 - 1).astype(np.int8)


def make_layer(seed: int, layer_id: int, m: int, n: int, bpw: int,
               weight_scale: float = 0.05, resid_scale: float = 0.125) -> LayerInputs:
    if n % 8:
        raise ValueError("n must be a multiple of 8")
    bits = stage_bits(bpw)
    rng = np.random.default_rng([seed, layer_id])
    G = n // 8
    idx1 = rng.integers(0, CODEBOOK_ENTRIES, size=(m, G), dtype=np.uint16)
    res = []
    for b in bits:
        if b == 16:
            res.append(rng.integers(0, CODEBOOK_ENTRIES, size=(m, G), dtype=np.uint16))
        else:
            res.append(rng.integers(0, RESIDUAL8_ENTRIES, size=(m, G), dtype=np.uint8))
    cb2 = None
    if bpw % 2:
        cb2 = rng.normal(0.0, 0.5, size=(RESIDUAL8_ENTRIES, 8)).astype(np.float16).view(np.uint16)
    s_in = _rademacher(rng, n)
    s_out = _rademacher(rng, m)
    if bpw <= 4:
        idx2 = res[0] if res else None
        rs = float(resid_scale)
    else:
        idx2 = res
        rs = [float(resid_scale) ** (s + 1) for s in range(len(res))]
    return LayerInputs(m, n, bpw, idx1, idx2, cb2, s_in, s_out, float(weight_scale), rs)


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float64 -> float32 -> bf16 (nearest even), as uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def make_x(seed: int, layer_id: int, B: int, n: int, x_dtype: str,
           outliers: bool = False) -> np.ndarray:
    """x[B][n] as uint16 fp16 / bf16 bit patterns."""
    rng = np.random.default_rng([seed, layer_id, 1_000_000 + B])
    x = rng.standard_normal(size=(B, n))
    if outliers:
        k = int(np.floor(0.01 * n))
        cols = rng.choice(n, size=k, replace=False)
        x[:, cols] *= 20.0
    if x_dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if x_dtype == "bf16":
        return f64_to_bf16_bits(x)
    raise ValueError(x_dtype)


def workload_layer(wl: Workload, layer_id: int) -> LayerInputs:
    spec = wl.layers[layer_id]
    return make_layer(wl.seed, layer_id, spec.m, spec.n, wl.bpw_of(layer_id), wl.weight_scale, wl.resid_scale)


def workload_x(wl: Workload, layer_id: int, B: int) -> np.ndarray:
    spec = wl.layers[layer_id]
    return make_x(wl.seed, layer_id, B, spec.n, wl.x_dtype, wl.outliers)
