"""ctypes wrapper around the fp64 CPU oracle in ``glq_oracle.c``.

TEST INFRASTRUCTURE ONLY: the test-suite, the package entry point's smoke
check and the benchmark's CPU-baseline leg are the only callers.  The CUDA
library never imports this module and this module never imports the CUDA
library.

Every function here is a thin marshalling layer over the C oracle; the
arithmetic lives in ``glq_oracle.c`` and follows the GLQ project pages cited
there (glq 0.5.1 PyPI page: "How it works", "Bit widths", "Inference
kernels").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "glq_oracle.c")
_LIB = os.path.join(_HERE, "libglq_oracle.so")

CODEBOOK_ENTRIES = 65536


def build(force: bool = False) -> str:
    """Compiles the oracle into ``libglq_oracle.so`` beside its source."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    # -ffp-contract=off: no silent a*b+c fusion; the one fused step is the
    # explicit fmaf() of the residual reconstruction.
    subprocess.check_call([
        "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
        "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    c_i64, c_int, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.glq_oracle_f16_to_double.restype = ctypes.c_double
    lib.glq_oracle_f16_to_double.argtypes = [ctypes.c_uint16]
    lib.glq_oracle_bf16_to_double.restype = ctypes.c_double
    lib.glq_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.glq_oracle_e8_points.restype = c_i64
    lib.glq_oracle_e8_points.argtypes = [c_int, vp, c_i64]
    lib.glq_oracle_hadamard_blocks.restype = c_int
    lib.glq_oracle_hadamard_blocks.argtypes = [c_i64, vp, c_int]
    lib.glq_oracle_hadamard_matrix.restype = None
    lib.glq_oracle_hadamard_matrix.argtypes = [c_i64, vp]
    lib.glq_oracle_hadamard_apply.restype = None
    lib.glq_oracle_hadamard_apply.argtypes = [c_i64, vp, vp, c_int]
    lib.glq_oracle_decode_rows.restype = c_int
    lib.glq_oracle_decode_rows.argtypes = [
        c_i64, c_i64, c_int, vp, vp, vp, vp, ctypes.c_float, ctypes.c_float,
        c_i64, c_i64, vp]
    lib.glq_oracle_linear.restype = c_int
    lib.glq_oracle_linear.argtypes = [
        c_i64, c_i64, c_int, vp, vp, vp, vp, ctypes.c_float, ctypes.c_float,
        vp, vp, vp, c_int, c_i64, vp]
    lib.glq_oracle_linear_mt.restype = c_int
    lib.glq_oracle_linear_mt.argtypes = [
        c_i64, c_i64, c_int, vp, vp, vp, vp, ctypes.c_float, ctypes.c_float,
        vp, vp, vp, c_int, c_i64, vp, c_int]
    lib.glq_oracle_stage_bits.restype = c_int
    lib.glq_oracle_stage_bits.argtypes = [c_int, vp]
    lib.glq_oracle_decode_stages.restype = c_int
    lib.glq_oracle_decode_stages.argtypes = [
        c_i64, c_i64, c_int, vp, vp, vp, vp, vp, ctypes.c_float, vp, c_i64, c_i64, vp]
    lib.glq_oracle_linear_stages_mt.restype = c_int
    lib.glq_oracle_linear_stages_mt.argtypes = [
        c_i64, c_i64, c_int, vp, vp, vp, vp, vp, ctypes.c_float, vp,
        vp, vp, vp, c_int, c_i64, vp, c_int]
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def f16_bits_to_double(bits) -> float:
    return _load().glq_oracle_f16_to_double(int(bits))


def bf16_bits_to_double(bits) -> float:
    return _load().glq_oracle_bf16_to_double(int(bits))


def e8_points(max_norm: int = 12, max_entries: int = 200000):
    """All E8 points of squared norm <= max_norm, sorted by (norm, x0..x7).

    Returns (points[k][8] float64, total) with k = min(total, max_entries).
    """
    out = np.zeros((max_entries, 8), dtype=np.float64)
    total = _load().glq_oracle_e8_points(int(max_norm), _ptr(out), int(max_entries))
    if total < 0:
        raise RuntimeError("oracle E8 enumeration failed")
    return out[:min(total, max_entries)].copy(), int(total)


_codebook_cache = None


def e8_codebook() -> np.ndarray:
    """The 65,536 x 8 E8 shell codebook (float64, every value a multiple of 1/2)."""
    global _codebook_cache
    if _codebook_cache is None:
        cb, total = e8_points(12, CODEBOOK_ENTRIES)
        if total < CODEBOOK_ENTRIES:
            raise RuntimeError("fewer than 65,536 E8 points of norm <= 12")
        cb.setflags(write=False)
        _codebook_cache = cb
    return _codebook_cache


def hadamard_blocks(n: int):
    sizes = np.zeros(64, dtype=np.int64)
    nb = _load().glq_oracle_hadamard_blocks(int(n), _ptr(sizes), 64)
    if nb < 0:
        raise ValueError(f"bad size {n}")
    return [int(s) for s in sizes[:nb]]


def hadamard_matrix(n: int) -> np.ndarray:
    H = np.zeros((n, n), dtype=np.float64)
    _load().glq_oracle_hadamard_matrix(int(n), _ptr(H))
    return H


def hadamard_apply(v, force_dense: bool = False) -> np.ndarray:
    """H_n v for a 1-D vector (block-diagonal normalised Hadamard)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty_like(v)
    _load().glq_oracle_hadamard_apply(v.shape[0], _ptr(v), _ptr(out), int(bool(force_dense)))
    return out


def stage_bits(bpw: int) -> list:
    """Index widths of the residual stages of a bit width, as the oracle reads
    the "Bit widths" table (16-bit E8 stages, then an 8-bit stage for an odd
    bpw)."""
    bits = np.zeros(4, dtype=np.int32)
    k = _load().glq_oracle_stage_bits(int(bpw), _ptr(bits))
    if k < 0:
        raise ValueError(f"bad bpw {bpw}")
    return [int(b) for b in bits[:k]]


def _table8(cb2):
    if cb2 is None:
        return None
    cb2 = np.asarray(cb2)
    if cb2.dtype == np.uint16:  # fp16 bits
        cb2 = f16_table_to_double(cb2)
    return np.ascontiguousarray(cb2, dtype=np.float64).reshape(256, 8)


def f16_table_to_double(bits) -> np.ndarray:
    """fp16 bit patterns -> float64 through the oracle's own binary16 decoder."""
    bits = np.asarray(bits, dtype=np.uint16)
    lib = _load()
    flat = [lib.glq_oracle_f16_to_double(int(b)) for b in bits.reshape(-1)]
    return np.array(flat, dtype=np.float64).reshape(bits.shape)


class _Stages:
    """The residual stages of a call, marshalled for the C oracle: index
    arrays (kept alive), their pointer array and the scale array."""

    def __init__(self, m, n, bpw, idx1, idx2, rs, cb2):
        G = n // 8
        self.bits = stage_bits(bpw)
        self.idx1 = np.ascontiguousarray(idx1, dtype=np.uint16).reshape(m, G)
        if not self.bits:
            arrays, scales = [], []
        elif bpw <= 4:
            arrays, scales = [idx2], [rs]
        else:
            arrays, scales = list(idx2), list(rs)
        if len(arrays) != len(self.bits) or len(scales) != len(self.bits):
            raise ValueError("residual stages do not match the bit width")
        self.arrays = [np.ascontiguousarray(a, dtype=np.uint16 if b == 16 else np.uint8).reshape(m, G)
                       for a, b in zip(arrays, self.bits)]
        self.ptrs = (ctypes.c_void_p * 4)(*([a.ctypes.data for a in self.arrays] + [None] * (4 - len(self.arrays))))
        self.scales = np.zeros(4, dtype=np.float32)
        self.scales[:len(scales)] = np.asarray(scales, dtype=np.float32)
        self.cb1 = e8_codebook()
        self.cb16 = self.cb1 if 16 in self.bits else None
        if 8 in self.bits and cb2 is None:
            raise ValueError("an odd bpw needs the 256-entry residual codebook")
        self.cb8 = _table8(cb2) if 8 in self.bits else None
        if bpw == 4 and cb2 is not None:  # an explicit table for the 16-bit stage
            self.cb16 = np.ascontiguousarray(cb2, dtype=np.float64)


def decode_rows(m, n, bpw, idx1, idx2, ws, rs, r0=0, r1=None, cb2=None) -> np.ndarray:
    """Explicit W^ rows [r0, r1) as float64 arrays holding fp32 values.

    bpw 2..4: idx2 an array (or None), rs a float; bpw 5..8: idx2 a list of
    the residual stages' index arrays and rs a list of their scales.  cb2:
    the 256-entry table of an odd bpw (fp16 bits or values).
    """
    r1 = m if r1 is None else r1
    st = _Stages(m, n, bpw, idx1, idx2, rs, cb2)
    w = np.zeros((r1 - r0, n), dtype=np.float64)
    rc = _load().glq_oracle_decode_stages(m, n, bpw, _ptr(st.idx1), ctypes.cast(st.ptrs, ctypes.c_void_p),
                                          _ptr(st.cb1), _ptr(st.cb16), _ptr(st.cb8), float(ws),
                                          _ptr(st.scales), r0, r1, _ptr(w))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return w


def default_threads() -> int:
    """Host threads the oracle uses when asked for all of them."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def linear(m, n, bpw, idx1, idx2, ws, rs, s_in, s_out, x_bits, x_is_bf16, cb2=None,
           threads: int = 1) -> np.ndarray:
    """y[B][m] (float64) = S_out . H_m . W^ . H_n . (S_in . x).

    x_bits: uint16 [B][n] holding fp16 (x_is_bf16 False) or bf16 bit patterns.
    idx2 / rs / cb2 as decode_rows (per-stage lists from 5 bpw).
    threads: POSIX threads the rows of W^ xr are split over (0: every host
    core); the result does not depend on it.
    """
    threads = default_threads() if threads == 0 else int(threads)
    st = _Stages(m, n, bpw, idx1, idx2, rs, cb2)
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1, n)
    B = x_bits.shape[0]
    s_in = np.ascontiguousarray(s_in, dtype=np.int8)
    s_out = np.ascontiguousarray(s_out, dtype=np.int8)
    y = np.zeros((B, m), dtype=np.float64)
    rc = _load().glq_oracle_linear_stages_mt(m, n, bpw, _ptr(st.idx1), ctypes.cast(st.ptrs, ctypes.c_void_p),
                                             _ptr(st.cb1), _ptr(st.cb16), _ptr(st.cb8), float(ws),
                                             _ptr(st.scales), _ptr(s_in), _ptr(s_out), _ptr(x_bits),
                                             int(bool(x_is_bf16)), B, _ptr(y), threads)
    if rc != 0:
        raise ValueError("oracle linear rejected its arguments")
    return y
