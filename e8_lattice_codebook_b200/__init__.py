"""glq-b200: B200-native (sm_100a) GLQ compressed-weight linear layer.

    y = S_out . H_m . W^ . H_n . (S_in . x)

W^ is stored as 16-bit indices into a 65,536-entry E8 lattice codebook (one
per 8 weights), optionally refined by a uint8 (256-entry) or uint16 (E8)
residual index times a residual scale, times a per-layer weight scale; H is
a normalised (block-diagonal) Walsh-Hadamard transform and S_in / S_out are
random +-1 signs (GLQ project pages: glq 0.5.1 PyPI page, "How it works",
"Bit widths", "Inference kernels"; GLQ v0.3.2 release notes).

This module is argument marshalling over the C ABI of ``libglq_b200.so``
(declared in include/glq.h): every step of the layer runs in the library's
CUDA kernels.  PyTorch is used only for device memory and streams.  There is
no CPU fallback: if the library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libglq_b200.so")

GLQ_F16, GLQ_BF16, GLQ_F32 = 0, 1, 2

STATUS = {
    0: "GLQ_OK", 1: "GLQ_ERR_INVALID_ARG", 2: "GLQ_ERR_SHAPE", 3: "GLQ_ERR_DTYPE",
    4: "GLQ_ERR_BPW", 5: "GLQ_ERR_NO_CODEBOOK", 6: "GLQ_ERR_OOM", 7: "GLQ_ERR_CUDA",
    8: "GLQ_ERR_DEVICE_CHECK", 9: "GLQ_ERR_TIMEOUT", 10: "GLQ_ERR_UNSUPPORTED", 11: "GLQ_ERR_CAPTURE",
}

# every symbol include/glq.h declares
EXPORTS = (
    "glq_status_str", "glq_version", "glq_e8_codebook", "glq_codebook_upload",
    "glq_codebook_destroy", "glq_layer_create", "glq_layer_destroy", "glq_layer_reserve",
    "glq_linear", "glq_dequant_reference", "glq_rht_input", "glq_rht_output",
    "glq_layer_check", "glq_layer_info", "glq_gemv_replay", "glq_linear_noalloc", "glq_decode_plan",
    "glq_prefill_replay", "glq_layer_set_fusion", "glq_layer_set_prefill_reconstruct",
    "glq_workspace_info", "glq_workspace_release", "glq_layer_create_stages",
    "glq_layer_set_batch_invariant", "glq_layer_create_shard", "glq_cast",
    "glq_rht_input_operand", "glq_layer_selftest_wait",
)


class GlqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS.get(status, status)}")
        self.status = status


_vp, _i64, _i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32

# argument / result types of every exported function
_SIGNATURES = {
    "glq_status_str": ([ctypes.c_int], ctypes.c_char_p),
    "glq_version": ([], ctypes.c_char_p),
    "glq_e8_codebook": ([_vp], ctypes.c_int),
    "glq_codebook_upload": ([_vp, _i32, _i32, ctypes.POINTER(_vp)], ctypes.c_int),
    "glq_codebook_destroy": ([_vp], ctypes.c_int),
    "glq_layer_create": ([_i64, _i64, _i32, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float,
                          _vp, _vp, ctypes.POINTER(_vp)], ctypes.c_int),
    "glq_layer_create_stages": ([_i64, _i64, _i32, _vp, _vp, _vp, _vp, ctypes.c_float, _vp,
                                 _vp, _vp, ctypes.POINTER(_vp)], ctypes.c_int),
    "glq_layer_create_shard": ([_i64, _i64, _i32, _vp, _vp, _vp, _vp, ctypes.c_float, _vp,
                                _vp, _vp, _i64, _i64, ctypes.POINTER(_vp)], ctypes.c_int),
    "glq_cast": ([_vp, _vp, ctypes.c_int, _i64, _vp], ctypes.c_int),
    "glq_layer_destroy": ([_vp], ctypes.c_int),
    "glq_layer_reserve": ([_vp, _i64], ctypes.c_int),
    "glq_linear": ([_vp, _vp, ctypes.c_int, _vp, ctypes.c_int, _i64, _vp], ctypes.c_int),
    "glq_linear_noalloc": ([_vp, _vp, ctypes.c_int, _vp, ctypes.c_int, _i64, _vp], ctypes.c_int),
    "glq_dequant_reference": ([_vp, _vp, _vp], ctypes.c_int),
    "glq_rht_input": ([_vp, _vp, ctypes.c_int, _vp, _i64, _vp], ctypes.c_int),
    "glq_rht_output": ([_vp, _vp, _vp, ctypes.c_int, _i64, _vp], ctypes.c_int),
    "glq_rht_input_operand": ([_vp, _vp, ctypes.c_int, _vp, _vp, _i64, ctypes.c_int, _vp], ctypes.c_int),
    "glq_layer_selftest_wait": ([_vp, ctypes.c_int, ctypes.c_int, _i64, _vp], ctypes.c_int),
    "glq_layer_check": ([_vp, _vp], ctypes.c_int),
    "glq_gemv_replay": ([_vp, _i64, _vp], ctypes.c_int),
    "glq_prefill_replay": ([_vp, _i64, _vp], ctypes.c_int),
    "glq_layer_set_fusion": ([_vp, ctypes.c_int32], ctypes.c_int),
    "glq_layer_set_prefill_reconstruct": ([_vp, _i64], ctypes.c_int),
    "glq_layer_set_batch_invariant": ([_vp, ctypes.c_int32], ctypes.c_int),
    "glq_decode_plan": ([_vp, _i64, ctypes.POINTER(_i32), ctypes.POINTER(_i32), ctypes.POINTER(_i32),
                         ctypes.POINTER(_i32), ctypes.POINTER(_i32)], ctypes.c_int),
    "glq_layer_info": ([_vp, ctypes.POINTER(_i64), ctypes.POINTER(_i64), ctypes.POINTER(_i32),
                        ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "glq_workspace_info": ([_i32, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "glq_workspace_release": ([_i32], ctypes.c_int),
}

_lib = None


def _L():
    """The loaded library (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m e8_lattice_codebook_b200.build` "
                "(the GLQ layer has no CPU fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
    return _lib


def _ok(st: int, what: str):
    if st != 0:
        raise GlqError(st, what)


# ---------------------------------------------------------------------------
# C-ABI mirrors (same names, same arguments; raw pointers and sizes)
# ---------------------------------------------------------------------------

def glq_status_str(status: int) -> str:
    return _L().glq_status_str(status).decode()


def glq_version() -> str:
    return _L().glq_version().decode()


def glq_e8_codebook() -> np.ndarray:
    """The library's 65,536 x 8 E8 codebook as fp16 bit patterns (uint16)."""
    out = np.zeros((65536, 8), dtype=np.uint16)
    _ok(_L().glq_e8_codebook(out.ctypes.data), "glq_e8_codebook")
    return out


def glq_codebook_upload(fp16_bits: np.ndarray) -> int:
    a = np.ascontiguousarray(fp16_bits, dtype=np.uint16)
    if a.ndim != 2:
        raise ValueError("codebook must be [entries][8]")
    h = _vp()
    _ok(_L().glq_codebook_upload(a.ctypes.data, a.shape[0], a.shape[1], ctypes.byref(h)), "glq_codebook_upload")
    return h.value


def glq_codebook_destroy(handle: int) -> None:
    _ok(_L().glq_codebook_destroy(handle), "glq_codebook_destroy")


def glq_layer_create(m, n, bpw, idx1, idx2, primary, residual, weight_scale, resid_scale,
                     s_in, s_out) -> int:
    idx1 = np.ascontiguousarray(idx1, dtype=np.uint16)
    if idx2 is not None:
        idx2 = np.ascontiguousarray(idx2, dtype=np.uint8 if bpw == 3 else np.uint16)
    s_in = np.ascontiguousarray(s_in, dtype=np.int8)
    s_out = np.ascontiguousarray(s_out, dtype=np.int8)
    if idx1.size != m * (n // 8) or s_in.size != n or s_out.size != m:
        raise ValueError("array sizes do not match m, n")
    if idx2 is not None and idx2.size != idx1.size:
        raise ValueError("idx2 size does not match idx1")
    h = _vp()
    _ok(_L().glq_layer_create(m, n, bpw, idx1.ctypes.data, None if idx2 is None else idx2.ctypes.data,
                          primary, residual, float(weight_scale), float(resid_scale),
                          s_in.ctypes.data, s_out.ctypes.data, ctypes.byref(h)),
        "glq_layer_create")
    return h.value


def stage_bits(bpw: int) -> list:
    """Index widths of the residual stages of a bit width (glq 0.5.1 PyPI
    page, "Bit widths"): 16-bit E8 stages, then an 8-bit stage for odd bpw."""
    if not 2 <= bpw <= 8:
        raise ValueError("bpw must be in 2..8")
    return [16] * ((bpw - 2) // 2) + ([8] if bpw % 2 else [])


def glq_layer_create_stages(m, n, bpw, idx1, idx_res, primary, residual, weight_scale, resid_scales,
                            s_in, s_out) -> int:
    """idx_res: one [m][n/8] index array per residual stage (stage order),
    resid_scales: one scale per stage."""
    bits = stage_bits(bpw)
    idx_res = list(idx_res or [])
    scales = np.ascontiguousarray(list(resid_scales or []), dtype=np.float32)
    if len(idx_res) != len(bits) or scales.size != len(bits):
        raise ValueError(f"bpw {bpw} has {len(bits)} residual stages")
    idx1 = np.ascontiguousarray(idx1, dtype=np.uint16)
    arrays = [np.ascontiguousarray(a, dtype=np.uint16 if b == 16 else np.uint8) for a, b in zip(idx_res, bits)]
    s_in = np.ascontiguousarray(s_in, dtype=np.int8)
    s_out = np.ascontiguousarray(s_out, dtype=np.int8)
    if idx1.size != m * (n // 8) or s_in.size != n or s_out.size != m or any(a.size != idx1.size for a in arrays):
        raise ValueError("array sizes do not match m, n")
    ptrs = (ctypes.c_void_p * max(1, len(arrays)))(*[a.ctypes.data for a in arrays])
    h = _vp()
    _ok(_L().glq_layer_create_stages(m, n, bpw, idx1.ctypes.data, ctypes.cast(ptrs, ctypes.c_void_p) if arrays else None,
                                     primary, residual, float(weight_scale),
                                     scales.ctypes.data if arrays else None, s_in.ctypes.data,
                                     s_out.ctypes.data, ctypes.byref(h)),
        "glq_layer_create_stages")
    return h.value


def _stage_args(m, n, bpw, idx1, idx_res, resid_scales, s_in, s_out):
    bits = stage_bits(bpw)
    idx_res = list(idx_res or [])
    scales = np.ascontiguousarray(list(resid_scales or []), dtype=np.float32)
    if len(idx_res) != len(bits) or scales.size != len(bits):
        raise ValueError(f"bpw {bpw} has {len(bits)} residual stages")
    idx1 = np.ascontiguousarray(idx1, dtype=np.uint16)
    arrays = [np.ascontiguousarray(a, dtype=np.uint16 if b == 16 else np.uint8) for a, b in zip(idx_res, bits)]
    s_in = np.ascontiguousarray(s_in, dtype=np.int8)
    s_out = np.ascontiguousarray(s_out, dtype=np.int8)
    if idx1.size != m * (n // 8) or s_in.size != n or s_out.size != m or any(a.size != idx1.size for a in arrays):
        raise ValueError("array sizes do not match m, n")
    ptrs = (ctypes.c_void_p * max(1, len(arrays)))(*[a.ctypes.data for a in arrays])
    keep = (idx1, arrays, scales, s_in, s_out, ptrs)
    return keep, (ctypes.cast(ptrs, ctypes.c_void_p) if arrays else None), (scales.ctypes.data if arrays else None)


def glq_layer_create_shard(m, n, bpw, idx1, idx_res, primary, residual, weight_scale, resid_scales,
                           s_in, s_out, k_begin, k_end) -> int:
    """The row-parallel part of a layer holding input columns [k_begin, k_end)
    (whole-layer host arrays; idx_res / resid_scales one per residual stage)."""
    keep, pres, pscales = _stage_args(m, n, bpw, idx1, idx_res, resid_scales, s_in, s_out)
    h = _vp()
    _ok(_L().glq_layer_create_shard(m, n, bpw, keep[0].ctypes.data, pres, primary, residual, float(weight_scale),
                                    pscales, keep[3].ctypes.data, keep[4].ctypes.data, int(k_begin), int(k_end),
                                    ctypes.byref(h)),
        "glq_layer_create_shard")
    return h.value


def glq_cast(src_ptr, dst_ptr, dtype, count, stream) -> None:
    _ok(_L().glq_cast(src_ptr, dst_ptr, dtype, int(count), stream), "glq_cast")


def glq_layer_destroy(handle: int) -> None:
    _ok(_L().glq_layer_destroy(handle), "glq_layer_destroy")


def glq_layer_reserve(handle: int, max_B: int) -> None:
    _ok(_L().glq_layer_reserve(handle, max_B), "glq_layer_reserve")


def glq_linear(handle, x_ptr, x_dtype, y_ptr, y_dtype, B, stream) -> None:
    _ok(_L().glq_linear(handle, x_ptr, x_dtype, y_ptr, y_dtype, B, stream), "glq_linear")


def glq_linear_noalloc(handle, x_ptr, x_dtype, y_ptr, y_dtype, B, stream) -> None:
    """glq_linear without device allocation (B <= 16; fixed 8 MiB device scratch)."""
    _ok(_L().glq_linear_noalloc(handle, x_ptr, x_dtype, y_ptr, y_dtype, B, stream),
        "glq_linear_noalloc")


def glq_dequant_reference(handle, w_ptr, stream) -> None:
    _ok(_L().glq_dequant_reference(handle, w_ptr, stream), "glq_dequant_reference")


def glq_rht_input(handle, x_ptr, x_dtype, xr_ptr, B, stream) -> None:
    _ok(_L().glq_rht_input(handle, x_ptr, x_dtype, xr_ptr, B, stream), "glq_rht_input")


def glq_rht_output(handle, z_ptr, y_ptr, y_dtype, B, stream) -> None:
    _ok(_L().glq_rht_output(handle, z_ptr, y_ptr, y_dtype, B, stream), "glq_rht_output")


def glq_rht_input_operand(handle, x_ptr, x_dtype, xh_ptr, info_ptr, B, kernel, stream) -> None:
    _ok(_L().glq_rht_input_operand(handle, x_ptr, x_dtype, xh_ptr, info_ptr, B, kernel, stream),
        "glq_rht_input_operand")


def glq_layer_selftest_wait(handle, kind, arrivals, limit, stream) -> None:
    _ok(_L().glq_layer_selftest_wait(handle, kind, arrivals, limit, stream), "glq_layer_selftest_wait")


def glq_gemv_replay(handle, B, stream) -> None:
    _ok(_L().glq_gemv_replay(handle, B, stream), "glq_gemv_replay")


def glq_prefill_replay(handle, B, stream) -> None:
    _ok(_L().glq_prefill_replay(handle, B, stream), "glq_prefill_replay")


GLQ_FUSE_INPUT, GLQ_FUSE_OUTPUT, GLQ_SPLITK_CLUSTER, GLQ_FUSE_DEFAULT = 1, 2, 4, -1


def glq_layer_set_fusion(handle, flags: int) -> None:
    _ok(_L().glq_layer_set_fusion(handle, int(flags)), "glq_layer_set_fusion")


def glq_layer_set_prefill_reconstruct(handle, min_batch: int) -> None:
    _ok(_L().glq_layer_set_prefill_reconstruct(handle, int(min_batch)), "glq_layer_set_prefill_reconstruct")


def glq_layer_set_batch_invariant(handle, enable: bool) -> None:
    _ok(_L().glq_layer_set_batch_invariant(handle, 1 if enable else 0), "glq_layer_set_batch_invariant")


def glq_layer_check(handle, stream) -> None:
    _ok(_L().glq_layer_check(handle, stream), "glq_layer_check")


def glq_decode_plan(handle, B: int) -> dict:
    vals = [_i32() for _ in range(5)]
    _ok(_L().glq_decode_plan(handle, int(B), *[ctypes.byref(v) for v in vals]), "glq_decode_plan")
    return dict(zip(("warps", "bands", "splits", "cluster", "fused_input"), (v.value for v in vals)))


def glq_workspace_info(device: int) -> int:
    """Bytes of the device's shared workspace (every layer's calls on it use it)."""
    nb = ctypes.c_size_t()
    _ok(_L().glq_workspace_info(int(device), ctypes.byref(nb)), "glq_workspace_info")
    return nb.value


def glq_workspace_release(device: int) -> None:
    _ok(_L().glq_workspace_release(int(device)), "glq_workspace_release")


def glq_layer_info(handle):
    m, n, bpw, nb = _i64(), _i64(), _i32(), ctypes.c_size_t()
    _ok(_L().glq_layer_info(handle, ctypes.byref(m), ctypes.byref(n), ctypes.byref(bpw), ctypes.byref(nb)),
        "glq_layer_info")
    return m.value, n.value, bpw.value, nb.value


# ---------------------------------------------------------------------------
# torch convenience (device memory and streams only)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def dtype_code(dt) -> int:
    torch = _torch()
    if dt == torch.float16:
        return GLQ_F16
    if dt == torch.bfloat16:
        return GLQ_BF16
    if dt == torch.float32:
        return GLQ_F32
    raise ValueError(f"unsupported dtype {dt}")


def _stream_ptr(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class Codebook:
    """A device codebook (65,536 x 8 E8 or 256 x 8 residual), fp16 bits on the host."""

    def __init__(self, fp16_bits: np.ndarray):
        self.entries = int(np.asarray(fp16_bits).shape[0])
        self.handle = glq_codebook_upload(fp16_bits)

    @classmethod
    def e8(cls) -> "Codebook":
        return cls(glq_e8_codebook())

    def close(self):
        if self.handle:
            glq_codebook_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class GlqLinear:
    """One compressed linear layer on the current CUDA device."""

    def __init__(self, m, n, bpw, idx1, idx2, primary: Codebook, residual: Codebook | None,
                 weight_scale, resid_scale, s_in, s_out):
        """bpw 2-4: idx2 the residual index array (or None) and resid_scale
        a float; bpw 5-8: idx2 a list of the residual stages' index arrays
        and resid_scale a list of their scales (stage order); residual: the
        256-entry codebook of an odd bpw, else None (or the E8 codebook)."""
        self.m, self.n, self.bpw = int(m), int(n), int(bpw)
        self._cbs = (primary, residual)  # keep codebooks alive
        rh = 0 if residual is None else residual.handle
        if self.bpw <= 4:
            self.handle = glq_layer_create(self.m, self.n, self.bpw, idx1, idx2, primary.handle, rh,
                                           weight_scale, resid_scale, s_in, s_out)
        else:
            self.handle = glq_layer_create_stages(self.m, self.n, self.bpw, idx1, idx2, primary.handle, rh,
                                                  weight_scale, resid_scale, s_in, s_out)

    def reserve(self, max_B: int):
        glq_layer_reserve(self.handle, max_B)

    def forward(self, x, out=None, out_dtype=None, stream=None):
        torch = _torch()
        if x.dim() != 2 or x.shape[1] != self.n or not x.is_cuda or not x.is_contiguous():
            raise ValueError("x must be a contiguous CUDA tensor [B][n]")
        B = x.shape[0]
        odt = out_dtype or x.dtype
        if out is None:
            out = torch.empty((B, self.m), dtype=odt, device=x.device)
        glq_linear(self.handle, x.data_ptr(), dtype_code(x.dtype), out.data_ptr(),
                   dtype_code(out.dtype), B, _stream_ptr(stream))
        return out

    __call__ = forward

    def dequant(self, stream=None):
        torch = _torch()
        w = torch.empty((self.m, self.n), dtype=torch.float32, device="cuda")
        glq_dequant_reference(self.handle, w.data_ptr(), _stream_ptr(stream))
        return w

    def rht_input(self, x, stream=None):
        torch = _torch()
        xr = torch.empty((x.shape[0], self.n), dtype=torch.float32, device=x.device)
        glq_rht_input(self.handle, x.data_ptr(), dtype_code(x.dtype), xr.data_ptr(), x.shape[0],
                      _stream_ptr(stream))
        return xr

    RHT_AUTO, RHT_BUTTERFLY, RHT_TENSOR = 0, 1, 2  # kernels of glq_rht_input_operand

    def rht_input_operand(self, x, kernel=0, stream=None):
        """(xh [B][n_pad] fp16 = xr 2^e per row, inv [B] fp32 = 2^-e): the
        tensor-core path's input stage with the chosen kernel."""
        torch = _torch()
        n_pad = (self.n + 127) // 128 * 128
        xh = torch.empty((x.shape[0], n_pad), dtype=torch.float16, device=x.device)
        info = torch.empty((x.shape[0], 4), dtype=torch.float32, device=x.device)
        glq_rht_input_operand(self.handle, x.data_ptr(), dtype_code(x.dtype), xh.data_ptr(), info.data_ptr(),
                              x.shape[0], kernel, _stream_ptr(stream))
        return xh, info[:, 2]

    def selftest_wait(self, kind: int, arrivals: int, limit: int, stream=None):
        """One bounded device wait on a barrier `arrivals` of its two arrivals
        reach (kind 0: cycle-bounded, 1: cluster scope, 2: poll-bounded);
        the outcome reads back through check()."""
        glq_layer_selftest_wait(self.handle, kind, arrivals, limit, _stream_ptr(stream))

    def rht_output(self, z, out_dtype=None, stream=None):
        torch = _torch()
        y = torch.empty((z.shape[0], self.m), dtype=out_dtype or torch.float32, device=z.device)
        glq_rht_output(self.handle, z.data_ptr(), y.data_ptr(), dtype_code(y.dtype), z.shape[0],
                       _stream_ptr(stream))
        return y

    def decode_plan(self, B: int) -> dict:
        return glq_decode_plan(self.handle, B)

    def gemv_replay(self, B, stream=None):
        glq_gemv_replay(self.handle, B, _stream_ptr(stream))

    def set_fusion(self, flags):
        """GLQ_FUSE_* bits; True / False mean both / neither."""
        if flags is True:
            flags = GLQ_FUSE_INPUT | GLQ_FUSE_OUTPUT
        elif flags is False:
            flags = 0
        glq_layer_set_fusion(self.handle, flags)

    def set_prefill_reconstruct(self, min_batch: int):
        """Batches >= min_batch reconstruct W in fp16 first (-1: default)."""
        glq_layer_set_prefill_reconstruct(self.handle, min_batch)

    def set_batch_invariant(self, enable: bool):
        """Every token's output independent of the batch size and path."""
        glq_layer_set_batch_invariant(self.handle, enable)

    def prefill_replay(self, B, stream=None):
        glq_prefill_replay(self.handle, B, _stream_ptr(stream))

    def check(self, stream=None):
        glq_layer_check(self.handle, _stream_ptr(stream))

    def close(self):
        if self.handle:
            glq_layer_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
