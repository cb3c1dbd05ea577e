"""Host-side checks of the C-ABI library that need no GPU: it builds for
sm_100a, loads, exports every symbol include/glq.h declares, its E8
codebook equals the oracle's (bit for bit), and argument checks that
precede any CUDA call return the documented statuses."""
import ctypes
import os
import re

import numpy as np
import pytest

from e8_lattice_codebook_b200 import build as glq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    path = glq_build.build()
    return ctypes.CDLL(path)


def header_symbols():
    with open(os.path.join(ROOT, "include", "glq.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"GLQ_API[^;(]*?\b(glq_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    syms = header_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(lib, s), s
    import e8_lattice_codebook_b200 as glq
    assert sorted(glq.EXPORTS) == syms


def test_status_strings(lib):
    import e8_lattice_codebook_b200 as glq
    for code, name in glq.STATUS.items():
        assert glq.glq_status_str(code) == name
    assert "sm_100a" in glq.glq_version()


def test_codebook_matches_oracle():
    import e8_lattice_codebook_b200 as glq
    from oracle import glq_oracle as orc
    ours = glq.glq_e8_codebook()
    ref = orc.e8_codebook().astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_codebook_upload_rejects_bad_tables_before_cuda():
    import e8_lattice_codebook_b200 as glq
    with pytest.raises(glq.GlqError) as e:
        glq.glq_codebook_upload(np.zeros((65536, 7), np.uint16))
    assert e.value.status == 2  # SHAPE
    with pytest.raises(glq.GlqError) as e:
        glq.glq_codebook_upload(np.zeros((100, 8), np.uint16))
    assert e.value.status == 2
    bad = glq.glq_e8_codebook().copy()
    bad[5, 3] = 0x7C00  # +inf
    with pytest.raises(glq.GlqError) as e:
        glq.glq_codebook_upload(bad)
    assert e.value.status == 1  # INVALID_ARG
    bad = glq.glq_e8_codebook().copy()
    bad[7, 0] = np.float16(0.25).view(np.uint16)  # not a multiple of 1/2
    with pytest.raises(glq.GlqError) as e:
        glq.glq_codebook_upload(bad)
    assert e.value.status == 10  # UNSUPPORTED
    dup = glq.glq_e8_codebook().copy()
    dup[9] = dup[8]
    with pytest.raises(glq.GlqError) as e:
        glq.glq_codebook_upload(dup)
    assert e.value.status == 10


def test_layer_create_argument_errors_before_cuda(lib):
    vp = ctypes.c_void_p
    f = lib.glq_layer_create
    f.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, vp, vp, vp, vp,
                  ctypes.c_float, ctypes.c_float, vp, vp, ctypes.POINTER(vp)]
    f.restype = ctypes.c_int
    h = vp()
    idx = np.zeros(64, np.uint16)
    s = np.ones(64, np.int8)
    p = idx.ctypes.data
    ps = s.ctypes.data
    assert f(0, 16, 2, p, None, None, None, 1.0, 0.0, ps, ps, ctypes.byref(h)) == 2
    assert f(16, 12, 2, p, None, None, None, 1.0, 0.0, ps, ps, ctypes.byref(h)) == 2
    assert f(16, 16, 5, p, None, None, None, 1.0, 0.0, ps, ps, ctypes.byref(h)) == 4
    assert f(16, 16, 2, None, None, None, None, 1.0, 0.0, ps, ps, ctypes.byref(h)) == 1
    assert f(16, 16, 2, p, None, None, None, 1.0, 0.0, ps, ps, ctypes.byref(h)) == 5  # no codebook
    assert f(16, 16, 2, p, None, None, None, 1.0, 0.0, ps, ps, None) == 1
    assert f(65536, 16, 2, p, None, None, None, 1.0, 0.0, ps, ps, ctypes.byref(h)) == 2


def test_linear_argument_errors_before_cuda(lib):
    f = lib.glq_linear
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                  ctypes.c_int64, ctypes.c_void_p]
    f.restype = ctypes.c_int
    assert f(None, None, 0, None, 0, 1, None) == 1
    assert lib.glq_layer_destroy(None) == 1
    assert lib.glq_codebook_destroy(None) == 1
