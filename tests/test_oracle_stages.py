"""Pins for the oracle's multi-stage reconstruction (5-8 bpw; glq 0.5.1 PyPI
page, "Bit widths": 16 b primary plus 16 b / 8 b residual stages), CPU only.

Independent of the oracle's code:
  * the stage structure of every bit width against the pages' table
    (tests/golden/bit_widths.txt), and the rate: exactly bpw bits per weight;
  * exact rational arithmetic (fractions) for the stage-by-stage single
    roundings c = fp32(rs_s cb_s + c), w = fp32(ws c), with the default
    power-of-two scales and with scales that force roundings, including a
    case whose result changes if the 8-bit stage were added before the 16-bit
    ones;
  * reductions that must hold exactly: a zero 8-bit table turns 5 (7) bpw
    into 4 (6) bpw, residual indices of the origin turn 8 bpw into 2 bpw;
  * brute force on tiny layers: W^ rebuilt here with fractions, H from the
    Sylvester recursion, numpy matmul.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import glq_inputs as gi
from oracle import glq_oracle as orc
from test_oracle_hadamard import blockdiag_sylvester
from test_oracle_linear import round_to_f32

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "bit_widths.txt")


def golden_stages():
    table = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                v = [int(t) for t in line.split()]
                table[v[0]] = v[1:]
    return table


def test_stage_structure_matches_the_pages_table():
    table = golden_stages()
    assert sorted(table) == list(range(2, 9))
    for bpw, widths in table.items():
        assert widths[0] == 16
        assert orc.stage_bits(bpw) == widths[1:], bpw
        assert gi.stage_bits(bpw) == widths[1:], bpw
        assert sum(widths) == 8 * bpw  # bpw bits per weight, 8 weights per group
    with pytest.raises(ValueError):
        orc.stage_bits(9)


@pytest.mark.parametrize("bpw", [5, 6, 7, 8])
def test_rate(bpw):
    L = gi.make_layer(1, 0, 24, 64, bpw)
    res, _ = L.stages()
    total = L.idx1.nbytes + sum(a.nbytes for a in res)
    assert total * 8 == bpw * L.m * L.n


def _exact_decode(L, scales=None):
    """W^ by exact rational arithmetic with one rounding per stage."""
    cb = orc.e8_codebook()
    res, rs = L.stages()
    rs = scales or rs
    bits = gi.stage_bits(L.bpw)
    cb8 = None if L.cb2_f16 is None else L.cb2_f16.view(np.float16).astype(np.float64)
    ws = Fraction(float(np.float32(L.weight_scale)))
    out = np.zeros((L.m, L.n))
    for r in range(L.m):
        for g in range(L.n // 8):
            for j in range(8):
                c = Fraction(float(cb[L.idx1[r, g], j]))
                for a, b, s in zip(res, bits, rs):
                    t = cb[a[r, g], j] if b == 16 else cb8[a[r, g], j]
                    c = Fraction(round_to_f32(Fraction(float(np.float32(s))) * Fraction(float(t)) + c))
                out[r, 8 * g + j] = round_to_f32(ws * c)
    return out


@pytest.mark.parametrize("bpw", [5, 6, 7, 8])
def test_decode_matches_exact_rational_rounding(bpw):
    L = gi.make_layer(21, 0, 3, 24, bpw)
    res, rs = L.stages()
    w = orc.decode_rows(L.m, L.n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, cb2=L.cb2_f16)
    np.testing.assert_array_equal(w, _exact_decode(L))
    # scales that are not powers of two: every stage rounds
    odd = [0.3, 0.0713, 0.00917][:len(res)]
    w2 = orc.decode_rows(L.m, L.n, bpw, L.idx1, L.idx2, L.weight_scale, odd, cb2=L.cb2_f16)
    np.testing.assert_array_equal(w2, _exact_decode(L, odd))


def test_stage_order_matters_and_is_the_tables():
    """5 bpw on one coordinate, ulp = 2^-23 (the spacing of fp32 at 1):
    primary x0 = 1; the 16-bit stage adds 1.5 ulp (codeword x0 = 1.5, scale
    2^-23): 1 + 1.5 ulp is a tie and rounds to the even 1 + 2 ulp; the 8-bit
    stage then adds 1 ulp (value 0.5, scale 2^-22): 1 + 3 ulp, exact.  Adding
    the 8-bit stage first would give 1 + 1 ulp, then 1 + 2.5 ulp, a tie that
    rounds to 1 + 2 ulp.  The oracle must give the table order's 1 + 3 ulp."""
    cb = orc.e8_codebook()
    i1 = int(np.flatnonzero(cb[:, 0] == 1.0)[0])
    i2 = int(np.flatnonzero(cb[:, 0] == 1.5)[0])
    cb8 = np.zeros((256, 8), dtype=np.float16)
    cb8[0, 0] = 0.5
    idx1 = np.array([[i1]], dtype=np.uint16)
    idx_a = np.array([[i2]], dtype=np.uint16)
    idx_b = np.zeros((1, 1), dtype=np.uint8)
    rs = [2.0 ** -23, 2.0 ** -22]
    w = orc.decode_rows(1, 8, 5, idx1, [idx_a, idx_b], 1.0, rs, cb2=cb8.view(np.uint16))
    ulp = 2.0 ** -23
    table_order = round_to_f32(Fraction(round_to_f32(Fraction(1) + Fraction(1.5 * ulp))) + Fraction(ulp))
    reversed_order = round_to_f32(Fraction(round_to_f32(Fraction(1) + Fraction(ulp))) + Fraction(1.5 * ulp))
    assert table_order == 1 + 3 * ulp and reversed_order == 1 + 2 * ulp
    assert w[0, 0] == table_order


@pytest.mark.parametrize("lo,hi", [(4, 5), (6, 7)])
def test_zero_eight_bit_table_reduces_to_the_even_rate(lo, hi):
    Lh = gi.make_layer(5, 0, 16, 40, hi)
    res, rs = Lh.stages()
    zero = np.zeros((256, 8), dtype=np.float16).view(np.uint16)
    wh = orc.decode_rows(16, 40, hi, Lh.idx1, Lh.idx2, Lh.weight_scale, Lh.resid_scale, cb2=zero)
    if lo == 4:
        wl = orc.decode_rows(16, 40, 4, Lh.idx1, res[0], Lh.weight_scale, rs[0])
    else:
        wl = orc.decode_rows(16, 40, 6, Lh.idx1, res[:-1], Lh.weight_scale, rs[:-1])
    np.testing.assert_array_equal(wh, wl)


def test_origin_residuals_reduce_eight_to_two_bpw():
    L8 = gi.make_layer(6, 0, 8, 32, 8)
    zeros = [np.zeros_like(a) for a in L8.stages()[0]]  # index 0 is the origin
    w8 = orc.decode_rows(8, 32, 8, L8.idx1, zeros, L8.weight_scale, L8.resid_scale)
    w2 = orc.decode_rows(8, 32, 2, L8.idx1, None, L8.weight_scale, 0.0)
    np.testing.assert_array_equal(w8, w2)
    xb = gi.make_x(6, 0, 2, 32, "bf16")
    y8 = orc.linear(8, 32, 8, L8.idx1, zeros, L8.weight_scale, L8.resid_scale, L8.s_in, L8.s_out, xb, True)
    y2 = orc.linear(8, 32, 2, L8.idx1, None, L8.weight_scale, 0.0, L8.s_in, L8.s_out, xb, True)
    np.testing.assert_array_equal(y8, y2)


@pytest.mark.parametrize("m,n,bpw", [(8, 16, 5), (16, 24, 6), (24, 8, 7), (8, 40, 8)])
def test_brute_force_tiny(m, n, bpw):
    L = gi.make_layer(m + 7 * n, 2, m, n, bpw)
    xb = gi.make_x(m + 7 * n, 2, 3, n, "bf16")
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    W = _exact_decode(L)
    Hn, Hm = blockdiag_sylvester(n), blockdiag_sylvester(m)
    ref = (((xf * L.s_in) @ Hn.T) @ W.T @ Hm.T) * L.s_out
    y = orc.linear(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb, True,
                   cb2=L.cb2_f16)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)
