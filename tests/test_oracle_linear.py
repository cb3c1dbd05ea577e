"""Pins for the oracle's codeword reconstruction and the full layer
y = S_out . H_m . W^ . H_n . (S_in . x) (CPU only).

Independent of the oracle's arithmetic:
  * a closed form worked by hand (one-hot x, all-plus signs, constant
    codeword rows) -- catches wrong normalisation, wrong sign/H order;
  * brute force on tiny shapes: W^ rebuilt here with numpy float32
    arithmetic from the (separately pinned) codebook, H from the Sylvester
    recursion with numpy.kron, numpy matmul;
  * exact rational arithmetic (fractions) for the single-rounding residual
    reconstruction, including a case where two roundings would differ;
  * structural invariants: zero codewords give y = 0, linearity in x,
    flipping S_in[j] is negating x[:, j], flipping S_out[r] negates y[:, r];
  * the 2 bpw rate: exactly one uint16 index per 8 weights.
"""
from fractions import Fraction

import numpy as np
import pytest

import glq_inputs as gi
from oracle import glq_oracle as orc
from test_oracle_hadamard import blockdiag_sylvester


def round_to_f32(q: Fraction) -> float:
    """Round an exact rational to the nearest binary32 (ties to even)."""
    if q == 0:
        return 0.0
    sign = -1 if q < 0 else 1
    q = abs(q)
    e = 0
    while q >= 2:
        q /= 2
        e += 1
    while q < 1:
        q *= 2
        e -= 1
    scaled = q * (1 << 23)  # 24 significant bits (normal range only)
    fl = scaled.numerator // scaled.denominator
    rem = scaled - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * float(Fraction(fl, 1 << 23) * Fraction(2) ** e)


def f16_bits(v):
    return np.array(v, dtype=np.float16).view(np.uint16)


def test_single_rounding_residual_reconstruction():
    # c = fma(rs, cb2, cb1) rounded once; two roundings would give 2 + 2^-10
    rs = np.float32(1 + 2.0 ** -23)
    cb2 = np.array([[1 + 2.0 ** -10] + [0.0] * 7] * 256, dtype=np.float16)
    idx1 = np.zeros((1, 1), dtype=np.uint16)
    cb = orc.e8_codebook()
    # any codeword whose x0 is 1 works; take the first one
    idx1[0, 0] = int(np.flatnonzero(cb[:, 0] == 1.0)[0])
    c1 = cb[idx1[0, 0]]
    idx2 = np.zeros((1, 1), dtype=np.uint8)
    w = orc.decode_rows(1, 8, 3, idx1, idx2, 1.0, float(rs), cb2=cb2.view(np.uint16))
    exact = Fraction(float(rs)) * Fraction(float(cb2[0, 0])) + Fraction(float(c1[0]))
    assert w[0, 0] == round_to_f32(exact) == 2 + 2.0 ** -10 + 2.0 ** -22
    # the remaining coordinates: cb1 + rs * 0 = cb1, times ws = 1
    np.testing.assert_array_equal(w[0, 1:], c1[1:])


@pytest.mark.parametrize("bpw", [2, 3, 4])
def test_decode_matches_exact_rational_rounding(bpw):
    L = gi.make_layer(11, 0, 4, 32, bpw, weight_scale=0.05, resid_scale=0.125)
    w = orc.decode_rows(L.m, L.n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale,
                        cb2=L.cb2_f16)
    cb = orc.e8_codebook()
    cb2 = None
    if bpw == 3:
        cb2 = L.cb2_f16.view(np.float16).astype(np.float64)
    ws = Fraction(float(np.float32(L.weight_scale)))
    rs = Fraction(float(np.float32(L.resid_scale)))
    for r in range(L.m):
        for g in range(L.n // 8):
            for j in range(8):
                c = Fraction(float(cb[L.idx1[r, g], j]))
                if bpw == 4:
                    c = Fraction(round_to_f32(rs * Fraction(float(cb[L.idx2[r, g], j])) + c))
                elif bpw == 3:
                    c = Fraction(round_to_f32(rs * Fraction(float(cb2[L.idx2[r, g], j])) + c))
                assert w[r, 8 * g + j] == round_to_f32(ws * c)


def test_closed_form_one_hot():
    # m = n = 8, every row's codeword = index 1 = (-1,-1,0,...,0), signs +1,
    # x = e_0:  H_8 e_0 = (1/sqrt 8) 1,  z_r = -2 w / sqrt 8 for all r,
    # H_8 z = sqrt 8 * z_0 e_0, so y = (-2 w, 0, ..., 0) with w = fp32(0.05).
    m = n = 8
    idx1 = np.ones((m, 1), dtype=np.uint16)
    s = np.ones(8, dtype=np.int8)
    x = np.zeros((1, n), dtype=np.float16)
    x[0, 0] = 1.0
    y = orc.linear(m, n, 2, idx1, None, 0.05, 0.0, s, s, x.view(np.uint16), False)
    w = float(np.float32(0.05))
    expect = np.zeros((1, 8))
    expect[0, 0] = -2 * w
    np.testing.assert_allclose(y, expect, rtol=0, atol=1e-15)


def test_zero_codewords_give_zero():
    L = gi.make_layer(3, 0, 24, 40, 2)
    idx1 = np.zeros_like(L.idx1)  # index 0 is the origin
    x = gi.make_x(3, 0, 3, 40, "f16")
    y = orc.linear(24, 40, 2, idx1, None, 0.05, 0.0, L.s_in, L.s_out, x, False)
    assert np.all(y == 0)


def _brute_force(L, x_f64):
    cb = orc.e8_codebook()
    G = L.n // 8
    c = cb[L.idx1.reshape(-1)].reshape(L.m, G, 8).astype(np.float32)
    if L.bpw == 4:
        c2 = cb[L.idx2.reshape(-1)].reshape(L.m, G, 8)
    elif L.bpw == 3:
        c2 = L.cb2_f16.view(np.float16).astype(np.float64)[L.idx2.reshape(-1)].reshape(L.m, G, 8)
    if L.bpw in (3, 4):
        # exact in float64 here (rs = 1/8, fp16 residuals), then one rounding
        c = (c.astype(np.float64) + L.resid_scale * c2).astype(np.float32)
    W = (np.float32(L.weight_scale) * c).reshape(L.m, L.n).astype(np.float64)
    Hn, Hm = blockdiag_sylvester(L.n), blockdiag_sylvester(L.m)
    xr = (x_f64 * L.s_in) @ Hn.T
    return (xr @ W.T @ Hm.T) * L.s_out


@pytest.mark.parametrize("m,n,bpw,xdt", [
    (8, 8, 2, "f16"), (16, 16, 4, "bf16"), (24, 16, 3, "f16"),
    (16, 24, 4, "f16"), (72, 64, 3, "bf16"), (56, 40, 2, "bf16")])
def test_brute_force_tiny(m, n, bpw, xdt):
    L = gi.make_layer(m * 100 + n, 1, m, n, bpw)
    xb = gi.make_x(m * 100 + n, 1, 3, n, xdt)
    if xdt == "f16":
        xf = xb.view(np.float16).astype(np.float64)
    else:
        xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y = orc.linear(m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out,
                   xb, xdt == "bf16", cb2=L.cb2_f16)
    np.testing.assert_allclose(y, _brute_force(L, xf), rtol=0, atol=1e-12)


def test_linearity_and_signs():
    m, n = 40, 48
    L = gi.make_layer(5, 0, m, n, 4)
    rng = np.random.default_rng(0)
    a = rng.integers(-8, 8, size=(2, n)).astype(np.float16)
    b = rng.integers(-8, 8, size=(2, n)).astype(np.float16)
    ab = (a + b).astype(np.float16)  # exact: small integers
    run = lambda xx, si=L.s_in, so=L.s_out: orc.linear(
        m, n, 4, L.idx1, L.idx2, L.weight_scale, L.resid_scale, si, so, xx.view(np.uint16), False)
    np.testing.assert_allclose(run(ab), run(a) + run(b), rtol=0, atol=1e-11)
    si = L.s_in.copy()
    si[5] = -si[5]
    a_neg = a.copy()
    a_neg[:, 5] = -a_neg[:, 5]
    np.testing.assert_allclose(run(a, si=si), run(a_neg), rtol=0, atol=1e-12)
    so = L.s_out.copy()
    so[7] = -so[7]
    y0, y1 = run(a), run(a, so=so)
    np.testing.assert_array_equal(y1[:, 7], -y0[:, 7])
    np.testing.assert_array_equal(np.delete(y1, 7, 1), np.delete(y0, 7, 1))


def test_empty_batch():
    L = gi.make_layer(1, 0, 16, 16, 2)
    y = orc.linear(16, 16, 2, L.idx1, None, 0.05, 0.0, L.s_in, L.s_out,
                   np.zeros((0, 16), np.uint16), False)
    assert y.shape == (0, 16)


def test_two_bpw_rate():
    # one uint16 index per 8 weights: index bytes = m * n / 4
    for m, n in [(1024, 1024), (960, 2560)]:
        L = gi.make_layer(0, 0, m, n, 2)
        assert L.idx2 is None
        assert L.idx1.nbytes * 8 == 2 * m * n


@pytest.mark.parametrize("m,n,bpw,B,threads", [(37, 64, 4, 3, 4), (200, 136, 3, 2, 7), (8, 8, 2, 1, 16)])
def test_threaded_oracle_is_bitwise_single_threaded(m, n, bpw, B, threads):
    """The rows of W^ xr dealt out to POSIX threads give the same bits as the
    single-threaded loop (each output element is computed by the same code);
    more threads than rows are capped."""
    L = gi.make_layer(m + n + bpw, 4, m, n, bpw)
    xb = gi.make_x(m + n + bpw, 4, B, n, "bf16")
    args = (m, n, bpw, L.idx1, L.idx2, L.weight_scale, L.resid_scale, L.s_in, L.s_out, xb, True)
    y1 = orc.linear(*args, cb2=L.cb2_f16)
    yt = orc.linear(*args, cb2=L.cb2_f16, threads=threads)
    assert np.array_equal(y1, yt)
