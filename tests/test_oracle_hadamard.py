"""Pins for the oracle's normalised block-diagonal Walsh-Hadamard transform
and its binary16 / bfloat16 decoders (CPU only).

Fixed independently of the oracle: hand-written H_2 / H_4 and the page's
printed block decomposition of 2688 (tests/golden/hadamard_small.txt), the
Sylvester recursion H_2k = [[H_k, H_k], [H_k, -H_k]] built here with
numpy.kron, orthogonality H H^T = I, norm preservation, H^2 = I (H is
symmetric), and numpy's own IEEE binary16 conversion.
"""
import os

import numpy as np
import pytest

from oracle import glq_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# every size the synthetic workloads use, plus small mixed decompositions
WORKLOAD_SIZES = [960, 1024, 2048, 2560, 4096, 5120, 11008, 14336, 32768]


def _golden():
    mats, blocks, cur, name = {}, {}, None, None
    with open(os.path.join(GOLDEN, "hadamard_small.txt")) as f:
        for ln in f:
            ln = ln.strip()
            if not ln or ln.startswith("#"):
                continue
            if ln.startswith("H"):
                name, cur = ln, []
                mats[name] = cur
            elif ln.startswith("BLOCKS"):
                name, cur = int(ln.split()[1]), None
            elif cur is not None:
                cur.append([int(v) for v in ln.split()])
            else:
                blocks[name] = [int(v) for v in ln.split()]
    return {k: np.array(v, dtype=np.float64) for k, v in mats.items()}, blocks


def sylvester(k):
    h = np.array([[1.0]])
    while h.shape[0] < k:
        h = np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), h)
    return h


def blockdiag_sylvester(n):
    sizes = [1 << b for b in range(62, -1, -1) if n & (1 << b)]
    H = np.zeros((n, n))
    off = 0
    for k in sizes:
        H[off:off + k, off:off + k] = sylvester(k) / np.sqrt(k)
        off += k
    return H


def test_golden_small_matrices():
    mats, blocks = _golden()
    np.testing.assert_allclose(orc.hadamard_matrix(2), mats["H2"] / np.sqrt(2), rtol=0, atol=1e-15)
    np.testing.assert_allclose(orc.hadamard_matrix(4), mats["H4"] / 2.0, rtol=0, atol=1e-15)
    for n, expect in blocks.items():
        assert orc.hadamard_blocks(n) == expect


def test_block_decompositions_of_workload_sizes():
    expect = {960: [512, 256, 128, 64], 1024: [1024], 2560: [2048, 512],
              5120: [4096, 1024], 11008: [8192, 2048, 512, 256],
              14336: [8192, 4096, 2048], 32768: [32768]}
    for n, blocks in expect.items():
        assert orc.hadamard_blocks(n) == blocks
        assert sum(blocks) == n


@pytest.mark.parametrize("n", [1, 2, 8, 24, 56, 64, 72, 960, 1024])
def test_dense_matrix_matches_sylvester_recursion(n):
    H = orc.hadamard_matrix(n)
    np.testing.assert_allclose(H, blockdiag_sylvester(n), rtol=0, atol=1e-15)
    np.testing.assert_allclose(H @ H.T, np.eye(n), rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [8, 24, 56, 64, 200, 960])
def test_apply_equals_dense_matrix(n):
    rng = np.random.default_rng(n)
    v = rng.standard_normal(n)
    np.testing.assert_allclose(orc.hadamard_apply(v), orc.hadamard_matrix(n) @ v, rtol=0, atol=1e-12)


@pytest.mark.parametrize("k", [8192, 16384])
def test_kronecker_split_equals_dense_block(k):
    rng = np.random.default_rng(k)
    v = rng.standard_normal(k)
    fast = orc.hadamard_apply(v)
    dense = orc.hadamard_apply(v, force_dense=True)
    np.testing.assert_allclose(fast, dense, rtol=0, atol=1e-10)


@pytest.mark.parametrize("n", WORKLOAD_SIZES)
def test_orthogonal_involution_on_workload_sizes(n):
    rng = np.random.default_rng(n + 7)
    v = rng.standard_normal(n)
    hv = orc.hadamard_apply(v)
    assert abs(np.linalg.norm(hv) - np.linalg.norm(v)) < 1e-10 * np.linalg.norm(v)
    np.testing.assert_allclose(orc.hadamard_apply(hv), v, rtol=0, atol=1e-10)
    # a unit vector maps to one column of H: entries +-1/sqrt(k) inside its
    # block, zero elsewhere
    j = n - 1
    e = np.zeros(n)
    e[j] = 1.0
    col = orc.hadamard_apply(e)
    blocks = orc.hadamard_blocks(n)
    off = n - blocks[-1]
    k = blocks[-1]
    np.testing.assert_allclose(np.abs(col[off:]), 1 / np.sqrt(k), rtol=1e-14)
    assert np.all(col[:off] == 0)


def test_rht_preserves_norm():
    n = 5120
    rng = np.random.default_rng(1)
    s = rng.integers(0, 2, n) * 2 - 1
    x = rng.standard_normal(n)
    xr = orc.hadamard_apply(s * x)
    assert abs(np.linalg.norm(xr) - np.linalg.norm(x)) < 1e-10 * np.linalg.norm(x)


def test_f16_decoder_matches_numpy_on_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.f16_table_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(ref)
    np.testing.assert_array_equal(ours[finite], ref[finite])
    assert np.all(np.isnan(ours[np.isnan(ref)]))
    assert np.all(ours[np.isinf(ref)] == ref[np.isinf(ref)])


def test_scalar_decoders_textbook_values():
    assert orc.f16_bits_to_double(0x3C00) == 1.0
    assert orc.f16_bits_to_double(0xC000) == -2.0
    assert orc.f16_bits_to_double(0x7BFF) == 65504.0
    assert orc.f16_bits_to_double(0x0001) == 2.0 ** -24
    assert orc.f16_bits_to_double(0x3555) == 1365 / 4096  # 0.333251953125
    assert orc.bf16_bits_to_double(0x3F80) == 1.0
    assert orc.bf16_bits_to_double(0xC0A0) == -5.0
    assert orc.bf16_bits_to_double(0x3E80) == 0.25
