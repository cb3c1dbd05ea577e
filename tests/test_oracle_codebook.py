"""Pins for the oracle's E8 shell codebook (CPU only).

What fixes the codebook, independently of the oracle's own enumeration:
  * E8 membership: all-integer or all-half-integer coordinates, even sum;
  * the E8 theta series 1 + 240 sum sigma_3(k) q^k (Conway & Sloane, the
    reference the glq 0.5.1 PyPI page's acknowledgments cite) gives the
    shell sizes; 65,536 = the 56,881 points of norm <= 10 + 8,655 of the
    60,480 norm-12 points;
  * the build's ordering rule (squared norm, then x0..x7 ascending), checked
    as a property plus hand-derived entries in tests/golden;
  * the truncated seventh shell keeps exactly the lexicographically smallest
    norm-12 points, checked against a brute-force enumeration of that shell.
"""
import os

import numpy as np
import pytest

from oracle import glq_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sigma3(k):
    return sum(d ** 3 for d in range(1, k + 1) if k % d == 0)


@pytest.fixture(scope="module")
def cb():
    return orc.e8_codebook()


def test_theta_series_shell_counts():
    pts, total = orc.e8_points(12)
    norms = (pts ** 2).sum(axis=1)
    for k in range(0, 7):
        expected = 1 if k == 0 else 240 * sigma3(k)
        assert int(np.sum(norms == 2 * k)) == expected, k
    assert total == 1 + sum(240 * sigma3(k) for k in range(1, 7))
    # smaller radius enumerations are prefixes of the full one
    small, t8 = orc.e8_points(8)
    assert t8 == 1 + sum(240 * sigma3(k) for k in range(1, 5))
    np.testing.assert_array_equal(small, pts[:t8])


def test_membership(cb):
    assert cb.shape == (65536, 8)
    y = 2 * cb
    assert np.all(y == np.round(y))
    y = y.astype(np.int64)
    parity = y % 2
    assert np.all((parity == 0).all(1) | (parity == 1).all(1))
    assert np.all(y.sum(1) % 4 == 0)  # sum(x) even
    assert np.all((cb ** 2).sum(1) <= 12)


def test_bijection_and_order(cb):
    y = (2 * cb).astype(np.int64)
    assert len({tuple(r) for r in y}) == 65536
    keys = np.concatenate([(y ** 2).sum(1, keepdims=True), y], axis=1)
    # sorted by (norm, x0, ..., x7); distinct keys make the order strict
    order = np.lexsort(keys[:, ::-1].T)
    np.testing.assert_array_equal(order, np.arange(65536))


def test_shell_composition(cb):
    norms = (cb ** 2).sum(1)
    assert int(np.sum(norms <= 10)) == 56881
    assert int(np.sum(norms == 12)) == 65536 - 56881 == 8655
    assert np.abs(cb).max() == 3.0


def test_golden_entries(cb):
    with open(os.path.join(GOLDEN, "e8_codebook_entries.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    assert rows
    for r in rows:
        idx = int(r[0])
        expect = np.array([float(v) for v in r[1:9]])
        np.testing.assert_array_equal(cb[idx], expect)


def test_negation_symmetry_of_full_shells(cb):
    # every full shell is closed under negation, and negation reverses
    # lexicographic order, so entry i of a full shell mirrors its last-i
    bounds = [0, 1, 241, 2401, 9121, 26641, 56881]
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        np.testing.assert_array_equal(cb[lo:hi], -cb[lo:hi][::-1])


def test_truncated_shell_is_lexicographic_prefix(cb):
    # brute-force enumeration of the whole norm-12 shell, independent of the
    # oracle's C enumeration, then check the codebook keeps its smallest 8655
    shell = []
    for parity in (0, 1):
        vals = np.arange(-6, 7, 2) if parity == 0 else np.arange(-5, 6, 2)
        grids = np.stack(np.meshgrid(*([vals] * 8), indexing="ij"), -1).reshape(-1, 8)
        keep = ((grids ** 2).sum(1) == 48) & (grids.sum(1) % 4 == 0)
        shell.append(grids[keep])
    shell = np.concatenate(shell)
    assert shell.shape[0] == 240 * sigma3(6)
    order = np.lexsort(shell[:, ::-1].T)
    smallest = shell[order[:8655]]
    np.testing.assert_array_equal((2 * cb[56881:]).astype(np.int64), smallest)


def test_second_moment(cb):
    # mean squared coordinate, used to size the synthetic workloads
    # (sum over shells of count * norm / 8 / 65536)
    counts = {0: 1, 2: 240, 4: 2160, 6: 6720, 8: 17520, 10: 30240, 12: 8655}
    expect = sum(c * k for k, c in counts.items()) / 8 / 65536
    assert abs((cb ** 2).mean() - expect) < 1e-12
