"""Host-side checks of the tensor-core GEMM's work split (plan_prefill in
e8_lattice_codebook_b200/csrc/glq_prefill.cu, the function glq_linear's
prefill path and its workspace sizing call), without a GPU.

A small host program includes that source and answers planner queries on
stdin with the library's own function.  The checks:

* every (row tile, token tile, K split) is covered exactly once by the
  items (whole tiles first, then two halves per remaining tile), the K
  splits are at most 8 and leave every split at least four chunks;
* half tiles only for a last partial wave of at most half the CTA pairs,
  without a K split, and only when every halved tile has two live halves
  (a ragged last token tile of at most 256 tokens keeps whole tiles);
* the schedules of the 8B-class MLP layers on 148 SMs that the measurements
  were taken on: 14336 x 4096 at 512 / 2048 / 8192 tokens is 56 whole tiles
  / 222 whole tiles and 4 halves / 888 whole tiles and 16 halves; 4096 x
  14336 splits K four ways at 512 tokens (64 items), takes one split at
  2048 (64 tiles) and two at 8192 (512 items, so no halves).
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "e8_lattice_codebook_b200", "csrc")

ROW_TILE, TOK_TILE, CHUNK_K, SMS = 256, 512, 128, 148

HARNESS = r"""
#include "glq_prefill.cu"
#include <cstdio>

int main() {
    long long m_pad, B;
    int KC, sms;
    while (std::scanf("%lld %d %lld %d", &m_pad, &KC, &B, &sms) == 4) {
        const glq::PrefillSplit ps = glq::plan_prefill(m_pad, KC, B, sms);
        std::printf("%d %d %d %d\n", ps.ksplit, ps.tiles_tok, ps.ntiles, ps.tiles_whole);
    }
    return 0;
}
"""


@pytest.fixture(scope="module")
def planner(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("pplan")
    src, exe = d / "pplan.cu", d / "pplan"
    src.write_text(HARNESS)
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
                    "--expt-relaxed-constexpr", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True, capture_output=True, timeout=600)

    def ask(queries):
        text = "".join(f"{m_pad} {kc} {b} {sms}\n" for m_pad, kc, b, sms in queries)
        out = subprocess.run([str(exe)], input=text, capture_output=True, text=True, timeout=120,
                             check=True).stdout
        return [tuple(int(v) for v in line.split()) for line in out.strip().splitlines()]

    return ask


def pad(v, unit):
    return (v + unit - 1) // unit * unit


def test_documented_schedules(planner):
    # (m, n, B) -> (ksplit, items, whole items)
    want = {
        (14336, 4096, 512): (1, 56, 56),
        (14336, 4096, 2048): (1, 226, 222),
        (14336, 4096, 8192): (1, 904, 888),
        (4096, 14336, 512): (4, 64, 64),
        (4096, 14336, 2048): (1, 64, 64),
        (4096, 14336, 8192): (2, 512, 512),
    }
    keys = list(want)
    got = planner([(pad(m, 16), pad(n, CHUNK_K) // CHUNK_K, B, SMS) for m, n, B in keys])
    for k, (ks, tt, nt, tw) in zip(keys, got):
        assert (ks, nt, tw) == want[k], (k, ks, nt, tw)
        assert tt == (k[2] + TOK_TILE - 1) // TOK_TILE


SHAPES = [(16, 2), (272, 3), (1000, 8), (14336, 32), (4096, 112), (19200, 2), (20480, 1), (8, 1),
          (11008, 16), (5120, 256), (32768, 40)]
BATCHES = [17, 100, 256, 257, 300, 511, 512, 513, 600, 768, 769, 1100, 2048, 2300, 4096, 8192, 8300]


def test_items_cover_every_tile_once(planner):
    queries = [(pad(m, 16), kc, B, sms) for m, kc in SHAPES for B in BATCHES for sms in (SMS, 132, 8, 2)]
    for (m_pad, kc, B, sms), (ks, tt, nt, tw) in zip(queries, planner(queries)):
        tiles_m = (m_pad + ROW_TILE - 1) // ROW_TILE
        assert tt == (B + TOK_TILE - 1) // TOK_TILE
        assert 1 <= ks <= 8 and (ks == 1 or ks <= kc // 4), (m_pad, kc, B, ks)
        total = tiles_m * tt * ks
        assert 0 <= tw <= total and nt == tw + 2 * (total - tw), (m_pad, kc, B, ks, nt, tw)
        # the items' (tile, half) pairs, as the kernel's geometry maps them
        seen = {}
        for item in range(nt):
            if item < tw:
                tile, halves = item, (0, 1)
            else:
                u = item - tw
                tile, halves = tw + (u >> 1), ((u & 1),)
            for h in halves:
                seen[(tile, h)] = seen.get((tile, h), 0) + 1
        assert all(seen.get((t, h), 0) == 1 for t in range(total) for h in (0, 1)), (m_pad, kc, B)
        pairs = max(1, sms // 2)
        if tw < total:  # halves: only a short last wave, no K split, two live halves per tile
            rest = total - tw
            assert ks == 1 and total > pairs and rest == total % pairs and 2 * rest <= pairs, (m_pad, kc, B)
            assert B % TOK_TILE == 0 or B % TOK_TILE > TOK_TILE // 2, (m_pad, kc, B)


def test_ragged_last_token_tile_keeps_whole_tiles(planner):
    # 75 row tiles for 74 pairs.  At 512 tokens the 75th tile runs as two
    # halves; at 600 (a last token tile of 88 tokens) nothing is halved, a
    # halved tile there would have an empty upper half; at 800 (288 tokens
    # in the last token tile) the partial wave is halved.
    got = planner([(19200, 2, 512, SMS), (19200, 2, 600, SMS), (19200, 2, 800, SMS)])
    assert got[0] == (1, 1, 76, 74)     # 75 tiles: 74 whole, the last as two halves
    assert got[1] == (1, 2, 150, 150)   # 150 tiles (2 waves + 2): the last token tile is ragged
    assert got[2][3] < got[2][2]        # 800 tokens: 288 in the last tile, halves allowed
