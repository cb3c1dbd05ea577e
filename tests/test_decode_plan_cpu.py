"""Host-side checks of the decode GEMV's work planner (plan_gemv in
e8_lattice_codebook_b200/csrc/glq_gemv.cu), without a GPU.

A small host program includes that source and answers planner queries on
stdin with the library's own function.  The checks:

* on every decode workload shape, for the warp counts, modes and caps the
  library uses: one band per `warps` row tiles, every split non-empty,
  power-of-two chunk counts when asked (the fused input transform needs
  aligned ranges), the caps honoured, the grid min(tasks, SMs);
* at 9-16 tokens (two token tiles, 16-warp CTAs, split tasks charged two
  chunks) the 32768 x 5120 layers take one split on 128 CTAs: with the
  one-tile charge of half a chunk the planner splits them 8 ways over
  148 CTAs, which measured 1.6x slower per 24B-class step;
* the SmolLM3-3B gate layer at one token with the fused input transform
  (aligned ranges) takes 29 bands x 4 splits on 116 CTAs.
"""
import math
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "e8_lattice_codebook_b200", "csrc")
sys.path.insert(0, ROOT)
import glq_inputs as gi  # noqa: E402

ROW_TILE, CHUNK_K = 16, 128  # rows per tile, columns per chunk (the layer's padding units)
SMS = 148
BIG = 1 << 30

HARNESS = r"""
#include "glq_gemv.cu"
#include <cstdio>

int main() {
    int RT, KC, sms, warps, pow2, max_cps, max_splits;
    double charge;
    while (std::scanf("%d %d %d %d %d %d %d %lf", &RT, &KC, &sms, &warps, &pow2, &max_cps, &max_splits,
                      &charge) == 8) {
        const glq::GemvPlan pl = glq::plan_gemv(RT, KC, sms, warps, pow2 != 0, max_cps, max_splits, charge);
        std::printf("%d %d %d %d\n", pl.bands, pl.splits, pl.cps, pl.grid);
    }
    return 0;
}
"""


@pytest.fixture(scope="module")
def planner(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("plan")
    src, exe = d / "plan.cu", d / "plan"
    src.write_text(HARNESS)
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    str(src), "-o", str(exe)], check=True, capture_output=True, timeout=600)

    def plan(queries):
        text = "".join(f"{rt} {kc} {sms} {w} {int(p2)} {mc} {ms} {ch}\n" for rt, kc, sms, w, p2, mc, ms, ch in queries)
        out = subprocess.run([str(exe)], input=text, capture_output=True, text=True, timeout=120, check=True)
        return [tuple(int(v) for v in line.split()) for line in out.stdout.splitlines()]

    return plan


def shape(m, n):
    return math.ceil(m / ROW_TILE), math.ceil(n / CHUNK_K)  # RT, KC


def decode_shapes():
    out = set()
    for wl in gi.WORKLOADS.values():
        if min(wl.batches) > 16:
            continue
        for spec in wl.layers:
            out.add(shape(spec.m, spec.n))
    return sorted(out)


def test_plans_are_valid_on_every_decode_shape(planner):
    queries = []
    for rt, kc in decode_shapes():
        for warps in (24, 16, 28):
            for pow2 in (False, True):
                for max_cps, max_splits in ((BIG, BIG), (4, BIG), (BIG, 8), (8, 16)):
                    for charge in (0.5, 2.0):
                        queries.append((rt, kc, SMS, warps, pow2, max_cps, max_splits, charge))
    plans = planner(queries)
    assert len(plans) == len(queries)
    for (rt, kc, sms, warps, pow2, max_cps, max_splits, charge), (bands, splits, cps, grid) in zip(queries, plans):
        q = (rt, kc, warps, pow2, max_cps, max_splits, charge)
        assert bands == math.ceil(rt / warps), q
        assert cps >= 1 and splits == math.ceil(kc / cps), (q, splits, cps)
        assert (splits - 1) * cps < kc, (q, splits, cps)  # no empty split
        if pow2:
            assert cps & (cps - 1) == 0, (q, cps)
        # the caps hold whenever some chunk count satisfies both
        feasible = any(
            c <= max_cps and math.ceil(kc / c) <= max_splits and (not pow2 or c & (c - 1) == 0)
            for c in range(1, 2 * kc + 1))
        if feasible:
            assert cps <= max_cps and splits <= max_splits, (q, splits, cps)
        assert grid == min(bands * splits, sms), (q, grid)


def test_two_token_tile_plan_of_the_32768_row_layers(planner):
    rt, kc = shape(32768, 5120)
    charged, light = planner([(rt, kc, SMS, 16, False, BIG, BIG, 2.0), (rt, kc, SMS, 16, False, BIG, BIG, 0.5)])
    assert charged == (128, 1, kc, 128)
    assert light[1] > 1 and light[3] == SMS  # what the one-tile charge would choose


def test_fused_one_token_plan_of_the_3b_gate_layer(planner):
    rt, kc = shape(11008, 2048)
    (plan,) = planner([(rt, kc, SMS, 24, True, BIG, BIG, 0.5)])
    assert plan == (29, 4, 4, 116)
