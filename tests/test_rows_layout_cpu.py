"""Host-side checks of the row-transform kernel's shared-memory layout
(e8_lattice_codebook_b200/csrc/glq_rht_rows.cu), without a GPU.

The layout functions of that file are constexpr host/device code, so a small
host program that includes the kernel source can evaluate exactly the
functions the kernels use.  For every row size 2^L (9 <= L <= 14) and every
butterfly phase it checks that

* (thread, register) -> position is a bijection onto [0, 2^L), with the
  thread's and the register's position bits disjoint;
* the padded word map word(p) = p + (p >> 5) is additive over those parts
  (every access is a per-thread base plus an immediate offset);
* the 32 lanes of a warp at one register index meet 32 distinct banks (the
  one exception by design: a two-way conflict in phase 1 at L = 9);
* phase 0 is the load layout (16 consecutive columns per thread), and the
  last phase's fill bits (the runs it stores to global memory) are clear in
  every thread's base;
* the row buffer holds every word.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "e8_lattice_codebook_b200", "csrc")

HARNESS = r"""
#include "glq_rht_rows.cu"
#include "glq_rht_mma.cu"  // the input side's tensor-core kernel, which glq_rht_rows.cu dispatches to
#include <cstdio>
#include <vector>

using namespace glq;

static uint32_t tpos_host(int L, int q, uint32_t t) {
    const TposRuns R = tpos_runs(L, q);
    uint32_t p = 0u;
    for (int i = 0; i < R.n; ++i) p |= ((t >> R.src[i]) & ((1u << R.len[i]) - 1u)) << R.dst[i];
    return p;
}

int main() {
    int fails = 0;
    for (int L = 9; L <= 14; ++L) {
        const int NPH = (L + 3) / 4, T = 1 << (L - 4);
        if (row_words(L) <= (int)word_of((1u << L) - 1u)) {
            std::printf("L=%d: row buffer too small\n", L);
            ++fails;
        }
        for (int q = 0; q < NPH; ++q) {
            std::vector<int> seen(1 << L, 0);
            const int fill = 4 - phase_na(L, q);
            for (int t = 0; t < T; ++t) {
                const uint32_t tp = tpos_host(L, q, (uint32_t)t);
                if (q == 0 && tp != 16u * (uint32_t)t) {
                    std::printf("L=%d phase 0: thread %d is not the load layout\n", L, t);
                    ++fails;
                }
                if (q == NPH - 1 && (tp & ((1u << fill) - 1u)) != 0u) {
                    std::printf("L=%d last phase: thread %d has fill bits set\n", L, t);
                    ++fails;
                }
                for (int j = 0; j < 16; ++j) {
                    const uint32_t jp = jpos(L, q, j);
                    const uint32_t p = tp | jp;
                    if ((tp & jp) != 0u || p >= (1u << L)) {
                        std::printf("L=%d phase %d: thread %d reg %d overlaps or leaves the row\n", L, q, t, j);
                        ++fails;
                        continue;
                    }
                    ++seen[p];
                    if (word_of(p) != word_of(tp) + word_of(jp)) {
                        std::printf("L=%d phase %d: word map not additive at %u\n", L, q, p);
                        ++fails;
                    }
                }
            }
            for (int p = 0; p < (1 << L); ++p)
                if (seen[p] != 1) {
                    std::printf("L=%d phase %d: position %d held %d times\n", L, q, p, seen[p]);
                    ++fails;
                    break;
                }
            const int allowed = (L == 9 && q == 1) ? 2 : 1;
            int worst = 0;
            for (int w = 0; w < T / 32; ++w)
                for (int j = 0; j < 16; ++j) {
                    int count[32] = {0};
                    for (int l = 0; l < 32; ++l) {
                        const uint32_t p = tpos_host(L, q, (uint32_t)(32 * w + l)) | jpos(L, q, j);
                        const int c = ++count[word_of(p) & 31u];
                        worst = c > worst ? c : worst;
                    }
                }
            if (worst != allowed) {
                std::printf("L=%d phase %d: bank depth %d, expected %d\n", L, q, worst, allowed);
                ++fails;
            }
        }
    }
    std::printf(fails ? "FAILED %d\n" : "OK\n", fails);
    return fails ? 1 : 0;
}
"""


def test_row_transform_layout(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "rows_layout.cu"
    src.write_text(HARNESS)
    exe = tmp_path / "rows_layout"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    str(src), "-o", str(exe)], check=True, capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), out.stdout
