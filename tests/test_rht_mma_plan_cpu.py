"""Host-side check of the tensor-core input transform's plan
(e8_lattice_codebook_b200/csrc/glq_rht_mma.cu), without a GPU.

A host program includes the kernel source and, with the kernel's own
constexpr / host-device functions (tile plan, lane addressing, swizzles,
fragment builders, stage-B matrix, norm factors), emulates every warp of one
CTA on one row in double precision: the x4 ldmatrix.trans loads, the
m16n8k16 products (register layouts as the PTX ISA defines them), the
cross-tile butterflies, the x4 stmatrix stores and the copy-out.  For every
row size 2^L (9 <= L <= 14) and several lengths (multiples of 256, one to
four Hadamard blocks) it checks that

* the result is the block-diagonal Hadamard of S_in x (dense, fp64) to
  2^-22 of the row's largest value, with the prescale undone (the products
  are exact in double; the norm factors sqrt2 and 1/sqrt2 are the kernel's
  fp32 constants, at most two per value, each within 2^-24 relative);
* the positions the fragment sign masks are built for are the positions the
  loads deliver;
* every 8-lane phase of every x4 load / store, of the staging copies and of
  the copy-out meets 8 distinct 16-byte bank groups;
* the row's prescale exponent, taken from the bits of its largest
  magnitude, equals the one frexp gives, for every 16-bit pattern of both
  dtypes (zero, infinite and NaN rows: 0);
* each swizzle is a permutation of the row's units; stage A writes every
  unit of the row buffer that holds positions of the row exactly once
  (the others keep the zeros the kernel stores at its start; the emulation
  starts the rest from NaN), stage B every unit of the output buffer.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "e8_lattice_codebook_b200", "csrc")

HARNESS = r"""
#include "glq_rht_mma.cu"
#include <array>
#include <cmath>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <random>
#include <vector>

using namespace glq;

static int fails = 0;
#define CHECK(c, ...) do { if (!(c)) { if (fails < 20) { std::printf(__VA_ARGS__); std::printf("\n"); } ++fails; } } while (0)

// 16-bit float bits -> double
static double half_bits(uint32_t h) {
    const int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    const double v = e == 31 ? (m ? std::nan("") : INFINITY)
                             : (e == 0 ? std::ldexp((double)m, -24) : std::ldexp(1.0 + m / 1024.0, e - 15));
    return s ? -v : v;
}
static double bf16_bits(uint32_t h) {
    uint32_t u = (h & 0xFFFFu) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return (double)f;
}

struct Pair { double lo, hi; };

// PTX m16n8k16 layouts (lane = 4 gq + t)
static void unpack_a(const uint32_t w[32][4], bool bf16, double A[16][16]) {
    auto d = [&](uint32_t h) { return bf16 ? bf16_bits(h) : half_bits(h); };
    for (int l = 0; l < 32; ++l) {
        const int gq = l >> 2, t = l & 3;
        const int rows[4] = {gq, gq + 8, gq, gq + 8}, cols[4] = {2 * t, 2 * t, 2 * t + 8, 2 * t + 8};
        for (int q = 0; q < 4; ++q) {
            A[rows[q]][cols[q]] = d(w[l][q] & 0xFFFFu);
            A[rows[q]][cols[q] + 1] = d(w[l][q] >> 16);
        }
    }
}
static void unpack_a_pairs(const Pair w[32][4], double A[16][16]) {
    for (int l = 0; l < 32; ++l) {
        const int gq = l >> 2, t = l & 3;
        const int rows[4] = {gq, gq + 8, gq, gq + 8}, cols[4] = {2 * t, 2 * t, 2 * t + 8, 2 * t + 8};
        for (int q = 0; q < 4; ++q) {
            A[rows[q]][cols[q]] = w[l][q].lo;
            A[rows[q]][cols[q] + 1] = w[l][q].hi;
        }
    }
}
// B fragment (16 x 8) of n-tile nt from two words per lane: (2t | 2t+1, gq), (2t+8 | 2t+9, gq)
static void unpack_b_pairs(const Pair w[32][2], double Bm[16][8]) {
    for (int l = 0; l < 32; ++l) {
        const int gq = l >> 2, t = l & 3;
        Bm[2 * t][gq] = w[l][0].lo;
        Bm[2 * t + 1][gq] = w[l][0].hi;
        Bm[2 * t + 8][gq] = w[l][1].lo;
        Bm[2 * t + 9][gq] = w[l][1].hi;
    }
}
static void unpack_b_bits(const uint32_t w[32][2], double Bm[16][8]) {
    for (int l = 0; l < 32; ++l) {
        const int gq = l >> 2, t = l & 3;
        Bm[2 * t][gq] = half_bits(w[l][0] & 0xFFFFu);
        Bm[2 * t + 1][gq] = half_bits(w[l][0] >> 16);
        Bm[2 * t + 8][gq] = half_bits(w[l][1] & 0xFFFFu);
        Bm[2 * t + 9][gq] = half_bits(w[l][1] >> 16);
    }
}
// D = A B (16 x 8) scattered to the accumulator layout d[lane][4]
static void mma_emul(const double A[16][16], const double Bm[16][8], double d[32][4]) {
    double D[16][8];
    for (int i = 0; i < 16; ++i)
        for (int n = 0; n < 8; ++n) {
            double s = 0;
            for (int k = 0; k < 16; ++k) s += A[i][k] * Bm[k][n];
            D[i][n] = s;
        }
    for (int l = 0; l < 32; ++l) {
        const int gq = l >> 2, t = l & 3;
        d[l][0] = D[gq][2 * t];
        d[l][1] = D[gq][2 * t + 1];
        d[l][2] = D[gq + 8][2 * t];
        d[l][3] = D[gq + 8][2 * t + 1];
    }
}

typedef std::vector<std::array<double, 8>> Buf;
typedef std::vector<std::array<long, 8>> PosBuf;

// x4 ldmatrix.trans: lane l gives unit addr[l] for row l & 7 of matrix l >> 3;
// lane (gq, t) receives (M_q[2t][gq], M_q[2t+1][gq]) in register q
static void ldsm_trans(const Buf &b, const PosBuf &pb, const uint32_t addr[32], Pair r[32][4], long pos[32][4][2],
                       const char *what) {
    for (int q = 0; q < 4; ++q) {
        int seen = 0;
        for (int k = 0; k < 8; ++k) {
            const int g = addr[8 * q + k] & 7;
            CHECK(!(seen >> g & 1), "%s: bank conflict in matrix %d", what, q);
            seen |= 1 << g;
        }
    }
    for (int l = 0; l < 32; ++l) {
        const int gq = l >> 2, t = l & 3;
        for (int q = 0; q < 4; ++q) {
            const uint32_t u0 = addr[8 * q + 2 * t], u1 = addr[8 * q + 2 * t + 1];
            CHECK(u0 < b.size() && u1 < b.size(), "%s: unit out of the buffer", what);
            if (u0 >= b.size() || u1 >= b.size()) continue;
            r[l][q] = Pair{b[u0][gq], b[u1][gq]};
            pos[l][q][0] = pb[u0][gq];
            pos[l][q][1] = pb[u1][gq];
        }
    }
}
// x4 stmatrix: row r of matrix q at unit addr[8q + r] gets elements c from
// lane (gq = r, t = c / 2), register q, half c & 1
static void stsm(Buf &b, PosBuf &pb, std::vector<int> &written, const uint32_t addr[32], const Pair r[32][4],
                 const long pos[32][4][2], const char *what) {
    for (int q = 0; q < 4; ++q) {
        int seen = 0;
        for (int k = 0; k < 8; ++k) {
            const int g = addr[8 * q + k] & 7;
            CHECK(!(seen >> g & 1), "%s: bank conflict in matrix %d", what, q);
            seen |= 1 << g;
        }
        for (int row = 0; row < 8; ++row) {
            const uint32_t u = addr[8 * q + row];
            CHECK(u < b.size(), "%s: unit out of the buffer", what);
            if (u >= b.size()) continue;
            ++written[u];
            for (int c = 0; c < 8; ++c) {
                const int l = 4 * row + c / 2;
                b[u][c] = (c & 1) ? r[l][q].hi : r[l][q].lo;
                pb[u][c] = pos[l][q][c & 1];
            }
        }
    }
}

static std::vector<double> dense_blocks(const std::vector<double> &v, int len) {
    std::vector<double> y(len, 0.0);
    int off = 0;
    for (int b = 20; b >= 0; --b) {
        const int sz = 1 << b;
        if (!(len & sz)) continue;
        for (int i = 0; i < sz; ++i) {
            double s = 0;
            for (int k = 0; k < sz; ++k) s += ((popc32((uint32_t)(i & k)) & 1) ? -1.0 : 1.0) * v[off + k];
            y[off + i] = s / std::sqrt((double)sz);
        }
        off += sz;
    }
    return y;
}

template <int L>
static void check(int len, unsigned seed) {
    constexpr int W = mma_warps(L), TPW = mma_tpw(L), C = mma_cross(L), UNITS = 1 << (L - 3);
    const int units = len >> 3;
    std::mt19937 rng(seed);
    std::normal_distribution<double> nd;
    std::vector<double> x(len), sx(len);
    std::vector<uint32_t> sign_bits((len + 31) / 32, 0u);
    for (int i = 0; i < len; ++i) {
        x[i] = nd(rng);
        if (rng() & 1) sign_bits[i >> 5] |= 1u << (i & 31);
        sx[i] = (sign_bits[i >> 5] >> (i & 31) & 1) ? -x[i] : x[i];
    }
    // swizzles: permutations of the units
    {
        std::vector<int> a(UNITS, 0), b(UNITS, 0), c(UNITS, 0);
        for (int u = 0; u < UNITS; ++u) {
            ++a[slot_s((uint32_t)u << 3)];
            ++b[slot_r(L, (uint32_t)u << 3)];
            ++c[slot_o(L, (uint32_t)u << 3)];
        }
        for (int u = 0; u < UNITS; ++u) CHECK(a[u] == 1 && b[u] == 1 && c[u] == 1, "L=%d: swizzle not a permutation", L);
        for (int u0 = 0; u0 < UNITS; u0 += 8) {  // copies and copy-out: 8 consecutive units per phase
            int ss = 0, so = 0;
            for (int u = u0; u < u0 + 8; ++u) {
                ss |= 1 << (slot_s((uint32_t)u << 3) & 7);
                so |= 1 << (slot_o(L, (uint32_t)u << 3) & 7);
            }
            CHECK(ss == 255 && so == 255, "L=%d: consecutive units meet a bank group twice", L);
        }
    }
    // staging: raw x (positions past len zero)
    Buf S(UNITS), R(UNITS), O(UNITS);
    PosBuf Sp(UNITS), Rp(UNITS), Op(UNITS);
    // the row buffer starts as stale shared memory (NaN), except the units
    // past the row, which the kernel zeroes at its start
    for (int u = 0; u < UNITS; ++u)
        for (int e = 0; e < 8; ++e) {
            const uint32_t p = 8u * u + e, su = slot_r(L, p);
            R[su][e] = p < (uint32_t)len ? std::nan("") : 0.0;
            Rp[su][e] = p;
        }
    for (int u = 0; u < UNITS; ++u)
        for (int e = 0; e < 8; ++e) {
            const long p = 8L * u + e;
            S[slot_s((uint32_t)p)][e] = p < len ? x[p] : 0.0;
            Sp[slot_s((uint32_t)p)][e] = p;
        }
    double mx = 0;
    for (int i = 0; i < len; ++i) mx = std::max(mx, std::fabs(x[i]));
    int E;
    std::frexp(mx, &E);
    const double scale = std::ldexp(1.0, 8 - E);
    std::vector<int> wR(UNITS, 0), wO(UNITS, 0);
    for (int w = 0; w < W; ++w) {
        // ---- stage A
        double d2[TPW][2][32][4];
        for (int i = 0; i < TPW; ++i) {
            const uint32_t base = (uint32_t)(w * TPW + i) << 8;
            if (base >= (uint32_t)len) continue;  // tiles past the row are skipped
            uint32_t addr[32];
            for (int l = 0; l < 32; ++l) addr[l] = (base >> 3) + slot_s(offa_of(l));
            Pair r[32][4];
            long pos[32][4][2];
            ldsm_trans(S, Sp, addr, r, pos, "stage A load");
            for (int l = 0; l < 32; ++l) {
                // the lane's sign words over all the warp's tiles, packed and
                // read back as the kernel does (sign_bit_of, sign_xor)
                uint32_t sgn[mma_sign_words(L)] = {};
                for (int i2 = 0; i2 < TPW; ++i2)
                    for (int q = 0; q < 4; ++q)
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t p2 = frag_pos((uint32_t)(w * TPW + i2) << 8, l, q, h);
                            if (p2 < (uint32_t)len && (sign_bits[p2 >> 5] >> (p2 & 31) & 1))
                                sgn[i2 >> 2] |= 1u << sign_bit_of(i2, q, h);
                        }
                for (int q = 0; q < 4; ++q)
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t fp = frag_pos(base, l, q, h);
                        CHECK((long)fp == pos[l][q][h], "L=%d: sign mask position %u, loaded %ld", L, fp, pos[l][q][h]);
                        const bool neg = (sign_xor(sgn[i >> 2], i, q) >> (15 + 16 * h)) & 1u;
                        const bool want = fp < (uint32_t)len && (sign_bits[fp >> 5] >> (fp & 31) & 1);
                        CHECK(neg == want, "L=%d: sign of position %u from the packed words", L, fp);
                        double &v = h ? r[l][q].hi : r[l][q].lo;
                        if (neg) v = -v;
                    }
            }
            uint32_t a1w[32][4];
            for (int l = 0; l < 32; ++l) a_frag(l, Had16{0x3E80u}, a1w[l]);  // bf16 0.25
            double A1[16][16];
            unpack_a(a1w, true, A1);
            double d1[2][32][4];
            for (int nt = 0; nt < 2; ++nt) {
                Pair bw[32][2];
                for (int l = 0; l < 32; ++l) { bw[l][0] = r[l][2 * nt]; bw[l][1] = r[l][2 * nt + 1]; }
                double Bm[16][8];
                unpack_b_pairs(bw, Bm);
                mma_emul(A1, Bm, d1[nt]);
            }
            Pair a2[32][4];
            for (int l = 0; l < 32; ++l) {
                a2[l][0] = Pair{d1[0][l][0] * scale, d1[0][l][1] * scale};
                a2[l][1] = Pair{d1[0][l][2] * scale, d1[0][l][3] * scale};
                a2[l][2] = Pair{d1[1][l][0] * scale, d1[1][l][1] * scale};
                a2[l][3] = Pair{d1[1][l][2] * scale, d1[1][l][3] * scale};
            }
            double A2[16][16];
            unpack_a_pairs(a2, A2);
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t bw[32][2];
                for (int l = 0; l < 32; ++l) b_frag(l, nt, Had16{0x3400u}, bw[l]);
                double Bm[16][8];
                unpack_b_bits(bw, Bm);
                mma_emul(A2, Bm, d2[i][nt]);
            }
        }
        for (int cb = 0; cb < C; ++cb)
            for (int a = 0; a < TPW; ++a)
                if (!((a >> cb) & 1) && bfly_active((uint32_t)(w * TPW + a) << 8, 8 + cb, (uint32_t)len))
                    for (int nt = 0; nt < 2; ++nt)
                        for (int l = 0; l < 32; ++l)
                            for (int e = 0; e < 4; ++e) {
                                const double x0 = d2[a][nt][l][e], x1 = d2[a | (1 << cb)][nt][l][e];
                                d2[a][nt][l][e] = x0 + x1;
                                d2[a | (1 << cb)][nt][l][e] = x0 - x1;
                            }
        for (int i = 0; i < TPW; ++i) {
            const uint32_t base = (uint32_t)(w * TPW + i) << 8;
            if (base >= (uint32_t)len) continue;
            const double f = cross_norm<L>(base, (uint32_t)len);
            uint32_t addr[32];
            Pair r[32][4];
            long pos[32][4][2];
            for (int l = 0; l < 32; ++l) {
                addr[l] = slot_r(L, base) ^ slot_r(L, offa_of(l));
                CHECK(addr[l] == slot_r(L, base | offa_of(l)), "L=%d: row-buffer slot not linear", L);
                const int gq = l >> 2, t = l & 3;
                for (int q = 0; q < 4; ++q) {
                    const int nt = q >> 1, hi = q & 1;
                    r[l][q] = Pair{d2[i][nt][l][2 * hi] * f, d2[i][nt][l][2 * hi + 1] * f};
                    // output (row j = gq + 8 hi: bits 4-7; col 2t + 8 nt (+1): bits 0-3)
                    for (int h = 0; h < 2; ++h) pos[l][q][h] = base + ((gq + 8 * hi) << 4) + 2 * t + h + 8 * nt;
                }
            }
            stsm(R, Rp, wR, addr, r, pos, "stage A store");
        }
    }
    for (int u = 0; u < UNITS; ++u) {
        const int want = Rp[u][0] < len ? 1 : 0;  // units past the row keep their zeros
        CHECK(wR[u] == want, "L=%d: row-buffer unit %d written %d times", L, u, wR[u]);
        for (int e = 0; e < 8; ++e) CHECK(Rp[u][e] >= 0 && slot_r(L, (uint32_t)Rp[u][e]) == (uint32_t)u && (Rp[u][e] & 7) == e,
                                          "L=%d: row buffer slot %d holds position %ld", L, u, Rp[u][e]);
    }
    // ---- stage B
    uint32_t aBw[32][4];
    for (int l = 0; l < 32; ++l) a_frag(l, StageB<L>{(uint32_t)len}, aBw[l]);
    double AB[16][16];
    unpack_a(aBw, false, AB);
    for (int w = 0; w < W; ++w) {
        double d[TPW][2][32][4];
        uint32_t tbs[TPW];
        for (int i = 0; i < TPW; ++i) {
            const uint32_t tb = tileb_pos(L, w * TPW + i);
            tbs[i] = tb;
            uint32_t addr[32];
            for (int l = 0; l < 32; ++l) addr[l] = slot_r(L, tb) ^ slot_r(L, offb_of(L, l));
            Pair r[32][4];
            long pos[32][4][2];
            ldsm_trans(R, Rp, addr, r, pos, "stage B load");
            for (int nt = 0; nt < 2; ++nt) {
                Pair bw[32][2];
                for (int l = 0; l < 32; ++l) { bw[l][0] = r[l][2 * nt]; bw[l][1] = r[l][2 * nt + 1]; }
                double Bm[16][8];
                unpack_b_pairs(bw, Bm);
                mma_emul(AB, Bm, d[i][nt]);
            }
        }
        for (int i = 0; i < TPW; ++i) {
            const uint32_t tb = tbs[i];
            uint32_t oaddr[32];
            for (int l = 0; l < 32; ++l) oaddr[l] = slot_o(L, tb) ^ slot_o(L, offb_of(L, l));
            Pair o[32][4];
            long opos[32][4][2];
            for (int l = 0; l < 32; ++l) {
                const int gq = l >> 2, t = l & 3;
                const double c0 = stageb_norm<L>(gq, (uint32_t)len), c1 = stageb_norm<L>(gq + 8, (uint32_t)len);
                for (int q = 0; q < 4; ++q) {
                    const int nt = q >> 1, hi = q & 1;
                    const double c = hi ? c1 : c0;
                    o[l][q] = Pair{d[i][nt][l][2 * hi] * c, d[i][nt][l][2 * hi + 1] * c};
                    for (int h = 0; h < 2; ++h)
                        opos[l][q][h] = tb | kb_pos(L, gq + 8 * hi) | (uint32_t)(2 * t + h + 8 * nt);
                }
            }
            stsm(O, Op, wO, oaddr, o, opos, "stage B store");
        }
    }
    for (int u = 0; u < UNITS; ++u) {
        CHECK(wO[u] == 1, "L=%d: output unit %d written %d times", L, u, wO[u]);
        for (int e = 0; e < 8; ++e) CHECK(slot_o(L, (uint32_t)Op[u][e]) == (uint32_t)u && (Op[u][e] & 7) == e,
                                          "L=%d: output slot %d holds position %ld", L, u, Op[u][e]);
    }
    // ---- copy-out and the dense transform
    const std::vector<double> ref = dense_blocks(sx, len);
    double err = 0, rmax = 0;
    for (int u = 0; u < units; ++u)
        for (int e = 0; e < 8; ++e) {
            const double y = O[slot_o(L, (uint32_t)u << 3)][e] / scale;
            err = std::max(err, std::fabs(y - ref[8 * u + e]));
            rmax = std::max(rmax, std::fabs(ref[8 * u + e]));
        }
    CHECK(err <= std::ldexp(rmax, -22), "L=%d len=%d: max error %.3e (max %.3e)", L, len, err, rmax);
}

template <int L>
static void check_lengths() {
    for (int len = (1 << (L - 1)) + 256; len <= (1 << L); len += 256) {
        const int nb = popc32((uint32_t)len);
        // every length up to 2^11, then those with the most blocks and the powers of two
        if (L <= 11 || nb >= 3 || len == (1 << L) || len == (1 << (L - 1)) + 256) check<L>(len, 1000u * L + len);
    }
}

// the prescale exponent from the 16-bit magnitude bits, against frexp of
// the value, for every magnitude pattern of both dtypes
template <bool BF16>
static void check_prescale() {
    for (uint32_t h = 0; h < 0x8000u; ++h) {
        const double v = BF16 ? bf16_bits(h) : half_bits(h);
        int want = 0;
        if (v != 0.0 && std::isfinite(v)) {
            int E;
            std::frexp(v, &E);  // v < 2^E
            want = std::min(126, std::max(-124, 8 - E));
        }
        CHECK(prescale_exp<BF16>(h) == want, "prescale_exp<%d>(0x%04x) = %d, want %d", (int)BF16, h,
              prescale_exp<BF16>(h), want);
    }
}

int main() {
    check_prescale<true>();
    check_prescale<false>();
    check_lengths<9>();
    check_lengths<10>();
    check_lengths<11>();
    check_lengths<12>();
    check_lengths<13>();
    check_lengths<14>();
    std::printf(fails ? "FAILED %d\n" : "OK\n", fails);
    return fails ? 1 : 0;
}
"""


def test_tensor_core_row_transform_plan(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "rht_mma_plan.cu"
    src.write_text(HARNESS)
    exe = tmp_path / "rht_mma_plan"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
                    str(src), "-o", str(exe)], check=True, capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), out.stdout
