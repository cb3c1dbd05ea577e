// glq_codebook_host.cpp -- host-side codebook work of glq-b200:
//   * the library's E8 shell codebook (glq 0.5.1 PyPI page, "How it works"
//     1: 65,536 vectors from the first shells of the E8 lattice; the exact
//     subset -- all points of squared norm <= 12 ordered by (norm, x0..x7),
//     first 65,536 -- is this library's fixed rule);
//   * the negation-folded nibble table and the index -> code map the decode
//     kernels use (layout described in glq_internal.h).
#include "glq_codebook_host.h"

#include <algorithm>
#include <array>
#include <cmath>
#include <cstring>
#include <map>
#include <vector>

#include "glq_internal.h"

namespace glq {

namespace {

struct Point {
    int norm4;              // sum of (2x_i)^2
    std::array<int8_t, 8> y;  // doubled coordinates
};

// Depth-first generation of doubled coordinates y_i of one parity class
// (even: integer points, odd: half-integer points) with sum(y^2) <= limit.
void grow(int depth, int parity, int budget, int ysum, Point &cur, std::vector<Point> &out) {
    if (depth == 8) {
        if (((ysum % 4) + 4) % 4 == 0) {  // sum of x even
            cur.norm4 = 48 - budget;
            out.push_back(cur);
        }
        return;
    }
    for (int y = -6; y <= 6; ++y) {
        if (((y % 2) + 2) % 2 != parity) continue;
        int sq = y * y;
        if (sq > budget) continue;
        cur.y[depth] = (int8_t)y;
        grow(depth + 1, parity, budget - sq, ysum + y, cur, out);
    }
}

}  // namespace

uint16_t half_bits_of_half_integer(int y2) {
    // exact binary16 of y2 / 2 for |y2| <= 12
    if (y2 == 0) return 0;
    uint16_t sign = y2 < 0 ? 0x8000 : 0;
    int a = y2 < 0 ? -y2 : y2;  // value = a / 2
    int e = 0;
    while ((a >> (e + 1)) != 0) ++e;  // a in [2^e, 2^(e+1))
    // value = a * 2^-1 = 1.f * 2^(e-1); mantissa = (a - 2^e) << (10 - e)
    uint16_t exp_field = (uint16_t)(e - 1 + 15);
    uint16_t mant = (uint16_t)((a - (1 << e)) << (10 - e));
    return (uint16_t)(sign | (exp_field << 10) | mant);
}

void build_e8_codebook(uint16_t *out_fp16_bits) {
    std::vector<Point> pts;
    pts.reserve(120000);
    Point cur{};
    grow(0, 0, 48, 0, cur, pts);
    grow(0, 1, 48, 0, cur, pts);
    std::sort(pts.begin(), pts.end(), [](const Point &a, const Point &b) {
        if (a.norm4 != b.norm4) return a.norm4 < b.norm4;
        return a.y < b.y;  // lexicographic on x0..x7
    });
    for (int e = 0; e < GLQ_CB_ENTRIES; ++e)
        for (int j = 0; j < 8; ++j) out_fp16_bits[e * 8 + j] = half_bits_of_half_integer(pts[e].y[j]);
}

float half_bits_to_float(uint16_t h) {
    uint32_t sign = (uint32_t)(h & 0x8000) << 16;
    uint32_t exp = (h >> 10) & 0x1f;
    uint32_t mant = h & 0x3ff;
    uint32_t bits;
    if (exp == 0) {
        if (mant == 0) {
            bits = sign;
        } else {  // subnormal: renormalise
            int shift = 0;
            while (!(mant & 0x400)) {
                mant <<= 1;
                ++shift;
            }
            mant &= 0x3ff;
            bits = sign | ((uint32_t)(127 - 15 - shift + 1) << 23) | (mant << 13);
        }
    } else if (exp == 31) {
        bits = sign | 0x7f800000u | (mant << 13);
    } else {
        bits = sign | ((exp - 15 + 127) << 23) | (mant << 13);
    }
    float f;
    std::memcpy(&f, &bits, sizeof f);
    return f;
}

int fold_table(const uint16_t *fp16_bits, FoldedTable *out) {
    // doubled coordinates of every entry, validated to lie in [-6, 6]
    std::vector<std::array<int8_t, 8>> ys(GLQ_CB_ENTRIES);
    for (int e = 0; e < GLQ_CB_ENTRIES; ++e) {
        for (int j = 0; j < 8; ++j) {
            float v = half_bits_to_float(fp16_bits[e * 8 + j]);
            float y = 2.0f * v;
            if (!(y >= -6.0f && y <= 6.0f) || y != std::floor(y)) return -1;
            ys[e][j] = (int8_t)y;
        }
    }
    std::map<std::array<int8_t, 8>, int> where;
    for (int e = 0; e < GLQ_CB_ENTRIES; ++e)
        if (!where.emplace(ys[e], e).second) return -2;  // duplicate entries

    // classify: self-symmetric (the origin), pair representative (the
    // smaller index of a +-pair), pair partner, unpaired
    std::vector<int> partner(GLQ_CB_ENTRIES, -1);
    std::vector<int> selfsym, reps, single;
    for (int e = 0; e < GLQ_CB_ENTRIES; ++e) {
        std::array<int8_t, 8> neg;
        for (int j = 0; j < 8; ++j) neg[j] = (int8_t)-ys[e][j];
        auto it = where.find(neg);
        if (it == where.end()) {
            single.push_back(e);
        } else if (it->second == e) {
            selfsym.push_back(e);
        } else {
            partner[e] = it->second;
            if (e < it->second) reps.push_back(e);
        }
    }
    int S = (int)selfsym.size();
    int NB = S + (int)reps.size() + (int)single.size();
    if (NB > GLQ_TABLE_MAX_WORDS) return -3;

    out->nb = NB;
    out->neg_base = NB - S;  // code e >= NB reads T[e - neg_base], negated
    out->words.assign((size_t)NB, 0u);
    out->code.assign(GLQ_CB_ENTRIES, 0);
    std::vector<int> pos(GLQ_CB_ENTRIES, -1);
    int p = 0;
    for (int e : selfsym) pos[e] = p++;
    for (int e : reps) pos[e] = p++;
    for (int e : single) pos[e] = p++;
    for (int e = 0; e < GLQ_CB_ENTRIES; ++e) {
        if (pos[e] >= 0) {
            uint32_t w = 0;
            static const int shift[8] = {0, 8, 16, 24, 4, 12, 20, 28};
            for (int j = 0; j < 8; ++j) w |= (uint32_t)(ys[e][j] + 6) << shift[j];
            out->words[(size_t)pos[e]] = w;
            out->code[e] = (uint16_t)pos[e];
        }
    }
    for (int e = 0; e < GLQ_CB_ENTRIES; ++e) {
        if (pos[e] < 0) {  // partner of a representative: negated code
            int rep = partner[e];
            out->code[e] = (uint16_t)(pos[rep] + out->neg_base);
        }
    }
    // the origin is code 0 when present (used as the padding code)
    out->zero_code = 0;
    for (int e : selfsym) out->zero_code = out->code[e];
    return 0;
}

}  // namespace glq
