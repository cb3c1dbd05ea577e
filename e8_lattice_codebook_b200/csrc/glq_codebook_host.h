// glq_codebook_host.h -- host-side codebook helpers of glq-b200.
#pragma once

#include <stdint.h>

#include <vector>

namespace glq {

// The library's 65,536 x 8 E8 shell codebook as fp16 bit patterns.
void build_e8_codebook(uint16_t *out_fp16_bits);

// Exact binary16 bits of y2 / 2 for an integer |y2| <= 12.
uint16_t half_bits_of_half_integer(int y2);

// IEEE binary16 bits -> float (exact).
float half_bits_to_float(uint16_t h);

struct FoldedTable {
    int nb = 0;                   // words in the on-chip table
    int neg_base = 0;             // code e >= nb reads words[e - neg_base] negated
    uint16_t zero_code = 0;       // code of the origin (padding)
    std::vector<uint32_t> words;  // nibble-packed entries
    std::vector<uint16_t> code;   // raw index -> code
};

// Builds the negation-folded nibble table of a 65,536-entry table.
// Returns 0, -1 (a value is not k/2 with |k| <= 6), -2 (duplicate
// entries) or -3 (folded table larger than the on-chip capacity).
int fold_table(const uint16_t *fp16_bits, FoldedTable *out);

}  // namespace glq
