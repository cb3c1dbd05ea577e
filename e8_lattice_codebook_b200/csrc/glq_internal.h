// glq_internal.h -- layouts shared by the host library and the kernels of
// glq-b200 (the CUDA implementation of the GLQ compressed-weight linear
// layer; the public C ABI is include/glq.h).
//
// Device layout of a layer (what glq_layer_create builds):
//
//   * Index streams in "fragment-native" order.  Rows are tiled by 16
//     (row tile rt) and columns by 128 (chunk kc = 16 groups of 8).  For
//     warp lane = 4*g + t (g = lane>>2, t = lane&3) the 16 bytes of stream 1
//     at [rt][kc][lane] hold, for super-tiles s = 0..3, the pair
//     (code of row 16rt+g, code of row 16rt+g+8) of group 16kc+4s+t.  That is
//     exactly the A fragment a lane of mma.m16n8k16 needs when the 32
//     columns of a super-tile are assigned lane-by-lane to whole codewords
//     (the contraction is invariant under a consistent column permutation).
//     Stream 2 (residual) has the same order: uint16 codes (4 bpw, 16 B per
//     lane and chunk) or uint8 indices (3 bpw, 8 B per lane and chunk).
//     Padding rows / groups hold code 0 (the origin for the E8 table; any
//     value for the 256-entry table: padded columns meet zero activations
//     and padded rows are never stored).
//
//   * Codes instead of raw indices.  A 65,536-entry table of E8 points is
//     folded under negation: every full shell is closed under x -> -x, so
//     the on-chip table T keeps the self-symmetric origin, one point of each
//     +-pair and the unpaired points (NB words).  Code e < NB reads T[e];
//     code e >= NB reads T[e - NB + S] negated (S = 1 when the origin is in
//     the table).  The host maps every raw index to its code once at layer
//     creation; glq_dequant_reference inverts nothing, it decodes codes.
//
//   * A table word packs the 8 coordinates as nibbles v = 2x + 6 in [0, 12]:
//     bits 0-3 x0, 16-19 x1, 4-7 x2, 20-23 x3, 8-11 x4, 24-27 x5,
//     12-15 x6, 28-31 x7.  A 16-bit half whose only set bits are a nibble
//     at bits 0-3 is the fp16 subnormal v * 2^-24 (at bits 4-7: 16 v * 2^-24),
//     so one AND per coordinate pair turns a word into exact MMA operands
//     with no exponent offset.  Columns k with k mod 8 in {2,3,6,7} (the
//     bits 4-7 nibbles) carry the factor 16, which the input RHT removes by
//     storing those activations divided by 16.  The MMA then yields
//     2^-24 sum_k v_k X_k with v = 2x + 6, so
//         sum_k x_k X_k = 2^23 acc - 3 sum_k X_k,
//     and the row-independent term 3 sum_k X_k is formed once per token in
//     fp64.  (A large per-column offset would not do: the warp MMA's fp32
//     accumulation truncates, and a bias common to every row becomes one
//     sqrt(m)-sized spike after the output Hadamard.)  Negation is
//     v -> 12 - v per nibble, i.e. word -> 0xCCCCCCCC - word.
#pragma once

#include <stdint.h>

#define GLQ_CB_ENTRIES 65536
#define GLQ_CB8_ENTRIES 256
#define GLQ_DIM 8

// kernel tiling
#define GLQ_ROW_TILE 16
#define GLQ_CHUNK_K 128
#define GLQ_GROUPS_PER_CHUNK 16

// on-chip folded table capacity (words); the library's E8 table needs 37,096
#define GLQ_TABLE_MAX_WORDS 40960

// decode batch limit (the GEMV handles up to two 8-column MMA tiles)
#define GLQ_DECODE_MAX_B 16

// size of the fixed device scratch array of glq_linear_noalloc (the public
// header states the same value)
#ifndef GLQ_NOALLOC_SCRATCH_BYTES
#define GLQ_NOALLOC_SCRATCH_BYTES (8u << 20)
#endif

// largest Hadamard block handled by the one-CTA-per-row RHT kernels
#define GLQ_RHT_MAX_N 32768
#define GLQ_MAX_BLOCKS 32

// the nibble decode: operand = v * 2^-24 (x 16 on columns k mod 8 in {2,3,6,7})
#define GLQ_ACC_SCALE 8388608.0f  // 2^23: sum x X = 2^23 acc - 3 sum X
#define GLQ_NIB_OFFSET 3.0        // x = v/2 - 3

// device error word bits
#define GLQ_DEVERR_TIMEOUT 1u
#define GLQ_DEVERR_BOUNDS 2u

struct glq_blocks {
    int count;
    int size[GLQ_MAX_BLOCKS];
    int offset[GLQ_MAX_BLOCKS];
    float inv_sqrt[GLQ_MAX_BLOCKS];  // 1/sqrt(size), computed on the host in double
};

// Row info written by the input RHT for every token: the activations X are
// xr * 2^scale_exp (stored /16 on columns k mod 8 in {2,3,6,7});
// inv_scale = 2^-scale_exp; corr = 3 sum_k X_k (fp64).
struct glq_rowinfo {
    double corr;
    float inv_scale;
    float pad;
};
