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
//     x0..x3 in the low nibbles of bytes 0..3, x4..x7 in the high nibbles.
//     w & 0x0F0F0F0F and (w >> 4) & 0x0F0F0F0F are then exactly the two
//     32-bit A-fragment registers (four u8 values each) one lane of the
//     integer mma.m16n8k32 needs for one row: a whole codeword per lane.
//     Negation is v -> 12 - v per nibble, i.e. word -> 0xCCCCCCCC - word.
//
//   * Activations for the integer MMA: per token the input RHT writes
//     X = round(xr * 2^e) (|X| <= 2^14, e per token from max |xr|) as
//     16 bytes per group of 8 columns: 8 high bytes (X >> 8, signed) then 8
//     low bytes (X & 255).  The MMA accumulates sum v X exactly in int32
//     (u8 x s8 and u8 x u8), and sum x X = (sum v X - 6 sum X) / 2 with the
//     exact integer row sum sum X.  Exact integer accumulation makes the
//     result independent of summation order and of the batch size.
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

// largest row of the RHT kernels (8 parts of 4096 in one cluster)
#define GLQ_RHT_MAX_N 32768
#define GLQ_MAX_BLOCKS 32
#define GLQ_RHT_SEG 4096
#define GLQ_RHT_THREADS 1024
#define GLQ_RHT_MAX_PARTS 8
#define GLQ_RHT_MAX_PIECES 32

// x = v/2 - 3 for a table nibble v
#define GLQ_NIB_OFFSET 6  // sum x X = (sum v X - 6 sum X) / 2

// device error word bits
#define GLQ_DEVERR_TIMEOUT 1u
#define GLQ_DEVERR_BOUNDS 2u

struct glq_blocks {
    int count;
    int size[GLQ_MAX_BLOCKS];
    int offset[GLQ_MAX_BLOCKS];
    float inv_sqrt[GLQ_MAX_BLOCKS];  // 1/sqrt(size), computed on the host in double
};

// Row info written by the input RHT for every token: X = round(xr 2^e),
// inv_scale = 2^-e, sum_x = exact sum over the row of X.
struct glq_rowinfo {
    long long sum_x;
    float inv_scale;
    float pad;
};
