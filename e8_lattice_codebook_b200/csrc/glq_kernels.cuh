// glq_kernels.cuh -- kernel parameter blocks and launchers of glq-b200.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "glq_device.cuh"
#include "glq_internal.h"

namespace glq {

// One piece of a part of the RHT row plan: `len` values at row offset
// `off`, belonging to a Hadamard block of size K split over C parts (this is
// part q; the block's parts are cluster ranks rank0 .. rank0+C-1).
struct RhtPiece {
    int off, len, K, C, q, rank0;
    float norm;  // 1/sqrt(K), computed on the host in double
};

struct RhtPlan {
    int parts, npieces, clustered;
    int first_piece[GLQ_RHT_MAX_PARTS + 1];
    RhtPiece piece[GLQ_RHT_MAX_PIECES];
};

RhtPlan make_rht_plan(int N);

struct RhtInParams {
    const void *x;  // [B][n] fp16 / bf16
    int x_bf16;
    int n, n_pad;
    int B;
    const uint32_t *sign_bits;  // bit k set: S_in[k] = -1
    RhtPlan plan;
    uint8_t *xq;        // [B][n_pad/8][16]: high bytes, low bytes of X (product path)
    __half *xh;         // [B][n_pad] fp16 X (the 8-bit residual stage of an odd bpw) or null
    glq_rowinfo *info;  // [B] (product path)
    float *xr_f32;      // [B][n] unscaled fp32 (test entry point) or null
    int xh_only;        // tensor-core path: write xh = fp16(xr 2^e) only (no xq, no sum)
};

struct RhtOutParams {
    int m, B;
    const float *z;  // [B][z_ld] fp32
    int z_ld;
    const uint32_t *sign_bits;  // bit r set: S_out[r] = -1
    RhtPlan plan;
    void *y;      // [B][m]
    int y_dtype;  // 0 f16, 1 bf16, 2 f32
    // input side, fp16 operand: 0 the tensor-core kernel where it applies,
    // 1 always the butterfly kernel
    int butterfly;
};

// Row transforms of the tensor-core path (glq_rht_rows.cu): one CTA per row.
struct RowsParams {
    int len, len_pad;           // row length (n or m) and, input side, the padded row of xh
    int nblk, max_blk;          // Hadamard blocks of len (descending powers of two)
    int blk_off[GLQ_MAX_BLOCKS], blk_len[GLQ_MAX_BLOCKS];
    float blk_norm[GLQ_MAX_BLOCKS];  // 1/sqrt(block)
    const uint32_t *sign_bits;
    // input: x [B][len] fp16 / bf16 -> xh [B][len_pad] fp16 (xr 2^e), info [B]
    const void *x;
    int x_bf16;
    __half *xh;
    glq_rowinfo *info;
    // input, decode format instead (when xq is set): X = round(xr 2^e) as
    // [B][len_pad / 8][16] high / low bytes, X as fp16 in xh (odd bpw, may
    // be null), info [B] = {exact sum of X, 2^-e}
    uint8_t *xq;
    // output: z [B][z_ld] fp32 (summed over zsplits slices zs floats apart,
    // in order) -> y [B][len]
    const float *z;
    int z_ld;
    int zsplits;
    size_t zs;
    void *y;
    int y_dtype;  // 0 f16, 1 bf16, 2 f32
    // input side, fp16 operand: 0 the tensor-core kernel where it applies,
    // 1 always the butterfly kernel
    int butterfly;
};

// Residual stages of a bit width ("Bit widths", glq 0.5.1 PyPI page): after
// the 16-bit primary, N16 16-bit E8 stages, then an 8-bit stage (U8) for an
// odd bpw.
template <int BPW>
struct Stages {
    static constexpr int N16 = (BPW - 2) / 2;
    static constexpr bool U8 = (BPW & 1) != 0;
    static constexpr int NA = N16 > 0 ? N16 : 1;  // extent of per-stage arrays
};
__host__ __device__ constexpr int stages16(int bpw) { return (bpw - 2) / 2; }
__host__ __device__ constexpr bool stage8(int bpw) { return (bpw & 1) != 0; }

struct GemvParams {
    const uint4 *idx1;     // [RT][KC][32] 16 B
    const uint4 *idx16[3]; // 16-bit residual stages: [RT][KC][32] 16 B each
    const uint2 *idx8;     // the 8-bit stage: [RT][KC][32] 8 B
    const uint32_t *table; // folded nibble table (global), table_words (multiple of 4)
    int table_words;
    FoldParams fold;
    LookupConsts kc;       // 4, 16, -1 (see LookupConsts)
    const uint4 *tab8;     // odd bpw: the 256-entry table, [256] x 8 fp16
    const uint8_t *xq;     // [B][n_pad/8][16]
    const __half *xh;      // [B][n_pad] (odd bpw)
    const glq_rowinfo *info;
    int B, n_pad, KC, RT;
    int bands, splits, cps;
    double rs16_d[3];      // weights of the 16-bit stages' sums in a partial: their scales
    double rs8_d;          // weight of the 8-bit stage's sum: 2 x its scale
    double corr_mult;      // 1 + the sum of the 16-bit stages' scales
    float ws;
    double *partials;      // [splits][B][m_pad]
    unsigned *counters;    // [bands], zero between launches
    float *z;              // [B][m_pad]
    int m_pad;
    unsigned *err;
    int warps;             // warps per CTA (gemv_warps(NT, bpw), or GEMV_WIDE_WARPS)
    // ---- fused transforms (small B) ----
    // input: every task rotates, scales and quantises its own column range
    // of x in shared memory (no separate input-RHT launch)
    const void *x;         // [B][n] fp16 / bf16, rows 16-byte aligned
    int x_bf16, n;
    const uint32_t *sin_bits;
    int nblk_n;            // Hadamard blocks of n: descending powers of two
    int blk_off_n[GLQ_MAX_BLOCKS], blk_len_n[GLQ_MAX_BLOCKS];
    // output: the last band to finish a Hadamard block of m transforms it
    // in shared memory and writes y (no separate output-RHT launch)
    int fuse_out;
    void *y;               // [B][m]
    int y_dtype, m;
    const uint32_t *sout_bits;
    int nblk_m;
    int blk_off_m[GLQ_MAX_BLOCKS], blk_len_m[GLQ_MAX_BLOCKS];
    int blk_bands[GLQ_MAX_BLOCKS];  // bands whose rows meet block i
    unsigned *blk_cnt;     // [GLQ_MAX_BLOCKS], zero between launches
    // split-K in a thread-block cluster (one task per CTA, the band's
    // splits form one cluster): clu = cluster size (= splits) or 0, and the
    // byte offset of the partial sums in dynamic shared memory
    int clu;
    size_t spart_off;
};

struct PrefillParams {
    const uint4 *idx1;       // [RT][KC][32] 16 B, fragment-native codes
    const uint4 *idx16[3];   // 16-bit residual stages, 16 B per slot
    const uint2 *idx8;       // the 8-bit stage, 8 B per slot
    const uint4 *cb_f16;     // E8 codewords as fp16 [folded code][8] (negated entries included)
    const uint32_t *table;   // folded nibble table (W materialisation), table_words
    int table_words;
    FoldParams fold;
    const uint4 *tab8;       // odd bpw: [256][8] fp16
    int bpw;
    uint32_t rs16_h2[3];     // the 16-bit stages' scales as fp16x2
    uint32_t rs8_h2;         // the 8-bit stage's scale as fp16x2
    const glq_rowinfo *info; // [B]: inv_scale per token
    float ws;
    float *z;                // [ksplit][B][m_pad]: one slice of partial sums per K split
    size_t zs;               // floats between slices
    int ksplit;              // K splits (chunk-aligned), >= 1
    int B, m_pad, KC, RT;
    int tiles_tok, ntiles;   // ntiles: work items (row tiles x token tiles x ksplit, halves counted twice)
    int tiles_whole;         // items [0, tiles_whole) are whole tiles, the rest halves of the tiles after them
    unsigned *err;
};

struct DequantParams {
    const uint4 *idx1;
    const uint4 *idx16[3];
    const uint2 *idx8;
    const uint32_t *table;
    FoldParams fold;
    const uint4 *tab8;
    int bpw;
    int64_t m;
    int n, G, KC;
    float ws, rs16[3], rs8;
    float *w;  // [m][n]
};

// cudaLaunchKernelExC with optional programmatic stream serialisation and
// an optional 1-D thread-block cluster of `cluster` CTAs.
inline cudaError_t launch_ex(const void *fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             bool pdl, void **args, int cluster = 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (cluster > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = cluster;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// Runs set() -- the cudaFuncSetAttribute calls of one kernel -- once per
// device (devices 0..63; attributes apply to the current device only), with
// `done` the kernel's static bit mask of devices already set.  A race only
// repeats set(), which is harmless.
template <typename F>
inline cudaError_t once_per_device(std::atomic<uint64_t> &done, F set) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
    e = set();
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

// Launchers (return cudaError_t of the launch).  `pdl` enables
// programmatic dependent launch on the stream.
cudaError_t launch_rht_in(const RhtInParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_rht_out(const RhtOutParams &p, cudaStream_t s, bool pdl);
// row transforms for many rows (B up to 65535 per launch), len <= 16384
bool rht_rows_supported(int len);
cudaError_t launch_rht_rows(const RowsParams &p, bool input, int B, cudaStream_t s, bool pdl);
// the input side on the warp tensor cores (fp16 operand of the tensor-core
// GEMM; rows of 512 .. 16384 values, a multiple of 256, len == len_pad)
bool rht_in_mma_supported(const RowsParams &p);
cudaError_t launch_rht_in_mma(const RowsParams &p, int B, cudaStream_t s, bool pdl);
// one bounded wait of kind (0 cycle-bounded, 1 its cluster-scope form, 2
// poll-bounded) on a barrier `arrivals` of its two arrivals reach; a timeout
// sets GLQ_DEVERR_TIMEOUT in *err
cudaError_t launch_wait_selftest(unsigned *err, int kind, int arrivals, unsigned long long limit, cudaStream_t s);
cudaError_t launch_gemv(const GemvParams &p, int bpw, int grid, cudaStream_t s, bool pdl, bool fused_in = false);
// dynamic shared memory of a launch with the input transform fused
// (the table, the residual table, the task's activations and scratch)
size_t gemv_fused_smem_bytes(int table_words, int bpw, int B, int klen);
// dynamic shared memory of a launch with these parameters
size_t gemv_launch_smem_bytes(const GemvParams &p, int bpw, bool fin, int warps);
// partial sums of one CTA in the cluster reduction
size_t gemv_cluster_partials_bytes(int warps, int B);
// clusters of csize CTAs of the selected GEMV kernel that fit at once
int gemv_max_clusters(int bpw, int nt, bool fin, int warps, int csize, size_t smem);
// (227 KB per block, less room for the kernels' static shared memory)
constexpr size_t GEMV_SMEM_LIMIT = 222 * 1024;

// GEMV work split: bands of row tiles x splits of the chunk range.
struct GemvPlan {
    int bands, splits, cps, grid;
};
// Work split of the GEMV over a persistent grid.  pow2: chunks per split a
// power of two (aligned column ranges, required by the fused input
// transform), at most max_cps chunks per split and max_splits splits;
// charge: the cost of a split task's band reduction, in chunks.
GemvPlan plan_gemv(int RT, int KC, int num_sms, int warps, bool pow2 = false, int max_cps = 1 << 30,
                   int max_splits = 1 << 30, double charge = 0.5);
cudaError_t launch_dequant(const DequantParams &p, cudaStream_t s);
// Row-parallel shards (glq_shard.cu): per token, the exact sum of X over the
// columns [c0, c1) of the decode activations xq (rows of row_bytes bytes), with
// the token's scale copied from `in`; and an elementwise fp32 -> dtype cast.
cudaError_t launch_shard_rowsum(const uint8_t *xq, size_t row_bytes, int c0, int c1, const glq_rowinfo *in,
                                glq_rowinfo *out, int B, cudaStream_t s, bool pdl);
cudaError_t launch_cast(const float *src, void *dst, int dtype, int64_t count, cudaStream_t s);
// wmap: TMA map of the dequantised fp16 W [m_pad][n_pad] (boxes 64 x 128,
// 128-byte swizzle), or null for the fused variant whose producer warps
// rebuild W from the codes.
cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &xmap, const CUtensorMap *wmap, int grid,
                           cudaStream_t s, bool pdl);
// W16 [m_pad][n_pad] fp16 = cb1 + rs cb2 + ... (unscaled, every residual
// stage), for the materialised variant
cudaError_t launch_wmat(const PrefillParams &p, __half *w16, int n_pad, int num_sms, cudaStream_t s, bool pdl);
size_t wmat_smem_bytes(int table_words, int bpw);
size_t prefill_smem_bytes();
int prefill_tile_tokens();  // tokens of one output tile (a multiple of the TMA box height)
int prefill_tile_rows();    // weight rows of one output tile (one CTA pair)

// Work split of the tensor-core GEMM of an m_pad x (KC chunks of 128
// columns) layer over B tokens on num_sms SMs (host only): the K splits
// (chunk-aligned, chosen from a cost model of CTA-pair waves against the
// extra partial-sum traffic) and the work items; items [0, tiles_whole)
// are whole tiles, the rest halves (256 tokens) of the tiles after them,
// for a last partial wave of at most half the CTA pairs whose tiles all
// have two live halves.
struct PrefillSplit {
    int ksplit, tiles_tok, ntiles, tiles_whole;
};
PrefillSplit plan_prefill(int64_t m_pad, int KC, int64_t B, int num_sms);

// warps per GEMV CTA (one 16-row tile each): 24 for one 8-column MMA tile
// (B <= 8), 16 for two (B <= 16, more live registers per lane); from 5 bpw
// every residual stage adds its accumulators and code registers per lane,
// so 16 and 12
__host__ __device__ constexpr int gemv_warps(int nt, int bpw) {
    return bpw <= 4 ? (nt == 1 ? 24 : 16) : (nt == 1 ? 16 : 12);
}
// warps of the wide variant (one 8-column tile) for large layers, where the
// GEMV is bound by instruction issue and more warps hide more latency
// (measured on the 24B-class layers: -12 % per step against 24 warps)
constexpr int GEMV_WIDE_WARPS = 28;
constexpr int GEMV_PREFETCH = 1;
size_t gemv_smem_bytes(int table_words, int bpw);

}  // namespace glq
