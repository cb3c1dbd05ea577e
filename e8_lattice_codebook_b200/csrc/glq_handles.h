// glq_handles.h -- the opaque handle types of the C ABI (include/glq.h):
// what a codebook and a layer own on the host and on the device, and the
// decode launch sequence shared by glq_linear and glq_linear_noalloc.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/glq.h"
#include "glq_codebook_host.h"
#include "glq_internal.h"
#include "glq_kernels.cuh"

struct glq_codebook_s {
    int entries = 0;
    int device = 0;
    uint16_t *d_fp16 = nullptr;  // [entries][8]
    bool folded = false;
    glq::FoldedTable fold;
    uint32_t *d_table = nullptr;  // table_words words
    int table_words = 0;          // nb rounded up to a multiple of 4
    uint4 *d_table_f16 = nullptr; // fp16 codewords by folded code [2 nb - 1][8] (tensor-core path gathers)
};

// Device buffers one tensor-core call (B > 16 tokens) works in: a view of
// the device's shared workspace.
struct glq_prefill_ws {
    __half *xh = nullptr;         // [B][n_pad]
    glq_rowinfo *info = nullptr;  // [B]
    float *z = nullptr;           // [ksplit][B][m_pad]: K-split slices of [B][m_pad]
    __half *w16 = nullptr;        // [m_pad][n_pad] reconstructed W (batches >= the reconstruct bound)
};

// Device buffers one decode call works in (B <= 16 tokens): a view of the
// device's shared workspace, except cnt, which the layer owns.
// Columns the layer's index streams cover (n_pad for a whole layer).
inline int64_t stream_cols(glq_layer L);

struct glq_workspace {
    uint8_t *xq = nullptr;        // [B][n_pad * 2] activations, high / low bytes per group
    __half *xh = nullptr;         // [B][n_pad] fp16 activations (3 bpw only)
    glq_rowinfo *info = nullptr;  // [B]
    double *part = nullptr;       // [splits][B][m_pad] split-K partial sums
    float *z = nullptr;           // [B][m_pad]
    unsigned *cnt = nullptr;      // [bands], zero between calls
};

// Hadamard block decomposition of a size (descending powers of two)
struct glq_hblocks {
    int count = 0;
    int off[GLQ_MAX_BLOCKS] = {};
    int len[GLQ_MAX_BLOCKS] = {};
};

struct glq_layer_s {
    int64_t m = 0, n = 0, m_pad = 0, n_pad = 0;
    int bpw = 0, RT = 0, KC = 0, G = 0;  // KC, G: chunks / groups of the index streams (the shard's)
    // row-parallel shard: the layer holds input columns [kc0 * 128, kc0 * 128
    // + KC * 128) of n (a whole layer: kc0 = 0, KC * 128 = n_pad); its output
    // is the fp32 partial sum of those columns
    bool shard = false;
    int kc0 = 0;
    int device = 0, num_sms = 0;
    glq_codebook primary = nullptr, residual = nullptr;
    float ws = 0.f;
    uint4 *d_idx1 = nullptr;
    // residual stages ("Bit widths"): nres16 16-bit E8 stages, then an 8-bit
    // stage into the 256-entry table `residual` when has8 (odd bpw)
    int nres16 = 0;
    bool has8 = false;
    uint4 *d_res16[3] = {};       // fragment-native code streams of the 16-bit stages
    uint2 *d_res8 = nullptr;      // fragment-native index stream of the 8-bit stage
    float rs16[3] = {}, rs8 = 0.f;
    size_t idx_bytes = 0;         // all index streams on the device
    uint32_t *d_sin = nullptr, *d_sout = nullptr;
    glq::RhtPlan plan_n{}, plan_m{};
    unsigned *d_err = nullptr;
    // GEMV work split for B <= 8 (plan[0]) and B <= 16 (plan[1])
    glq::GemvPlan plan[2]{};
    // the transient buffers live in the device's shared workspace (sized by
    // glq_layer_reserve or on first use); the layer owns its band counters
    unsigned *d_cnt = nullptr;   // [bands] split-K arrival counters, zero between calls
    int64_t last_B = 0;          // batch of the last decode slice (glq_gemv_replay)
    int64_t last_prefill_B = 0;  // batch of the last tensor-core call (glq_prefill_replay)
    bool last_prefill_mat = false;
    glq_hblocks hb_n, hb_m;
    unsigned *d_blk_cnt = nullptr;  // [GLQ_MAX_BLOCKS] output-block counters, zero between calls
    int fusion = -1;                // GLQ_FUSE_* bits, or -1: the library default (glq_layer_set_fusion)
    bool invariant = false;         // every batch through the exact decode path (glq_layer_set_batch_invariant)
    int64_t prefill_mat_min_b = GLQ_DECODE_MAX_B + 1;  // batches from here reconstruct W16 first (glq_layer_set_prefill_reconstruct)
    // the last decode launch (glq_gemv_replay)
    const void *last_x = nullptr;
    void *last_y = nullptr;
    int last_x_bf16 = 0, last_y_dtype = 0;
    bool last_fin = false, last_fout = false;
    glq::GemvPlan last_plan{};
    size_t device_bytes = 0;
};

inline int64_t stream_cols(glq_layer L) { return (int64_t)L->KC * GLQ_CHUNK_K; }

namespace glq {

// How one decode call of nb <= 16 tokens runs: the GEMV split plan and
// whether the input / output transforms are fused into the GEMV launch.
struct DecodeCfg {
    GemvPlan plan{};
    bool fin = false, fout = false;
    int warps = 0;  // warps per GEMV CTA
    int clu = 0;    // split-K through a cluster of this many CTAs (0: global reduction)
    size_t spart_off = 0;  // shared-memory offset of the cluster partial sums
};

// max_splits: at most this many K splits (callers whose partial-sum buffer
// is small); x and y decide the fused paths' alignment condition.
DecodeCfg decode_config(glq_layer L, int nb, const void *x, const void *y, int y_dtype, int max_splits = 1 << 30);

// (input RHT ->) codebook GEMV (-> output RHT) for nb <= 16 tokens, in the
// buffers of `w`.
cudaError_t run_decode(glq_layer L, const glq_workspace &w, const DecodeCfg &cfg, const void *x, bool x_bf16,
                       void *y, int y_dtype, int nb, cudaStream_t s);

GemvParams gemv_params(glq_layer L, const glq_workspace &w, const DecodeCfg &cfg, int nb, const void *x,
                       bool x_bf16, void *y, int y_dtype);

inline const GemvPlan &plan_for(glq_layer L, int nb) { return L->plan[nb > 8 ? 1 : 0]; }

// largest split count any decode configuration of nb tokens can use
int max_decode_splits(glq_layer L, int nb);

// The decode configuration of the batch-invariant mode for a slice of nb
// <= 16 tokens: separate transforms and a split of the chunk range that
// does not depend on nb (the layer's one-token plan's chunks per split).
DecodeCfg invariant_config(glq_layer L, int nb);

}  // namespace glq
