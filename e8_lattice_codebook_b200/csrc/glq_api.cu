// glq_api.cu -- the C ABI of glq-b200 (include/glq.h): argument checks,
// the host-side re-layout of index arrays into the kernels' fragment-native
// streams, device memory ownership and kernel dispatch.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/glq.h"
#include "glq_codebook_host.h"
#include "glq_handles.h"
#include "glq_internal.h"
#include "glq_kernels.cuh"

using glq::FoldedTable;

namespace {

constexpr int64_t MAX_DIM = GLQ_RHT_MAX_N;

struct DeviceGuard {
    int prev = -1;
    bool switched = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
            switched = cudaSetDevice(dev) == cudaSuccess;
        }
    }
    ~DeviceGuard() {
        if (switched) cudaSetDevice(prev);
    }
};

bool all_signs(const int8_t *s, int64_t k) {
    for (int64_t i = 0; i < k; ++i)
        if (s[i] != 1 && s[i] != -1) return false;
    return true;
}

std::vector<uint32_t> pack_signs(const int8_t *s, int64_t k) {
    std::vector<uint32_t> bits((size_t)((k + 31) / 32 + 1), 0u);
    for (int64_t i = 0; i < k; ++i)
        if (s[i] < 0) bits[(size_t)(i >> 5)] |= 1u << (i & 31);
    return bits;
}

// block-diagonal Hadamard blocks of a size: its binary decomposition,
// descending powers of two at increasing offsets
glq_hblocks hadamard_blocks_of(int64_t k) {
    glq_hblocks hb;
    int64_t off = 0;
    for (int bit = 30; bit >= 0; --bit) {
        const int64_t sz = (int64_t)1 << bit;
        if (k & sz) {
            hb.off[hb.count] = (int)off;
            hb.len[hb.count] = (int)sz;
            ++hb.count;
            off += sz;
        }
    }
    return hb;
}

template <typename T>
glq_status dmalloc(T **p, size_t bytes, size_t *total) {
    *p = nullptr;
    if (bytes == 0) bytes = 16;
    if (cudaMalloc((void **)p, bytes) != cudaSuccess) {
        cudaGetLastError();
        return GLQ_ERR_OOM;
    }
    if (total) *total += bytes;
    return GLQ_OK;
}

void free_layer(glq_layer L) {
    if (!L) return;
    cudaFree(L->d_blk_cnt);
    cudaFree(L->d_idx1);
    for (int k = 0; k < 3; ++k) cudaFree(L->d_res16[k]);
    cudaFree(L->d_res8);
    cudaFree(L->d_sin);
    cudaFree(L->d_sout);
    cudaFree(L->d_err);
    cudaFree(L->d_cnt);
    delete L;
}

// ---------------------------------------------------------------------------
// The device's shared workspace: every transient buffer of glq_linear, for
// all layers on the device.  Each buffer grows to the largest size a call or
// a reservation has asked for; growth synchronises the device and frees the
// previous buffer (so work captured in a CUDA graph before a growth must not
// be replayed after it: reserve first).  Calls that use it must be serialised
// on the GPU (one stream, or explicit ordering).
// ---------------------------------------------------------------------------

enum WsBuf { WS_XQ, WS_XH, WS_INFO, WS_PART, WS_Z, WS_PXH, WS_PINFO, WS_PZ, WS_W16, WS_COUNT };

struct DeviceWs {
    void *buf[WS_COUNT] = {};
    size_t cap[WS_COUNT] = {};
};

constexpr int WS_MAX_DEVICES = 128;
std::mutex g_ws_mu;
DeviceWs g_ws[WS_MAX_DEVICES];

struct WsNeed {
    size_t b[WS_COUNT] = {};
};

size_t ws_bytes_locked(int dev) {
    size_t t = 0;
    for (int i = 0; i < WS_COUNT; ++i) t += g_ws[dev].cap[i];
    return t;
}

// Makes every buffer of `dev` (the current device) at least `need` bytes and
// returns their addresses.  `s` is the stream of the call: if it is being
// captured and a buffer must grow, nothing is allocated (GLQ_ERR_CAPTURE).
glq_status ws_acquire(int dev, const WsNeed &need, cudaStream_t s, void *out[WS_COUNT]) {
    if (dev < 0 || dev >= WS_MAX_DEVICES) return GLQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_ws_mu);
    DeviceWs &w = g_ws[dev];
    bool grow = false;
    for (int i = 0; i < WS_COUNT; ++i) grow |= need.b[i] > w.cap[i];
    if (grow) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
            cudaGetLastError();
            return GLQ_ERR_CUDA;
        }
        if (cs != cudaStreamCaptureStatusNone) return GLQ_ERR_CAPTURE;
        if (cudaDeviceSynchronize() != cudaSuccess) {
            cudaGetLastError();
            return GLQ_ERR_CUDA;
        }
        for (int i = 0; i < WS_COUNT; ++i) {
            if (need.b[i] <= w.cap[i]) continue;
            cudaFree(w.buf[i]);
            w.buf[i] = nullptr;
            w.cap[i] = 0;
            const size_t bytes = (need.b[i] + 255) & ~(size_t)255;
            if (cudaMalloc(&w.buf[i], bytes) != cudaSuccess) {
                cudaGetLastError();
                w.buf[i] = nullptr;
                return GLQ_ERR_OOM;
            }
            w.cap[i] = bytes;
        }
    }
    for (int i = 0; i < WS_COUNT; ++i) out[i] = w.buf[i];
    return GLQ_OK;
}

// Decode buffers for calls of up to `rows` (<= 16) tokens on layer L.
void decode_need(glq_layer L, int64_t rows, WsNeed &n) {
    if (rows <= 0) return;
    rows = std::min<int64_t>(rows, GLQ_DECODE_MAX_B);
    int max_splits = 1;
    for (int nb = 1; nb <= rows; ++nb) max_splits = std::max(max_splits, glq::max_decode_splits(L, nb));
    n.b[WS_XQ] = std::max(n.b[WS_XQ], (size_t)rows * L->n_pad * 2);
    if (L->has8) n.b[WS_XH] = std::max(n.b[WS_XH], (size_t)rows * L->n_pad * sizeof(__half));
    // a shard also keeps the row sums over its own columns, after 16 rows
    n.b[WS_INFO] = std::max(n.b[WS_INFO], (L->shard ? 2 * GLQ_DECODE_MAX_B : rows) * sizeof(glq_rowinfo));
    if (max_splits > 1)
        n.b[WS_PART] = std::max(n.b[WS_PART], (size_t)max_splits * rows * L->m_pad * sizeof(double));
    n.b[WS_Z] = std::max(n.b[WS_Z], (size_t)rows * L->m_pad * sizeof(float));
}

// Buffers of a batch-invariant call of B tokens: activations, row info and
// outputs for every token, split-K partial sums for one 16-token slice.
void invariant_need(glq_layer L, int64_t B, WsNeed &n) {
    decode_need(L, std::min<int64_t>(B, GLQ_DECODE_MAX_B), n);
    n.b[WS_XQ] = std::max(n.b[WS_XQ], (size_t)B * L->n_pad * 2);
    if (L->has8) n.b[WS_XH] = std::max(n.b[WS_XH], (size_t)B * L->n_pad * sizeof(__half));
    n.b[WS_INFO] = std::max(n.b[WS_INFO], (size_t)B * sizeof(glq_rowinfo));
    n.b[WS_Z] = std::max(n.b[WS_Z], (size_t)B * L->m_pad * sizeof(float));
}

// Tensor-core buffers for one call of exactly B (> 16) tokens on layer L.
void prefill_need(glq_layer L, int64_t B, WsNeed &n) {
    const int ks = glq::plan_prefill(L->m_pad, L->KC, B, L->num_sms).ksplit;
    n.b[WS_PXH] = std::max(n.b[WS_PXH], (size_t)B * L->n_pad * sizeof(__half));
    n.b[WS_PINFO] = std::max(n.b[WS_PINFO], (size_t)B * sizeof(glq_rowinfo));
    n.b[WS_PZ] = std::max(n.b[WS_PZ], (size_t)ks * B * L->m_pad * sizeof(float));
    if (B >= L->prefill_mat_min_b)
        n.b[WS_W16] = std::max(n.b[WS_W16], (size_t)L->m_pad * stream_cols(L) * sizeof(__half));
}

glq_workspace decode_view(glq_layer L, void *const buf[WS_COUNT]) {
    glq_workspace w;
    w.xq = static_cast<uint8_t *>(buf[WS_XQ]);
    // the fp16 activations exist for the 8-bit stage only: the buffer may be
    // held (sized by an odd-bpw layer) while this layer needs none, and a
    // non-null pointer makes the input transform write it
    w.xh = L->has8 ? static_cast<__half *>(buf[WS_XH]) : nullptr;
    w.info = static_cast<glq_rowinfo *>(buf[WS_INFO]);
    w.part = static_cast<double *>(buf[WS_PART]);
    w.z = static_cast<float *>(buf[WS_Z]);
    w.cnt = L->d_cnt;
    return w;
}

glq_prefill_ws prefill_view(void *const buf[WS_COUNT]) {
    glq_prefill_ws w;
    w.xh = static_cast<__half *>(buf[WS_PXH]);
    w.info = static_cast<glq_rowinfo *>(buf[WS_PINFO]);
    w.z = static_cast<float *>(buf[WS_PZ]);
    w.w16 = static_cast<__half *>(buf[WS_W16]);
    return w;
}

// TMA descriptor of the fp16 activations [B][n_pad]: boxes of 64 columns x
// 128 tokens, 128-byte swizzle, zero fill past the last token.
// TMA descriptor of the reconstructed W16 [m_pad][n_pad]: boxes of 64 columns
// x 128 rows, 128-byte swizzle.
bool encode_w_map(CUtensorMap *map, const __half *w16, int64_t n_pad, int64_t m_pad);

// cols columns of rows `ld` fp16 apart (a shard reads its column range of the
// whole rows)
bool encode_x_map(CUtensorMap *map, const __half *xh, int64_t cols, int64_t B, int64_t ld) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn) {
            cudaGetLastError();
            return false;
        }
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)B};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * sizeof(__half)};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half *>(xh), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tcgen05 GEMM of the tensor-core path on the layer's prefill
// workspace: z[0..B) from xh[0..B).
bool encode_w_map(CUtensorMap *map, const __half *w16, int64_t n_pad, int64_t m_pad) {
    // same layout rules as the activations: rows of n_pad fp16, 128-byte swizzle
    return encode_x_map(map, w16, n_pad, m_pad, n_pad);
}

glq::PrefillParams prefill_params(glq_layer L, const glq_prefill_ws &ws, int64_t B) {
    glq::PrefillParams pp{};
    pp.idx1 = L->d_idx1;
    for (int k = 0; k < 3; ++k) {
        pp.idx16[k] = L->d_res16[k];
        const __half2 h = __floats2half2_rn(L->rs16[k], L->rs16[k]);
        pp.rs16_h2[k] = *reinterpret_cast<const uint32_t *>(&h);
    }
    pp.idx8 = L->d_res8;
    const __half2 h8 = __floats2half2_rn(L->rs8, L->rs8);
    pp.rs8_h2 = *reinterpret_cast<const uint32_t *>(&h8);
    pp.cb_f16 = L->primary->d_table_f16;
    pp.tab8 = L->has8 ? reinterpret_cast<const uint4 *>(L->residual->d_fp16) : nullptr;
    pp.bpw = L->bpw;
    pp.info = ws.info;
    pp.ws = L->ws;
    pp.z = ws.z;
    pp.B = (int)B;
    pp.m_pad = (int)L->m_pad;
    pp.KC = L->KC;
    pp.RT = L->RT;
    const glq::PrefillSplit ps = glq::plan_prefill(L->m_pad, L->KC, B, L->num_sms);
    pp.tiles_tok = ps.tiles_tok;
    pp.ksplit = ps.ksplit;
    pp.ntiles = ps.ntiles;
    pp.tiles_whole = ps.tiles_whole;
    pp.zs = (size_t)B * L->m_pad;
    pp.err = L->d_err;
    pp.table = L->primary->d_table;
    pp.table_words = L->primary->table_words;
    pp.fold = glq::FoldParams{L->primary->fold.nb, L->primary->fold.neg_base};
    return pp;
}

// The tcgen05 GEMM of the tensor-core path on the layer's prefill
// workspace: z[0..B) from xh[0..B); mat: against the reconstructed W16.
cudaError_t launch_prefill_gemm(glq_layer L, const glq_prefill_ws &ws, int64_t B, bool mat, cudaStream_t s,
                                bool pdl) {
    CUtensorMap xmap, wmap;
    const int64_t k0 = (int64_t)L->kc0 * GLQ_CHUNK_K;  // a shard's first column (256-byte aligned)
    if (!encode_x_map(&xmap, ws.xh + k0, stream_cols(L), B, L->n_pad)) return cudaErrorInvalidValue;
    if (mat && !encode_w_map(&wmap, ws.w16, stream_cols(L), L->m_pad)) return cudaErrorInvalidValue;
    const glq::PrefillParams pp = prefill_params(L, ws, B);
    const int grid = 2 * std::min(pp.ntiles, L->num_sms / 2);  // CTA pairs
    return glq::launch_prefill(pp, xmap, mat ? &wmap : nullptr, grid, s, pdl);
}

glq::RowsParams rows_params(const glq_hblocks &hb, int len, int len_pad, const uint32_t *signs) {
    glq::RowsParams r{};
    r.len = len;
    r.len_pad = len_pad;
    r.nblk = hb.count;
    r.max_blk = hb.count ? hb.len[0] : 0;
    for (int i = 0; i < hb.count; ++i) {
        r.blk_off[i] = hb.off[i];
        r.blk_len[i] = hb.len[i];
        r.blk_norm[i] = (float)(1.0 / std::sqrt((double)hb.len[i]));
    }
    r.sign_bits = signs;
    r.zsplits = 1;
    r.zs = 0;
    return r;
}

// Tensor-core path for B > 16 tokens: input RHT (fp16 activations), tcgen05
// GEMM with the dequantising producer, output RHT.  Rows of up to 16384
// values use the one-CTA-per-row transform kernels; longer rows the
// clustered ones.
glq_status run_prefill(glq_layer L, const void *x, bool x_bf16, void *y, int y_dtype, int64_t B, cudaStream_t s) {
    const bool mat = B >= L->prefill_mat_min_b;
    WsNeed need;
    prefill_need(L, B, need);
    void *buf[WS_COUNT];
    glq_status st = ws_acquire(L->device, need, s, buf);
    if (st != GLQ_OK) return st;
    const glq_prefill_ws ws = prefill_view(buf);
    const int ksplit = prefill_params(L, ws, B).ksplit;
    const bool rows_in = glq::rht_rows_supported((int)L->n_pad), rows_out = glq::rht_rows_supported((int)L->m);
    for (int64_t b0 = 0; b0 < B;) {
        const int nb = (int)std::min<int64_t>(B - b0, 65535);  // grid limit of the clustered kernels
        if (rows_in) {
            glq::RowsParams r = rows_params(L->hb_n, (int)L->n, (int)L->n_pad, L->d_sin);
            r.x = static_cast<const char *>(x) + (size_t)b0 * L->n * 2;
            r.x_bf16 = x_bf16 ? 1 : 0;
            r.xh = ws.xh + (size_t)b0 * L->n_pad;
            r.info = ws.info + b0;
            if (glq::launch_rht_rows(r, true, nb, s, true) != cudaSuccess) return GLQ_ERR_CUDA;
        } else {
            glq::RhtInParams pin{};
            pin.x = static_cast<const char *>(x) + (size_t)b0 * L->n * 2;
            pin.x_bf16 = x_bf16 ? 1 : 0;
            pin.n = (int)L->n;
            pin.n_pad = (int)L->n_pad;
            pin.B = nb;
            pin.sign_bits = L->d_sin;
            pin.plan = L->plan_n;
            pin.xh = ws.xh + (size_t)b0 * L->n_pad;
            pin.info = ws.info + b0;
            pin.xh_only = 1;
            if (glq::launch_rht_in(pin, s, true) != cudaSuccess) return GLQ_ERR_CUDA;
        }
        b0 += nb;
    }
    if (mat && glq::launch_wmat(prefill_params(L, ws, B), ws.w16, (int)stream_cols(L), L->num_sms, s, true) !=
                   cudaSuccess)
        return GLQ_ERR_CUDA;
    // The dequantising-producer variant is launched without programmatic
    // dependent launch: started early behind the previous kernels, calls
    // issued back to back stalled until a bounded wait gave up (measured:
    // 8B-class layers at 17-64 tokens); launched after its predecessor
    // completes, they do not.
    if (launch_prefill_gemm(L, ws, B, mat, s, mat) != cudaSuccess) return GLQ_ERR_CUDA;
    L->last_prefill_B = B;
    L->last_prefill_mat = mat;
    for (int64_t b0 = 0; b0 < B;) {
        const int nb = (int)std::min<int64_t>(B - b0, 65535);
        void *yb = static_cast<char *>(y) + (size_t)b0 * L->m * (y_dtype == GLQ_F32 ? 4 : 2);
        if (rows_out) {
            glq::RowsParams r = rows_params(L->hb_m, (int)L->m, (int)L->m, L->d_sout);
            r.z = ws.z + (size_t)b0 * L->m_pad;
            r.z_ld = (int)L->m_pad;
            r.zsplits = ksplit;
            r.zs = (size_t)B * L->m_pad;
            r.y = yb;
            r.y_dtype = y_dtype;
            if (glq::launch_rht_rows(r, false, nb, s, true) != cudaSuccess) return GLQ_ERR_CUDA;
        } else {
            glq::RhtOutParams pout{};
            pout.m = (int)L->m;
            pout.B = nb;
            pout.z = ws.z + (size_t)b0 * L->m_pad;
            pout.z_ld = (int)L->m_pad;
            pout.sign_bits = L->d_sout;
            pout.plan = L->plan_m;
            pout.y = yb;
            pout.y_dtype = y_dtype;
            if (glq::launch_rht_out(pout, s, true) != cudaSuccess) return GLQ_ERR_CUDA;
        }
        b0 += nb;
    }
    return GLQ_OK;
}

}  // namespace

namespace glq {

// fused transforms: at most this many values (tokens x largest Hadamard
// block) are folded per task (input) or rotated by one CTA (output)
constexpr long long FUSED_IN_MAX_VALUES = 32768;
constexpr long long FUSED_OUT_MAX_VALUES = 32768;
// Measured on B200 (CUDA graphs, B = 1 and 8): fusing the input transform
// saves a launch when every CTA has one short task (below); the output
// transform done by one CTA at the end of the GEMV is slower than the
// separate, parallel kernel at every size measured, so it is off by default.
constexpr int FUSE_DEFAULT_FLAGS = GLQ_FUSE_INPUT | GLQ_SPLITK_CLUSTER;

void choose_cluster(glq_layer L, int nb, int flags, DecodeCfg &c);

DecodeCfg decode_config(glq_layer L, int nb, const void *x, const void *y, int y_dtype, int max_splits) {
    DecodeCfg c;
    const int nt = nb > 8 ? 2 : 1;
    const int warps = gemv_warps(nt, L->bpw);
    const size_t base = gemv_smem_bytes(L->primary->table_words, L->bpw);
    const bool x_al = (reinterpret_cast<uintptr_t>(x) & 15) == 0;
    const bool y_al = (reinterpret_cast<uintptr_t>(y) & 15) == 0;
    (void)y_dtype;
    const int flags = L->fusion < 0 ? FUSE_DEFAULT_FLAGS : L->fusion;
    c.fout = !L->shard && (flags & GLQ_FUSE_OUTPUT) && y_al && (long long)nb * L->hb_m.len[0] <= FUSED_OUT_MAX_VALUES &&
             (size_t)nb * L->hb_m.len[0] * sizeof(float) <= base;
    c.warps = warps;
    if (!L->shard && (flags & GLQ_FUSE_INPUT) && x_al && (long long)nb * L->hb_n.len[0] <= FUSED_IN_MAX_VALUES) {
        int cap = 1;  // largest power-of-two chunk count whose activations fit shared memory
        while (cap < L->KC &&
               gemv_fused_smem_bytes(L->primary->table_words, L->bpw, nb, std::min(cap * 2, L->KC) * GLQ_CHUNK_K) <=
                   GEMV_SMEM_LIMIT)
            cap *= 2;
        const GemvPlan fp = plan_gemv(L->RT, L->KC, L->num_sms, warps, true, cap, max_splits);
        const size_t need =
            gemv_fused_smem_bytes(L->primary->table_words, L->bpw, nb, std::min(fp.cps, L->KC) * GLQ_CHUNK_K);
        // Measured: the fold pays for the launch it saves when every CTA has
        // one task and a short range (<= 1024 columns, <= 4096 values in
        // all), and the row is long enough (n_pad > 8192) that the separate
        // transform is a slow one-CTA row; for shorter rows the separate
        // transform, launched early behind the previous kernel, costs less
        // (steps back to back: 24B-class 153.7 -> 149.8 us, SmolLM3-3B-shaped
        // 77.3 -> 75.0 us, SmolLM2-360M-shaped at two tokens 60.7 -> 54.1 us).
        // A 4096-column range per CTA is slower than the separate transform
        // kernel.  An explicit setting always fuses.  (Narrower CTAs of 16 or
        // 20 warps that fill more SMs made the 3B-shaped step slower, 74 -> 82
        // us: no SM was left for the next kernel's early launch.)
        const int klen = std::min(fp.cps, L->KC) * GLQ_CHUNK_K;
        const bool cheap = (long long)fp.bands * fp.splits <= L->num_sms && klen <= 1024 && nb * klen <= 4096 &&
                           L->n_pad > 8192;
        if (need <= GEMV_SMEM_LIMIT && (cheap || L->fusion >= 0)) {
            c.fin = true;
            c.plan = fp;
        }
    }
    if (!c.fin) {
        c.plan = plan_for(L, nb);
        if (nt == 1 && L->bpw <= 4 && (long long)L->RT * L->KC >= 200LL * L->num_sms) {  // large layer: wide CTAs
            c.warps = GEMV_WIDE_WARPS;
            c.plan = plan_gemv(L->RT, L->KC, L->num_sms, c.warps);
        }
        if (c.plan.splits > max_splits)
            c.plan = plan_gemv(L->RT, L->KC, L->num_sms, c.warps, false, 1 << 30, max_splits);
    }
    choose_cluster(L, nb, flags, c);
    return c;
}

// Split-K through a thread-block cluster: one task per CTA, the band's
// splits in one cluster (at most 16), all clusters resident at once.  The
// summation order is that of the global reduction.
void choose_cluster(glq_layer L, int nb, int flags, DecodeCfg &c) {
    const int nt = nb > 8 ? 2 : 1;
    const int S = c.plan.splits;
    if ((flags & GLQ_SPLITK_CLUSTER) && S > 1 && S <= 16 && !c.fout &&
        (long long)c.plan.bands * S == (long long)c.plan.grid) {
        const size_t base = c.fin ? gemv_fused_smem_bytes(L->primary->table_words, L->bpw, nb,
                                                          std::min(c.plan.cps, L->KC) * GLQ_CHUNK_K)
                                  : gemv_smem_bytes(L->primary->table_words, L->bpw);
        const size_t off = (base + 255) & ~(size_t)255;
        const size_t need = off + gemv_cluster_partials_bytes(c.warps, nb);
        if (need <= GEMV_SMEM_LIMIT && gemv_max_clusters(L->bpw, nt, c.fin, c.warps, S, need) >= c.plan.bands) {
            c.clu = S;
            c.spart_off = off;
        }
    }
}

DecodeCfg invariant_config(glq_layer L, int nb) {
    DecodeCfg c;
    const int nt = nb > 8 ? 2 : 1;
    c.warps = gemv_warps(nt, L->bpw);
    // the chunks per split of the layer's one-token plan, for every slice
    const int cps = L->plan[0].cps;
    c.plan.cps = cps;
    c.plan.splits = (L->KC + cps - 1) / cps;
    c.plan.bands = (L->RT + c.warps - 1) / c.warps;
    const long long tasks = (long long)c.plan.bands * c.plan.splits;
    c.plan.grid = (int)std::min<long long>(tasks, L->num_sms);
    const int flags = L->fusion < 0 ? FUSE_DEFAULT_FLAGS : L->fusion;
    choose_cluster(L, nb, flags, c);
    return c;
}

int max_decode_splits(glq_layer L, int nb) {
    const int warps = gemv_warps(nb > 8 ? 2 : 1, L->bpw);
    int cap = 1;
    while (cap < L->KC &&
           gemv_fused_smem_bytes(L->primary->table_words, L->bpw, nb, std::min(cap * 2, L->KC) * GLQ_CHUNK_K) <=
               GEMV_SMEM_LIMIT)
        cap *= 2;
    const int fs = plan_gemv(L->RT, L->KC, L->num_sms, warps, true, cap).splits;
    const int ws = L->bpw <= 4 ? plan_gemv(L->RT, L->KC, L->num_sms, GEMV_WIDE_WARPS).splits : 1;
    return std::max(std::max(plan_for(L, nb).splits, fs), ws);
}

GemvParams gemv_params(glq_layer L, const glq_workspace &w, const DecodeCfg &cfg, int nb, const void *x,
                       bool x_bf16, void *y, int y_dtype) {
    const GemvPlan &plan = cfg.plan;
    GemvParams p{};
    p.idx1 = L->d_idx1;
    double rsum = 0.0;
    for (int k = 0; k < 3; ++k) {
        p.idx16[k] = L->d_res16[k];
        p.rs16_d[k] = k < L->nres16 ? (double)L->rs16[k] : 0.0;
        rsum += p.rs16_d[k];
    }
    p.idx8 = L->d_res8;
    p.rs8_d = L->has8 ? 2.0 * (double)L->rs8 : 0.0;
    p.corr_mult = 1.0 + rsum;
    p.table = L->primary->d_table;
    p.table_words = L->primary->table_words;
    p.fold = FoldParams{L->primary->fold.nb, L->primary->fold.neg_base};
    p.kc = LookupConsts{4u, 16u, 0xFFFFFFFFu};
    p.tab8 = L->has8 ? reinterpret_cast<const uint4 *>(L->residual->d_fp16) : nullptr;
    // a shard reads its column range of the activation rows, and the row
    // sums over that range (stored after the first 16 rows of row info)
    const int64_t k0 = (int64_t)L->kc0 * GLQ_CHUNK_K;
    p.xq = w.xq ? w.xq + k0 * 2 : nullptr;
    p.xh = w.xh ? w.xh + k0 : nullptr;
    p.info = L->shard ? w.info + GLQ_DECODE_MAX_B : w.info;
    p.B = nb;
    p.n_pad = (int)L->n_pad;
    p.KC = L->KC;
    p.RT = L->RT;
    p.bands = plan.bands;
    p.splits = plan.splits;
    p.cps = plan.cps;
    p.ws = L->ws;
    p.partials = w.part;
    p.counters = w.cnt;
    p.z = w.z;
    p.m_pad = (int)L->m_pad;
    p.err = L->d_err;
    p.warps = cfg.warps;
    // fused transforms
    p.x = x;
    p.x_bf16 = x_bf16 ? 1 : 0;
    p.n = (int)L->n;
    p.sin_bits = L->d_sin;
    p.nblk_n = L->hb_n.count;
    for (int i = 0; i < L->hb_n.count; ++i) {
        p.blk_off_n[i] = L->hb_n.off[i];
        p.blk_len_n[i] = L->hb_n.len[i];
    }
    p.fuse_out = cfg.fout ? 1 : 0;
    p.clu = cfg.clu;
    p.spart_off = cfg.spart_off;
    p.y = y;
    p.y_dtype = y_dtype;
    p.m = (int)L->m;
    p.sout_bits = L->d_sout;
    p.nblk_m = L->hb_m.count;
    const int band_rows = cfg.warps * GLQ_ROW_TILE;
    for (int i = 0; i < L->hb_m.count; ++i) {
        const int o = L->hb_m.off[i], N = L->hb_m.len[i];
        p.blk_off_m[i] = o;
        p.blk_len_m[i] = N;
        int cnt = 0;
        for (int band = 0; band < plan.bands; ++band) {
            const int r0 = band * band_rows, r1 = std::min<int>(r0 + band_rows, (int)L->m);
            if (r0 < o + N && o < r1) ++cnt;
        }
        p.blk_bands[i] = cnt;
    }
    p.blk_cnt = L->d_blk_cnt;
    return p;
}

cudaError_t run_decode(glq_layer L, const glq_workspace &w, const DecodeCfg &cfg, const void *x, bool x_bf16,
                       void *y, int y_dtype, int nb, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    if (!cfg.fin) {
        if (rht_rows_supported((int)L->n_pad)) {  // one CTA per token
            RowsParams r = rows_params(L->hb_n, (int)L->n, (int)L->n_pad, L->d_sin);
            r.x = x;
            r.x_bf16 = x_bf16 ? 1 : 0;
            r.xq = w.xq;
            r.xh = w.xh;
            r.info = w.info;
            e = launch_rht_rows(r, true, nb, s, true);
        } else {
            RhtInParams pin{};
            pin.x = x;
            pin.x_bf16 = x_bf16 ? 1 : 0;
            pin.n = (int)L->n;
            pin.n_pad = (int)L->n_pad;
            pin.B = nb;
            pin.sign_bits = L->d_sin;
            pin.plan = L->plan_n;
            pin.xq = w.xq;
            pin.xh = w.xh;
            pin.info = w.info;
            e = launch_rht_in(pin, s, true);
        }
        if (e != cudaSuccess) return e;
        if (L->shard) {  // the row sums of X over the shard's columns
            const int c0 = L->kc0 * GLQ_CHUNK_K;
            const int c1 = (int)std::min<int64_t>(c0 + stream_cols(L), L->n);
            e = launch_shard_rowsum(w.xq, (size_t)L->n_pad * 2, c0, c1, w.info, w.info + GLQ_DECODE_MAX_B, nb, s,
                                    true);
            if (e != cudaSuccess) return e;
        }
    }
    e = launch_gemv(gemv_params(L, w, cfg, nb, x, x_bf16, y, y_dtype), L->bpw, cfg.plan.grid, s, true, cfg.fin);
    if (e != cudaSuccess || cfg.fout) return e;
    // one CTA per row, except for one or two long rows, where the clustered
    // kernel spreads a row over several SMs (measured: 0.6 us less at m = 11008, B = 1)
    if (rht_rows_supported((int)L->m) && (nb > 2 || L->m <= 8192)) {
        RowsParams r = rows_params(L->hb_m, (int)L->m, (int)L->m, L->d_sout);
        r.z = w.z;
        r.z_ld = (int)L->m_pad;
        r.y = y;
        r.y_dtype = y_dtype;
        return launch_rht_rows(r, false, nb, s, true);
    }
    RhtOutParams pout{};
    pout.m = (int)L->m;
    pout.B = nb;
    pout.z = w.z;
    pout.z_ld = (int)L->m_pad;
    pout.sign_bits = L->d_sout;
    pout.plan = L->plan_m;
    pout.y = y;
    pout.y_dtype = y_dtype;
    return launch_rht_out(pout, s, true);
}

// The batch-invariant mode (glq_layer_set_batch_invariant): every batch
// takes the exact decode arithmetic.  The input transform (the kernel chosen
// by n alone) rotates and quantises every token, the GEMV runs on slices of
// at most 16 tokens with the split plan of invariant_config (the same for
// every slice size), and the output transform (the kernel chosen by m alone)
// rotates every token: each token's y is the same bits whatever the batch.
glq_status run_invariant(glq_layer L, const void *x, bool x_bf16, void *y, int y_dtype, int64_t B,
                         cudaStream_t s, void *const buf[], size_t xq_row_bytes) {
    glq_workspace w;
    w.xq = static_cast<uint8_t *>(buf[0]);
    w.xh = L->has8 ? static_cast<__half *>(buf[1]) : nullptr;  // 8-bit stage only
    w.info = static_cast<glq_rowinfo *>(buf[2]);
    w.part = static_cast<double *>(buf[3]);
    w.z = static_cast<float *>(buf[4]);
    w.cnt = L->d_cnt;
    for (int64_t b0 = 0; b0 < B;) {  // input transform, every token
        const int nb = (int)std::min<int64_t>(B - b0, 65535);
        const void *xb = static_cast<const char *>(x) + (size_t)b0 * L->n * 2;
        cudaError_t e;
        if (rht_rows_supported((int)L->n_pad)) {
            RowsParams r{};
            r.len = (int)L->n;
            r.len_pad = (int)L->n_pad;
            r.nblk = L->hb_n.count;
            r.max_blk = L->hb_n.count ? L->hb_n.len[0] : 0;
            for (int i = 0; i < L->hb_n.count; ++i) {
                r.blk_off[i] = L->hb_n.off[i];
                r.blk_len[i] = L->hb_n.len[i];
                r.blk_norm[i] = (float)(1.0 / std::sqrt((double)L->hb_n.len[i]));
            }
            r.sign_bits = L->d_sin;
            r.zsplits = 1;
            r.x = xb;
            r.x_bf16 = x_bf16 ? 1 : 0;
            r.xq = w.xq + (size_t)b0 * xq_row_bytes;
            r.xh = w.xh ? w.xh + (size_t)b0 * L->n_pad : nullptr;
            r.info = w.info + b0;
            e = launch_rht_rows(r, true, nb, s, true);
        } else {
            RhtInParams pin{};
            pin.x = xb;
            pin.x_bf16 = x_bf16 ? 1 : 0;
            pin.n = (int)L->n;
            pin.n_pad = (int)L->n_pad;
            pin.B = nb;
            pin.sign_bits = L->d_sin;
            pin.plan = L->plan_n;
            pin.xq = w.xq + (size_t)b0 * xq_row_bytes;
            pin.xh = w.xh ? w.xh + (size_t)b0 * L->n_pad : nullptr;
            pin.info = w.info + b0;
            e = launch_rht_in(pin, s, true);
        }
        if (e != cudaSuccess) return GLQ_ERR_CUDA;
        b0 += nb;
    }
    for (int64_t b0 = 0; b0 < B; b0 += GLQ_DECODE_MAX_B) {  // GEMV, 16 tokens at a time
        const int nb = (int)std::min<int64_t>(B - b0, GLQ_DECODE_MAX_B);
        glq_workspace ws = w;
        ws.xq = w.xq + (size_t)b0 * xq_row_bytes;
        ws.xh = w.xh ? w.xh + (size_t)b0 * L->n_pad : nullptr;
        ws.info = w.info + b0;
        ws.z = w.z + (size_t)b0 * L->m_pad;
        const DecodeCfg cfg = invariant_config(L, nb);
        if (launch_gemv(gemv_params(L, ws, cfg, nb, nullptr, x_bf16, nullptr, y_dtype), L->bpw, cfg.plan.grid, s,
                        true, false) != cudaSuccess)
            return GLQ_ERR_CUDA;
    }
    for (int64_t b0 = 0; b0 < B;) {  // output transform, every token
        const int nb = (int)std::min<int64_t>(B - b0, 65535);
        void *yb = static_cast<char *>(y) + (size_t)b0 * L->m * (y_dtype == GLQ_F32 ? 4 : 2);
        cudaError_t e;
        if (rht_rows_supported((int)L->m)) {
            RowsParams r{};
            r.len = (int)L->m;
            r.len_pad = (int)L->m;
            r.nblk = L->hb_m.count;
            r.max_blk = L->hb_m.count ? L->hb_m.len[0] : 0;
            for (int i = 0; i < L->hb_m.count; ++i) {
                r.blk_off[i] = L->hb_m.off[i];
                r.blk_len[i] = L->hb_m.len[i];
                r.blk_norm[i] = (float)(1.0 / std::sqrt((double)L->hb_m.len[i]));
            }
            r.sign_bits = L->d_sout;
            r.zsplits = 1;
            r.z = w.z + (size_t)b0 * L->m_pad;
            r.z_ld = (int)L->m_pad;
            r.y = yb;
            r.y_dtype = y_dtype;
            e = launch_rht_rows(r, false, nb, s, true);
        } else {
            RhtOutParams pout{};
            pout.m = (int)L->m;
            pout.B = nb;
            pout.z = w.z + (size_t)b0 * L->m_pad;
            pout.z_ld = (int)L->m_pad;
            pout.sign_bits = L->d_sout;
            pout.plan = L->plan_m;
            pout.y = yb;
            pout.y_dtype = y_dtype;
            e = launch_rht_out(pout, s, true);
        }
        if (e != cudaSuccess) return GLQ_ERR_CUDA;
        b0 += nb;
    }
    return GLQ_OK;
}

}  // namespace glq

extern "C" {

const char *glq_status_str(glq_status s) {
    switch (s) {
        case GLQ_OK: return "GLQ_OK";
        case GLQ_ERR_INVALID_ARG: return "GLQ_ERR_INVALID_ARG";
        case GLQ_ERR_SHAPE: return "GLQ_ERR_SHAPE";
        case GLQ_ERR_DTYPE: return "GLQ_ERR_DTYPE";
        case GLQ_ERR_BPW: return "GLQ_ERR_BPW";
        case GLQ_ERR_NO_CODEBOOK: return "GLQ_ERR_NO_CODEBOOK";
        case GLQ_ERR_OOM: return "GLQ_ERR_OOM";
        case GLQ_ERR_CUDA: return "GLQ_ERR_CUDA";
        case GLQ_ERR_DEVICE_CHECK: return "GLQ_ERR_DEVICE_CHECK";
        case GLQ_ERR_TIMEOUT: return "GLQ_ERR_TIMEOUT";
        case GLQ_ERR_UNSUPPORTED: return "GLQ_ERR_UNSUPPORTED";
        case GLQ_ERR_CAPTURE: return "GLQ_ERR_CAPTURE";
    }
    return "GLQ_ERR_UNKNOWN";
}

const char *glq_version(void) { return "glq-b200 0.1.0 (sm_100a)"; }

glq_status glq_e8_codebook(uint16_t *out_fp16_bits) {
    if (!out_fp16_bits) return GLQ_ERR_INVALID_ARG;
    glq::build_e8_codebook(out_fp16_bits);
    return GLQ_OK;
}

glq_status glq_codebook_upload(const uint16_t *host_fp16_bits, int32_t entries, int32_t dim,
                               glq_codebook *out) {
    if (!host_fp16_bits || !out) return GLQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (dim != GLQ_DIM || (entries != GLQ_CB_ENTRIES && entries != GLQ_CB8_ENTRIES)) return GLQ_ERR_SHAPE;
    for (int64_t i = 0; i < (int64_t)entries * dim; ++i) {
        if ((host_fp16_bits[i] & 0x7C00u) == 0x7C00u) return GLQ_ERR_INVALID_ARG;  // inf / nan
    }
    glq_codebook cb = new (std::nothrow) glq_codebook_s;
    if (!cb) return GLQ_ERR_OOM;
    cb->entries = entries;
    if (entries == GLQ_CB_ENTRIES) {
        int rc = glq::fold_table(host_fp16_bits, &cb->fold);
        if (rc != 0) {
            delete cb;
            return GLQ_ERR_UNSUPPORTED;
        }
        cb->folded = true;
        cb->table_words = (cb->fold.nb + 3) & ~3;
        cb->fold.words.resize((size_t)cb->table_words, 0u);
    }
    if (cudaGetDevice(&cb->device) != cudaSuccess) {
        cudaGetLastError();
        delete cb;
        return GLQ_ERR_CUDA;
    }
    size_t bytes = (size_t)entries * dim * sizeof(uint16_t);
    glq_status st = dmalloc(&cb->d_fp16, bytes, nullptr);
    if (st == GLQ_OK && cudaMemcpy(cb->d_fp16, host_fp16_bits, bytes, cudaMemcpyHostToDevice) != cudaSuccess)
        st = GLQ_ERR_CUDA;
    if (st == GLQ_OK && cb->folded) {
        // fp16 codewords indexed by folded code (x = v/2 - 3, exact; codes
        // past nb are the negated words), for the tensor-core path's gathers
        const size_t ncodes = (size_t)cb->fold.neg_base + (size_t)cb->fold.nb;
        std::vector<uint16_t> f16(ncodes * 8, 0);
        static const int shift[8] = {0, 8, 16, 24, 4, 12, 20, 28};
        for (size_t e = 0; e < ncodes; ++e) {
            const bool neg = e >= (size_t)cb->fold.nb;
            const uint32_t w = cb->fold.words[neg ? e - (size_t)cb->fold.neg_base : e];
            for (int j = 0; j < 8; ++j) {
                const int y2 = (int)((w >> shift[j]) & 0xF) - 6;  // 2x
                f16[e * 8 + j] = glq::half_bits_of_half_integer(neg ? -y2 : y2);
            }
        }
        st = dmalloc(&cb->d_table_f16, f16.size() * 2, nullptr);
        if (st == GLQ_OK && cudaMemcpy(cb->d_table_f16, f16.data(), f16.size() * 2, cudaMemcpyHostToDevice) !=
                                cudaSuccess)
            st = GLQ_ERR_CUDA;
    }
    if (st == GLQ_OK && cb->folded) {
        st = dmalloc(&cb->d_table, (size_t)cb->table_words * 4, nullptr);
        if (st == GLQ_OK && cudaMemcpy(cb->d_table, cb->fold.words.data(), (size_t)cb->table_words * 4,
                                       cudaMemcpyHostToDevice) != cudaSuccess)
            st = GLQ_ERR_CUDA;
    }
    if (st != GLQ_OK) {
        cudaFree(cb->d_fp16);
        cudaFree(cb->d_table);
        cudaFree(cb->d_table_f16);
        delete cb;
        return st;
    }
    *out = cb;
    return GLQ_OK;
}

glq_status glq_codebook_destroy(glq_codebook cb) {
    if (!cb) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(cb->device);
    cudaFree(cb->d_fp16);
    cudaFree(cb->d_table);
    cudaFree(cb->d_table_f16);
    delete cb;
    return GLQ_OK;
}

// A layer over input columns [k_begin, k_end) of n (the whole layer, or a
// row-parallel shard): the index arrays are the whole layer's.
static glq_status create_layer(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1, const void *const *idx_res,
                        glq_codebook primary, glq_codebook residual, float weight_scale,
                        const float *resid_scales, const int8_t *s_in, const int8_t *s_out, int64_t k_begin,
                        int64_t k_end, glq_layer *out) {
    if (!out) return GLQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (m <= 0 || n <= 0 || m % 8 || n % 8 || m > MAX_DIM || n > MAX_DIM) return GLQ_ERR_SHAPE;
    if (k_begin < 0 || k_end > n || k_begin >= k_end || k_begin % GLQ_CHUNK_K ||
        (k_end % GLQ_CHUNK_K && k_end != n))
        return GLQ_ERR_SHAPE;
    if (bpw < 2 || bpw > 8) return GLQ_ERR_BPW;
    const int n16 = glq::stages16(bpw);
    const bool has8 = glq::stage8(bpw);
    const int nres = n16 + (has8 ? 1 : 0);
    if (!idx1 || !s_in || !s_out) return GLQ_ERR_INVALID_ARG;
    if (nres > 0 && (!idx_res || !resid_scales)) return GLQ_ERR_BPW;
    for (int k = 0; k < nres; ++k)
        if (!idx_res[k]) return GLQ_ERR_BPW;
    if (!primary) return GLQ_ERR_NO_CODEBOOK;
    if (primary->entries != GLQ_CB_ENTRIES || !primary->folded) return GLQ_ERR_NO_CODEBOOK;
    if (has8) {  // the 8-bit stage indexes a 256-entry table
        if (!residual) return GLQ_ERR_NO_CODEBOOK;
        if (residual->entries != GLQ_CB8_ENTRIES) return GLQ_ERR_BPW;
    } else if (residual && residual != primary) {  // 16-bit stages index the E8 table
        return GLQ_ERR_BPW;
    }
    if (!std::isfinite(weight_scale)) return GLQ_ERR_INVALID_ARG;
    for (int k = 0; k < nres; ++k)
        if (!std::isfinite(resid_scales[k])) return GLQ_ERR_INVALID_ARG;
    if (!all_signs(s_in, n) || !all_signs(s_out, m)) return GLQ_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return GLQ_ERR_CUDA;
    }
    if (primary->device != dev || (residual && residual->device != dev)) return GLQ_ERR_NO_CODEBOOK;

    glq_layer L = new (std::nothrow) glq_layer_s;
    if (!L) return GLQ_ERR_OOM;
    L->m = m;
    L->n = n;
    L->bpw = bpw;
    const int G_full = (int)(n / 8), g0 = (int)(k_begin / 8);
    L->G = (int)((k_end - k_begin) / 8);
    L->m_pad = (m + GLQ_ROW_TILE - 1) / GLQ_ROW_TILE * GLQ_ROW_TILE;
    L->n_pad = (n + GLQ_CHUNK_K - 1) / GLQ_CHUNK_K * GLQ_CHUNK_K;
    L->RT = (int)(L->m_pad / GLQ_ROW_TILE);
    L->KC = (int)((k_end - k_begin + GLQ_CHUNK_K - 1) / GLQ_CHUNK_K);
    L->kc0 = (int)(k_begin / GLQ_CHUNK_K);
    L->shard = k_begin != 0 || k_end != n;
    L->device = dev;
    L->primary = primary;
    L->residual = has8 ? residual : (n16 ? primary : nullptr);
    L->ws = weight_scale;
    L->nres16 = n16;
    L->has8 = has8;
    for (int k = 0; k < n16; ++k) L->rs16[k] = resid_scales[k];
    L->rs8 = has8 ? resid_scales[n16] : 0.f;
    // every batch of the tensor-core path reconstructs W first (measured on
    // the 8B-class layers from 17 to 255 tokens: 70-87 us per call against
    // 175-217 us for the dequantising producer); the producer stays available
    // for 2-4 bpw through glq_layer_set_prefill_reconstruct
    L->prefill_mat_min_b = GLQ_DECODE_MAX_B + 1;
    L->plan_n = glq::make_rht_plan((int)n);
    L->plan_m = glq::make_rht_plan((int)m);
    cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (L->num_sms <= 0) L->num_sms = 1;
    L->plan[0] = glq::plan_gemv(L->RT, L->KC, L->num_sms, glq::gemv_warps(1, bpw));
    // two token tiles: a band's split-K partials are twice as many, and
    // with several tasks per CTA they go through the global workspace;
    // charging 2 chunks per split (measured: 24B-class step at 16 tokens
    // 424 -> 266 us, the 32768-row layers then take one split)
    L->plan[1] = glq::plan_gemv(L->RT, L->KC, L->num_sms, glq::gemv_warps(2, bpw), false, 1 << 30, 1 << 30, 2.0);
    const int max_bands = std::max(L->plan[0].bands, L->plan[1].bands);
    L->hb_n = hadamard_blocks_of(n);
    L->hb_m = hadamard_blocks_of(m);

    // fragment-native index streams (layout: glq_internal.h): the primary and
    // every 16-bit stage as folded codes, the 8-bit stage as raw indices
    const FoldedTable &F = primary->fold;
    const size_t slots = (size_t)L->RT * L->KC * 32;
    std::vector<std::vector<uint16_t>> s16(1 + n16, std::vector<uint16_t>(slots * 8, F.zero_code));
    std::vector<uint8_t> s8;
    if (has8) s8.assign(slots * 8, 0);
    for (int64_t r = 0; r < m; ++r) {
        const int64_t rt = r / GLQ_ROW_TILE;
        const int rr = (int)(r % GLQ_ROW_TILE);
        const int g = rr & 7, hi = rr >> 3;
        for (int grp = 0; grp < L->G; ++grp) {
            const int kc = grp / GLQ_GROUPS_PER_CHUNK;
            const int s = (grp % GLQ_GROUPS_PER_CHUNK) / 4;
            const int t = grp % 4;
            const size_t slot = ((size_t)rt * L->KC + kc) * 32 + (size_t)(4 * g + t);
            const size_t src = (size_t)r * G_full + g0 + grp;
            const size_t dst = slot * 8 + 2 * s + hi;
            s16[0][dst] = F.code[idx1[src]];
            for (int k = 0; k < n16; ++k) s16[1 + k][dst] = F.code[static_cast<const uint16_t *>(idx_res[k])[src]];
            if (has8) s8[dst] = static_cast<const uint8_t *>(idx_res[n16])[src];
        }
    }
    std::vector<uint32_t> sin_bits = pack_signs(s_in, n), sout_bits = pack_signs(s_out, m);
    size_t total = 0;
    const size_t bytes16 = slots * 8 * sizeof(uint16_t);
    L->idx_bytes = bytes16 * (1 + n16) + s8.size();
    glq_status st = dmalloc(&L->d_idx1, bytes16, &total);
    for (int k = 0; k < n16 && st == GLQ_OK; ++k) st = dmalloc(&L->d_res16[k], bytes16, &total);
    if (st == GLQ_OK && has8) st = dmalloc(&L->d_res8, s8.size(), &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_sin, sin_bits.size() * 4, &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_sout, sout_bits.size() * 4, &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_err, sizeof(unsigned), &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_cnt, (size_t)max_bands * sizeof(unsigned), &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_blk_cnt, GLQ_MAX_BLOCKS * sizeof(unsigned), &total);
    if (st == GLQ_OK) {
        bool ok = cudaMemcpy(L->d_idx1, s16[0].data(), bytes16, cudaMemcpyHostToDevice) == cudaSuccess;
        for (int k = 0; k < n16 && ok; ++k)
            ok = cudaMemcpy(L->d_res16[k], s16[1 + k].data(), bytes16, cudaMemcpyHostToDevice) == cudaSuccess;
        if (ok && has8) ok = cudaMemcpy(L->d_res8, s8.data(), s8.size(), cudaMemcpyHostToDevice) == cudaSuccess;
        ok = ok && cudaMemcpy(L->d_sin, sin_bits.data(), sin_bits.size() * 4, cudaMemcpyHostToDevice) ==
                       cudaSuccess;
        ok = ok && cudaMemcpy(L->d_sout, sout_bits.data(), sout_bits.size() * 4, cudaMemcpyHostToDevice) ==
                       cudaSuccess;
        ok = ok && cudaMemset(L->d_err, 0, sizeof(unsigned)) == cudaSuccess;
        ok = ok && cudaMemset(L->d_cnt, 0, (size_t)max_bands * sizeof(unsigned)) == cudaSuccess;
        ok = ok && cudaMemset(L->d_blk_cnt, 0, GLQ_MAX_BLOCKS * sizeof(unsigned)) == cudaSuccess;
        if (!ok) st = GLQ_ERR_CUDA;
    }
    if (st != GLQ_OK) {
        cudaGetLastError();
        free_layer(L);
        return st;
    }
    L->device_bytes = total;
    *out = L;
    return GLQ_OK;
}

glq_status glq_layer_create_stages(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1,
                                   const void *const *idx_res, glq_codebook primary, glq_codebook residual,
                                   float weight_scale, const float *resid_scales, const int8_t *s_in,
                                   const int8_t *s_out, glq_layer *out) {
    return create_layer(m, n, bpw, idx1, idx_res, primary, residual, weight_scale, resid_scales, s_in, s_out, 0, n,
                        out);
}

glq_status glq_layer_create_shard(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1,
                                  const void *const *idx_res, glq_codebook primary, glq_codebook residual,
                                  float weight_scale, const float *resid_scales, const int8_t *s_in,
                                  const int8_t *s_out, int64_t k_begin, int64_t k_end, glq_layer *out) {
    return create_layer(m, n, bpw, idx1, idx_res, primary, residual, weight_scale, resid_scales, s_in, s_out,
                        k_begin, k_end, out);
}

glq_status glq_cast(const float *src_dev, void *dst_dev, glq_dtype dtype, int64_t count, void *stream) {
    if (count < 0) return GLQ_ERR_SHAPE;
    if (dtype != GLQ_F16 && dtype != GLQ_BF16 && dtype != GLQ_F32) return GLQ_ERR_DTYPE;
    if (count == 0) return GLQ_OK;
    if (!src_dev || !dst_dev) return GLQ_ERR_INVALID_ARG;
    if (glq::launch_cast(src_dev, dst_dev, (int)dtype, count, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return GLQ_ERR_CUDA;
    }
    return GLQ_OK;
}

glq_status glq_layer_create(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1, const void *idx2,
                            glq_codebook primary, glq_codebook residual, float weight_scale,
                            float resid_scale, const int8_t *s_in, const int8_t *s_out,
                            glq_layer *out) {
    if (!out) return GLQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (bpw < 2 || bpw > 4) return GLQ_ERR_BPW;
    if (bpw == 2 && (idx2 || residual)) return GLQ_ERR_BPW;
    if (bpw > 2 && !idx2) return GLQ_ERR_BPW;
    if (!std::isfinite(resid_scale)) return GLQ_ERR_INVALID_ARG;
    const void *res[1] = {idx2};
    return glq_layer_create_stages(m, n, bpw, idx1, bpw > 2 ? res : nullptr, primary, residual, weight_scale,
                                   bpw > 2 ? &resid_scale : nullptr, s_in, s_out, out);
}

glq_status glq_layer_destroy(glq_layer layer) {
    if (!layer) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(layer->device);
    free_layer(layer);
    return GLQ_OK;
}

glq_status glq_layer_reserve(glq_layer layer, int64_t max_B) {
    if (!layer) return GLQ_ERR_INVALID_ARG;
    if (max_B < 0) return GLQ_ERR_SHAPE;
    DeviceGuard guard(layer->device);
    WsNeed need;
    decode_need(layer, std::max<int64_t>(max_B, 1), need);
    if (layer->invariant) invariant_need(layer, std::max<int64_t>(max_B, 1), need);
    // every tensor-core batch up to max_B (the K-split count, and with it
    // the partial-sum slices, depends on the batch); past 65536 tokens the
    // output has far more tiles than CTA pairs and the largest batch decides
    for (int64_t B = GLQ_DECODE_MAX_B + 1; B <= std::min<int64_t>(max_B, 65536); ++B) prefill_need(layer, B, need);
    if (max_B > 65536) prefill_need(layer, max_B, need);
    void *buf[WS_COUNT];
    return ws_acquire(layer->device, need, 0, buf);
}

glq_status glq_workspace_info(int32_t device, size_t *bytes) {
    if (!bytes || device < 0 || device >= WS_MAX_DEVICES) return GLQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_ws_mu);
    *bytes = ws_bytes_locked(device);
    return GLQ_OK;
}

glq_status glq_workspace_release(int32_t device) {
    if (device < 0 || device >= WS_MAX_DEVICES) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(device);
    std::lock_guard<std::mutex> lock(g_ws_mu);
    if (cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return GLQ_ERR_CUDA;
    }
    DeviceWs &w = g_ws[device];
    for (int i = 0; i < WS_COUNT; ++i) {
        cudaFree(w.buf[i]);
        w.buf[i] = nullptr;
        w.cap[i] = 0;
    }
    return GLQ_OK;
}

glq_status glq_decode_plan(glq_layer layer, int64_t B, int32_t *warps, int32_t *bands, int32_t *splits,
                           int32_t *cluster, int32_t *fused_input) {
    if (!layer) return GLQ_ERR_INVALID_ARG;
    if (B < 1 || B > GLQ_DECODE_MAX_B) return GLQ_ERR_SHAPE;
    DeviceGuard guard(layer->device);
    const void *aligned = reinterpret_cast<const void *>(static_cast<uintptr_t>(256));
    const glq::DecodeCfg c = layer->invariant ? glq::invariant_config(layer, (int)B)
                                              : glq::decode_config(layer, (int)B, aligned, aligned, GLQ_F32);
    if (warps) *warps = c.warps;
    if (bands) *bands = c.plan.bands;
    if (splits) *splits = c.plan.splits;
    if (cluster) *cluster = c.clu;
    if (fused_input) *fused_input = c.fin ? 1 : 0;
    return GLQ_OK;
}

glq_status glq_layer_set_fusion(glq_layer layer, int32_t flags) {
    if (!layer) return GLQ_ERR_INVALID_ARG;
    if (flags != GLQ_FUSE_DEFAULT && (flags & ~(GLQ_FUSE_INPUT | GLQ_FUSE_OUTPUT | GLQ_SPLITK_CLUSTER)))
        return GLQ_ERR_INVALID_ARG;
    layer->fusion = flags;
    return GLQ_OK;
}

glq_status glq_layer_set_batch_invariant(glq_layer layer, int32_t enable) {
    if (!layer || (enable != 0 && enable != 1)) return GLQ_ERR_INVALID_ARG;
    if (layer->shard && enable) return GLQ_ERR_INVALID_ARG;
    layer->invariant = enable != 0;
    return GLQ_OK;
}

glq_status glq_layer_set_prefill_reconstruct(glq_layer layer, int64_t min_batch) {
    if (!layer) return GLQ_ERR_INVALID_ARG;
    if (layer->bpw > 4) return GLQ_OK;  // always reconstructed: the dequantising producer holds two stages
    layer->prefill_mat_min_b = min_batch < 0 ? GLQ_DECODE_MAX_B + 1 : std::max<int64_t>(min_batch, GLQ_DECODE_MAX_B + 1);
    return GLQ_OK;
}

glq_status glq_layer_info(glq_layer layer, int64_t *m, int64_t *n, int32_t *bpw, size_t *device_bytes) {
    if (!layer) return GLQ_ERR_INVALID_ARG;
    if (m) *m = layer->m;
    if (n) *n = layer->n;
    if (bpw) *bpw = layer->bpw;
    if (device_bytes) *device_bytes = layer->device_bytes;
    return GLQ_OK;
}

glq_status glq_linear(glq_layer L, const void *x_dev, glq_dtype x_dtype, void *y_dev, glq_dtype y_dtype,
                      int64_t B, void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B < 0) return GLQ_ERR_SHAPE;
    if (x_dtype != GLQ_F16 && x_dtype != GLQ_BF16) return GLQ_ERR_DTYPE;
    if (y_dtype != x_dtype && y_dtype != GLQ_F32) return GLQ_ERR_DTYPE;
    if (B == 0) return GLQ_OK;
    if (!x_dev || !y_dev) return GLQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x_dev) & 15) || (reinterpret_cast<uintptr_t>(y_dev) & 15))
        return GLQ_ERR_INVALID_ARG;  // the kernels use 8- and 16-byte accesses
    if (L->shard && y_dtype != GLQ_F32) return GLQ_ERR_DTYPE;  // partial sums stay fp32 until summed
    DeviceGuard guard(L->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (L->invariant) {
        WsNeed need;
        invariant_need(L, B, need);
        void *buf[WS_COUNT];
        glq_status st = ws_acquire(L->device, need, s, buf);
        if (st != GLQ_OK) return st;
        void *const v[5] = {buf[WS_XQ], buf[WS_XH], buf[WS_INFO], buf[WS_PART], buf[WS_Z]};
        st = glq::run_invariant(L, x_dev, x_dtype == GLQ_BF16, y_dev, (int)y_dtype, B, s, v, (size_t)L->n_pad * 2);
        if (st != GLQ_OK) cudaGetLastError();
        return st;
    }
    if (B > GLQ_DECODE_MAX_B) return run_prefill(L, x_dev, x_dtype == GLQ_BF16, y_dev, (int)y_dtype, B, s);
    WsNeed need;
    decode_need(L, B, need);
    void *buf[WS_COUNT];
    glq_status st = ws_acquire(L->device, need, s, buf);
    if (st != GLQ_OK) return st;
    const glq_workspace wsp = decode_view(L, buf);
    const size_t xe = 2, ye = y_dtype == GLQ_F32 ? 4 : 2;
    for (int64_t b0 = 0; b0 < B; b0 += GLQ_DECODE_MAX_B) {
        const int nb = (int)std::min<int64_t>(GLQ_DECODE_MAX_B, B - b0);
        const void *x = static_cast<const char *>(x_dev) + (size_t)b0 * L->n * xe;
        void *y = static_cast<char *>(y_dev) + (size_t)b0 * L->m * ye;
        const glq::DecodeCfg cfg = glq::decode_config(L, nb, x, y, (int)y_dtype);
        if (glq::run_decode(L, wsp, cfg, x, x_dtype == GLQ_BF16, y, (int)y_dtype, nb, s) != cudaSuccess) {
            cudaGetLastError();
            return GLQ_ERR_CUDA;
        }
        L->last_B = nb;
        L->last_x = x;
        L->last_y = y;
        L->last_x_bf16 = x_dtype == GLQ_BF16 ? 1 : 0;
        L->last_y_dtype = (int)y_dtype;
    }
    return GLQ_OK;
}

glq_status glq_dequant_reference(glq_layer L, float *w_dev, void *stream) {
    if (!L || !w_dev) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(L->device);
    glq::DequantParams p{};
    p.idx1 = L->d_idx1;
    for (int k = 0; k < 3; ++k) {
        p.idx16[k] = L->d_res16[k];
        p.rs16[k] = L->rs16[k];
    }
    p.idx8 = L->d_res8;
    p.rs8 = L->rs8;
    p.table = L->primary->d_table;
    p.fold = glq::FoldParams{L->primary->fold.nb, L->primary->fold.neg_base};
    p.tab8 = L->has8 ? reinterpret_cast<const uint4 *>(L->residual->d_fp16) : nullptr;
    p.bpw = L->bpw;
    p.m = L->m;
    p.n = L->G * 8;  // a shard's own columns
    p.G = L->G;
    p.KC = L->KC;
    p.ws = L->ws;
    p.w = w_dev;
    return glq::launch_dequant(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GLQ_OK : GLQ_ERR_CUDA;
}

glq_status glq_rht_input(glq_layer L, const void *x_dev, glq_dtype x_dtype, float *xr_dev, int64_t B,
                         void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B < 0) return GLQ_ERR_SHAPE;
    if (x_dtype != GLQ_F16 && x_dtype != GLQ_BF16) return GLQ_ERR_DTYPE;
    if (B == 0) return GLQ_OK;
    if (!x_dev || !xr_dev) return GLQ_ERR_INVALID_ARG;
    if (B > 65535) return GLQ_ERR_SHAPE;
    DeviceGuard guard(L->device);
    glq::RhtInParams p{};
    p.x = x_dev;
    p.x_bf16 = x_dtype == GLQ_BF16;
    p.n = (int)L->n;
    p.n_pad = (int)L->n_pad;
    p.B = (int)B;
    p.sign_bits = L->d_sin;
    p.plan = L->plan_n;
    p.xr_f32 = xr_dev;
    return glq::launch_rht_in(p, static_cast<cudaStream_t>(stream), false) == cudaSuccess ? GLQ_OK
                                                                                         : GLQ_ERR_CUDA;
}

// the row information the transform kernels write: word 2 of each 16-byte
// record is 2^-e (the layout glq_rht_input_operand documents)
static_assert(sizeof(glq_rowinfo) == 16 && offsetof(glq_rowinfo, inv_scale) == 8, "glq_rowinfo layout");

glq_status glq_rht_input_operand(glq_layer L, const void *x_dev, glq_dtype x_dtype, void *xh_dev,
                                 void *row_info_dev, int64_t B, int kernel, void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B < 0 || B > 65535) return GLQ_ERR_SHAPE;
    if (x_dtype != GLQ_F16 && x_dtype != GLQ_BF16) return GLQ_ERR_DTYPE;
    if (kernel < 0 || kernel > 2) return GLQ_ERR_INVALID_ARG;
    if (B == 0) return GLQ_OK;
    if (!x_dev || !xh_dev || !row_info_dev || (reinterpret_cast<uintptr_t>(x_dev) & 15u)) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(L->device);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    glq::RowsParams r = rows_params(L->hb_n, (int)L->n, (int)L->n_pad, L->d_sin);
    r.x = x_dev;
    r.x_bf16 = x_dtype == GLQ_BF16 ? 1 : 0;
    r.xh = static_cast<__half *>(xh_dev);
    r.info = static_cast<glq_rowinfo *>(row_info_dev);
    r.butterfly = kernel == 1 ? 1 : 0;
    if (kernel == 2 && !glq::rht_in_mma_supported(r)) return GLQ_ERR_SHAPE;
    if (glq::rht_rows_supported((int)L->n_pad))
        return glq::launch_rht_rows(r, true, (int)B, s, false) == cudaSuccess ? GLQ_OK : GLQ_ERR_CUDA;
    if (kernel != 0) return GLQ_ERR_SHAPE;
    glq::RhtInParams pin{};
    pin.x = x_dev;
    pin.x_bf16 = r.x_bf16;
    pin.n = (int)L->n;
    pin.n_pad = (int)L->n_pad;
    pin.B = (int)B;
    pin.sign_bits = L->d_sin;
    pin.plan = L->plan_n;
    pin.xh = r.xh;
    pin.info = r.info;
    pin.xh_only = 1;
    return glq::launch_rht_in(pin, s, false) == cudaSuccess ? GLQ_OK : GLQ_ERR_CUDA;
}

glq_status glq_rht_output(glq_layer L, const float *z_dev, void *y_dev, glq_dtype y_dtype, int64_t B,
                          void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B < 0) return GLQ_ERR_SHAPE;
    if (y_dtype != GLQ_F16 && y_dtype != GLQ_BF16 && y_dtype != GLQ_F32) return GLQ_ERR_DTYPE;
    if (B == 0) return GLQ_OK;
    if (!z_dev || !y_dev) return GLQ_ERR_INVALID_ARG;
    if (B > 65535) return GLQ_ERR_SHAPE;
    DeviceGuard guard(L->device);
    // the kernel glq_linear's output stage takes for this batch: one CTA per
    // row, except for one or two rows longer than 8192
    if (glq::rht_rows_supported((int)L->m) && (B > 2 || L->m <= 8192)) {
        glq::RowsParams r = rows_params(L->hb_m, (int)L->m, (int)L->m, L->d_sout);
        r.z = z_dev;
        r.z_ld = (int)L->m;
        r.y = y_dev;
        r.y_dtype = (int)y_dtype;
        return glq::launch_rht_rows(r, false, (int)B, static_cast<cudaStream_t>(stream), false) == cudaSuccess
                   ? GLQ_OK
                   : GLQ_ERR_CUDA;
    }
    glq::RhtOutParams p{};
    p.m = (int)L->m;
    p.B = (int)B;
    p.z = z_dev;
    p.z_ld = (int)L->m;
    p.sign_bits = L->d_sout;
    p.plan = L->plan_m;
    p.y = y_dev;
    p.y_dtype = (int)y_dtype;
    return glq::launch_rht_out(p, static_cast<cudaStream_t>(stream), false) == cudaSuccess ? GLQ_OK
                                                                                          : GLQ_ERR_CUDA;
}

glq_status glq_gemv_replay(glq_layer L, int64_t B, void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B < 1 || B > L->last_B) return GLQ_ERR_SHAPE;
    DeviceGuard guard(L->device);
    const glq::DecodeCfg cfg = glq::decode_config(L, (int)B, L->last_x, L->last_y, L->last_y_dtype);
    WsNeed need;  // buffers large enough for this layer (their contents are the last call's)
    decode_need(L, B, need);
    void *buf[WS_COUNT];
    glq_status st = ws_acquire(L->device, need, static_cast<cudaStream_t>(stream), buf);
    if (st != GLQ_OK) return st;
    glq::GemvParams pg = glq::gemv_params(L, decode_view(L, buf), cfg, (int)B, L->last_x, L->last_x_bf16 != 0,
                                          L->last_y, L->last_y_dtype);
    return glq::launch_gemv(pg, L->bpw, cfg.plan.grid, static_cast<cudaStream_t>(stream), true, cfg.fin) ==
                   cudaSuccess
               ? GLQ_OK
               : GLQ_ERR_CUDA;
}

glq_status glq_prefill_replay(glq_layer L, int64_t B, void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B <= GLQ_DECODE_MAX_B || B > L->last_prefill_B) return GLQ_ERR_SHAPE;
    DeviceGuard guard(L->device);
    WsNeed need;  // buffers large enough for this layer (their contents are the last call's)
    prefill_need(L, B, need);
    if (L->last_prefill_mat)
        need.b[WS_W16] = std::max(need.b[WS_W16], (size_t)L->m_pad * stream_cols(L) * sizeof(__half));
    void *buf[WS_COUNT];
    glq_status st = ws_acquire(L->device, need, static_cast<cudaStream_t>(stream), buf);
    if (st != GLQ_OK) return st;
    return launch_prefill_gemm(L, prefill_view(buf), B, L->last_prefill_mat, static_cast<cudaStream_t>(stream),
                               false) == cudaSuccess
               ? GLQ_OK
               : GLQ_ERR_CUDA;
}

glq_status glq_layer_selftest_wait(glq_layer L, int kind, int arrivals, int64_t limit, void *stream) {
    if (!L || kind < 0 || kind > 2 || arrivals < 1 || arrivals > 2 || limit <= 0) return GLQ_ERR_INVALID_ARG;
    if (kind == 2 && limit > (int64_t)0xFFFFFFFFll) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(L->device);
    return glq::launch_wait_selftest(L->d_err, kind, arrivals, (unsigned long long)limit,
                                     static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? GLQ_OK
               : GLQ_ERR_CUDA;
}

glq_status glq_layer_check(glq_layer L, void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(L->device);
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return GLQ_ERR_CUDA;
    }
    unsigned err = 0;
    if (cudaMemcpy(&err, L->d_err, sizeof err, cudaMemcpyDeviceToHost) != cudaSuccess) return GLQ_ERR_CUDA;
    if (err) {
        cudaMemset(L->d_err, 0, sizeof(unsigned));
        return (err & GLQ_DEVERR_TIMEOUT) ? GLQ_ERR_TIMEOUT : GLQ_ERR_DEVICE_CHECK;
    }
    return GLQ_OK;
}

}  // extern "C"
