// glq_api.cu -- the C ABI of glq-b200 (include/glq.h): argument checks,
// the host-side re-layout of index arrays into the kernels' fragment-native
// streams, device memory ownership and kernel dispatch.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
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

glq_blocks make_blocks(int64_t n) {
    glq_blocks b{};
    int off = 0;
    for (int bit = 30; bit >= 0; --bit) {
        if (n & (int64_t(1) << bit)) {
            int k = 1 << bit;
            b.size[b.count] = k;
            b.offset[b.count] = off;
            b.inv_sqrt[b.count] = (float)(1.0 / std::sqrt((double)k));
            off += k;
            ++b.count;
        }
    }
    return b;
}

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
    cudaFree(L->d_idx1);
    cudaFree(L->d_idx2);
    cudaFree(L->d_sin);
    cudaFree(L->d_sout);
    cudaFree(L->d_err);
    cudaFree(L->d_r8);
    cudaFree(L->d_xr);
    cudaFree(L->d_info);
    cudaFree(L->d_part);
    delete L;
}

// Chooses the split of the chunk range so that (bands x splits) tasks spread
// over the persistent grid with the least makespan (in chunks per CTA).
void plan_gemv(glq_layer L) {
    L->bands = (L->RT + glq::GEMV_WARPS - 1) / glq::GEMV_WARPS;
    int best_s = 1;
    double best = 1e30;
    for (int s = 1; s <= L->KC; ++s) {
        int cps = (L->KC + s - 1) / s;
        int used = (L->KC + cps - 1) / cps;  // splits actually populated
        if (used != s) continue;
        int64_t tasks = (int64_t)L->bands * s;
        int64_t waves = (tasks + L->num_sms - 1) / L->num_sms;
        double cost = (double)waves * cps + 0.02 * s;
        if (cost < best) {
            best = cost;
            best_s = s;
        }
    }
    L->splits = best_s;
    L->cps = (L->KC + best_s - 1) / best_s;
    int64_t tasks = (int64_t)L->bands * L->splits;
    L->grid = (int)std::min<int64_t>(tasks, L->num_sms);
}

glq_status grow_workspace(glq_layer L, int64_t rows) {
    if (rows <= L->cap_rows) return GLQ_OK;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return GLQ_ERR_CUDA;
    cudaFree(L->d_xr);
    cudaFree(L->d_info);
    cudaFree(L->d_part);
    L->d_xr = nullptr;
    L->d_info = nullptr;
    L->d_part = nullptr;
    L->cap_rows = 0;
    size_t dummy = 0;
    int64_t dec_rows = std::min<int64_t>(rows, GLQ_DECODE_MAX_B);
    glq_status st = dmalloc(&L->d_xr, (size_t)rows * L->n_pad * sizeof(__half), &dummy);
    if (st == GLQ_OK) st = dmalloc(&L->d_info, (size_t)rows * sizeof(glq_rowinfo), &dummy);
    if (st == GLQ_OK)
        st = dmalloc(&L->d_part, (size_t)L->splits * dec_rows * L->m_pad * sizeof(float), &dummy);
    if (st != GLQ_OK) return st;
    L->cap_rows = rows;
    return GLQ_OK;
}

glq::GemvParams gemv_params(glq_layer L, const __half *xr, const glq_rowinfo *, int B) {
    glq::GemvParams p{};
    p.idx1 = L->d_idx1;
    p.idx2 = L->d_idx2;
    p.table = L->primary->d_table;
    p.table_words = L->primary->table_words;
    p.fold = glq::FoldParams{L->primary->fold.nb, L->primary->fold.neg_base};
    p.res8 = (L->bpw == 3) ? reinterpret_cast<const uint4 *>(L->d_r8) : nullptr;
    p.xr = xr;
    p.B = B;
    p.n_pad = (int)L->n_pad;
    p.KC = L->KC;
    p.RT = L->RT;
    p.bands = L->bands;
    p.splits = L->splits;
    p.cps = L->cps;
    p.rs_acc = L->bpw == 3 ? L->rs / GLQ_ACC_SCALE : L->rs;
    p.partials = L->d_part;
    p.m_pad = (int)L->m_pad;
    p.err = L->d_err;
    return p;
}

}  // namespace

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
    if (entries == GLQ_CB8_ENTRIES) {
        cb->host.assign(host_fp16_bits, host_fp16_bits + (size_t)entries * dim);
        // the decode kernels hold columns 2,3,6,7 scaled by 16 in fp16
        for (int e = 0; e < entries; ++e)
            for (int j : {2, 3, 6, 7})
                if (std::fabs(glq::half_bits_to_float(host_fp16_bits[e * dim + j])) >= 4094.0f) {
                    delete cb;
                    return GLQ_ERR_UNSUPPORTED;
                }
    }
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
        st = dmalloc(&cb->d_table, (size_t)cb->table_words * 4, nullptr);
        if (st == GLQ_OK && cudaMemcpy(cb->d_table, cb->fold.words.data(), (size_t)cb->table_words * 4,
                                       cudaMemcpyHostToDevice) != cudaSuccess)
            st = GLQ_ERR_CUDA;
    }
    if (st != GLQ_OK) {
        cudaFree(cb->d_fp16);
        cudaFree(cb->d_table);
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
    delete cb;
    return GLQ_OK;
}

glq_status glq_layer_create(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1, const void *idx2,
                            glq_codebook primary, glq_codebook residual, float weight_scale,
                            float resid_scale, const int8_t *s_in, const int8_t *s_out,
                            glq_layer *out) {
    if (!out) return GLQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (m <= 0 || n <= 0 || m % 8 || n % 8 || m > MAX_DIM || n > MAX_DIM) return GLQ_ERR_SHAPE;
    if (bpw < 2 || bpw > 4) return GLQ_ERR_BPW;
    if (!idx1 || !s_in || !s_out) return GLQ_ERR_INVALID_ARG;
    if (!primary) return GLQ_ERR_NO_CODEBOOK;
    if (primary->entries != GLQ_CB_ENTRIES || !primary->folded) return GLQ_ERR_NO_CODEBOOK;
    if (bpw == 2 && (idx2 || residual)) return GLQ_ERR_BPW;
    if (bpw == 3) {
        if (!idx2) return GLQ_ERR_BPW;
        if (!residual) return GLQ_ERR_NO_CODEBOOK;
        if (residual->entries != GLQ_CB8_ENTRIES) return GLQ_ERR_BPW;
    }
    if (bpw == 4) {
        if (!idx2) return GLQ_ERR_BPW;
        if (residual && residual != primary) return GLQ_ERR_BPW;
    }
    if (!std::isfinite(weight_scale) || !std::isfinite(resid_scale)) return GLQ_ERR_INVALID_ARG;
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
    L->G = (int)(n / 8);
    L->m_pad = (m + GLQ_ROW_TILE - 1) / GLQ_ROW_TILE * GLQ_ROW_TILE;
    L->n_pad = (n + GLQ_CHUNK_K - 1) / GLQ_CHUNK_K * GLQ_CHUNK_K;
    L->RT = (int)(L->m_pad / GLQ_ROW_TILE);
    L->KC = (int)(L->n_pad / GLQ_CHUNK_K);
    L->device = dev;
    L->primary = primary;
    L->residual = bpw == 4 ? primary : residual;
    L->ws = weight_scale;
    L->rs = bpw == 2 ? 0.f : resid_scale;
    L->bn = make_blocks(n);
    L->bm = make_blocks(m);
    cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (L->num_sms <= 0) L->num_sms = 1;
    plan_gemv(L);

    // fragment-native index streams (layout: glq_internal.h)
    const FoldedTable &F = primary->fold;
    const size_t slots = (size_t)L->RT * L->KC * 32;
    std::vector<uint16_t> s1(slots * 8, F.zero_code);
    std::vector<uint16_t> s2u16;
    std::vector<uint8_t> s2u8;
    if (bpw == 4) s2u16.assign(slots * 8, F.zero_code);
    if (bpw == 3) s2u8.assign(slots * 8, 0);
    const uint16_t *i2u16 = static_cast<const uint16_t *>(idx2);
    const uint8_t *i2u8 = static_cast<const uint8_t *>(idx2);
    for (int64_t r = 0; r < m; ++r) {
        const int64_t rt = r / GLQ_ROW_TILE;
        const int rr = (int)(r % GLQ_ROW_TILE);
        const int g = rr & 7, hi = rr >> 3;
        for (int grp = 0; grp < L->G; ++grp) {
            const int kc = grp / GLQ_GROUPS_PER_CHUNK;
            const int s = (grp % GLQ_GROUPS_PER_CHUNK) / 4;
            const int t = grp % 4;
            const size_t slot = ((size_t)rt * L->KC + kc) * 32 + (size_t)(4 * g + t);
            const size_t src = (size_t)r * L->G + grp;
            s1[slot * 8 + 2 * s + hi] = F.code[idx1[src]];
            if (bpw == 4) s2u16[slot * 8 + 2 * s + hi] = F.code[i2u16[src]];
            if (bpw == 3) s2u8[slot * 8 + 2 * s + hi] = i2u8[src];
        }
    }
    std::vector<uint32_t> sin_bits = pack_signs(s_in, n), sout_bits = pack_signs(s_out, m);
    std::vector<uint16_t> r8;
    if (bpw == 3) {
        r8 = residual->host;
        for (int e = 0; e < GLQ_CB8_ENTRIES; ++e)
            for (int j : {2, 3, 6, 7}) r8[e * 8 + j] = glq::half_bits_times16(r8[e * 8 + j]);
    }

    size_t total = 0;
    L->idx1_bytes = s1.size() * sizeof(uint16_t);
    L->idx2_bytes = bpw == 4 ? s2u16.size() * 2 : (bpw == 3 ? s2u8.size() : 0);
    glq_status st = dmalloc(&L->d_idx1, L->idx1_bytes, &total);
    if (st == GLQ_OK && bpw > 2) st = dmalloc((char **)&L->d_idx2, L->idx2_bytes, &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_sin, sin_bits.size() * 4, &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_sout, sout_bits.size() * 4, &total);
    if (st == GLQ_OK) st = dmalloc(&L->d_err, sizeof(unsigned), &total);
    if (st == GLQ_OK && bpw == 3) st = dmalloc(&L->d_r8, r8.size() * 2, &total);
    if (st == GLQ_OK) {
        bool ok = cudaMemcpy(L->d_idx1, s1.data(), L->idx1_bytes, cudaMemcpyHostToDevice) == cudaSuccess;
        if (ok && bpw == 4)
            ok = cudaMemcpy(L->d_idx2, s2u16.data(), L->idx2_bytes, cudaMemcpyHostToDevice) == cudaSuccess;
        if (ok && bpw == 3)
            ok = cudaMemcpy(L->d_idx2, s2u8.data(), L->idx2_bytes, cudaMemcpyHostToDevice) == cudaSuccess;
        ok = ok && cudaMemcpy(L->d_sin, sin_bits.data(), sin_bits.size() * 4, cudaMemcpyHostToDevice) ==
                       cudaSuccess;
        ok = ok && cudaMemcpy(L->d_sout, sout_bits.data(), sout_bits.size() * 4, cudaMemcpyHostToDevice) ==
                       cudaSuccess;
        ok = ok && cudaMemset(L->d_err, 0, sizeof(unsigned)) == cudaSuccess;
        if (ok && bpw == 3)
            ok = cudaMemcpy(L->d_r8, r8.data(), r8.size() * 2, cudaMemcpyHostToDevice) == cudaSuccess;
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
    return grow_workspace(layer, std::min<int64_t>(std::max<int64_t>(max_B, 1), GLQ_DECODE_MAX_B));
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
    DeviceGuard guard(L->device);
    glq_status st = grow_workspace(L, std::min<int64_t>(B, GLQ_DECODE_MAX_B));
    if (st != GLQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t xe = 2, ye = y_dtype == GLQ_F32 ? 4 : 2;
    for (int64_t b0 = 0; b0 < B; b0 += GLQ_DECODE_MAX_B) {
        const int nb = (int)std::min<int64_t>(GLQ_DECODE_MAX_B, B - b0);
        glq::RhtInParams pin{};
        pin.x = static_cast<const char *>(x_dev) + (size_t)b0 * L->n * xe;
        pin.x_bf16 = x_dtype == GLQ_BF16;
        pin.n = (int)L->n;
        pin.n_pad = (int)L->n_pad;
        pin.B = nb;
        pin.sign_bits = L->d_sin;
        pin.blocks = L->bn;
        pin.xr_h = L->d_xr;
        pin.info = L->d_info;
        if (glq::launch_rht_in(pin, s, true) != cudaSuccess) return GLQ_ERR_CUDA;

        glq::GemvParams pg = gemv_params(L, L->d_xr, L->d_info, nb);
        if (glq::launch_gemv(pg, L->bpw, L->grid, s, true) != cudaSuccess) return GLQ_ERR_CUDA;
        L->last_B = nb;

        glq::RhtOutParams pout{};
        pout.m = (int)L->m;
        pout.m_pad = (int)L->m_pad;
        pout.B = nb;
        pout.partials = L->d_part;
        pout.splits = L->splits;
        pout.info = L->d_info;
        pout.ws = L->ws;
        pout.corr_mult = L->bpw == 4 ? 1.f + L->rs : 1.f;
        pout.sign_bits = L->d_sout;
        pout.blocks = L->bm;
        pout.y = static_cast<char *>(y_dev) + (size_t)b0 * L->m * ye;
        pout.y_dtype = (int)y_dtype;
        if (glq::launch_rht_out(pout, s, true) != cudaSuccess) return GLQ_ERR_CUDA;
    }
    return GLQ_OK;
}

glq_status glq_dequant_reference(glq_layer L, float *w_dev, void *stream) {
    if (!L || !w_dev) return GLQ_ERR_INVALID_ARG;
    DeviceGuard guard(L->device);
    glq::DequantParams p{};
    p.idx1 = L->d_idx1;
    p.idx2 = L->d_idx2;
    p.table = L->primary->d_table;
    p.fold = glq::FoldParams{L->primary->fold.nb, L->primary->fold.neg_base};
    p.res8 = (L->bpw == 3) ? reinterpret_cast<const uint4 *>(L->residual->d_fp16) : nullptr;
    p.bpw = L->bpw;
    p.m = L->m;
    p.n = (int)L->n;
    p.G = L->G;
    p.KC = L->KC;
    p.ws = L->ws;
    p.rs = L->rs;
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
    p.blocks = L->bn;
    p.xr_f32 = xr_dev;
    return glq::launch_rht_in(p, static_cast<cudaStream_t>(stream), false) == cudaSuccess ? GLQ_OK
                                                                                         : GLQ_ERR_CUDA;
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
    glq::RhtOutParams p{};
    p.m = (int)L->m;
    p.m_pad = (int)L->m_pad;
    p.B = (int)B;
    p.z = z_dev;
    p.z_ld = (int)L->m;
    p.sign_bits = L->d_sout;
    p.blocks = L->bm;
    p.y = y_dev;
    p.y_dtype = (int)y_dtype;
    return glq::launch_rht_out(p, static_cast<cudaStream_t>(stream), false) == cudaSuccess ? GLQ_OK
                                                                                          : GLQ_ERR_CUDA;
}

glq_status glq_gemv_replay(glq_layer L, int64_t B, void *stream) {
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B < 1 || B > L->last_B) return GLQ_ERR_SHAPE;
    DeviceGuard guard(L->device);
    glq::GemvParams pg = gemv_params(L, L->d_xr, L->d_info, (int)B);
    return glq::launch_gemv(pg, L->bpw, L->grid, static_cast<cudaStream_t>(stream), false) == cudaSuccess
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
