// glq_rht_rows.cu -- the input and output randomized Hadamard transforms of
// the tensor-core (many-token) path: xr = H_n (S_in x) and y = S_out (H_m z),
// H block-diagonal over the binary decomposition of the size, each block a
// Sylvester-ordered FWHT normalised by 1/sqrt(block) (glq 0.5.1 PyPI page,
// "How it works" 2 and "Bit widths": block-diagonal FHT for sizes that are
// not powers of two; GLQ v0.3.2 release notes, input_rht / output_rht).
//
// Design (B200): throughput over many rows, sizes up to 16384, bound by the
// per-value instruction count rather than by DRAM.  A persistent grid of CTAs
// transforms one row at a time per CTA, with the next row already streaming
// into a shared-memory staging buffer (16-byte asynchronous copies):
//   * a row of up to 2^L values (9 <= L <= 14) is held 16 values per thread;
//     the butterflies run in registers, four position bits per phase, and the
//     row changes layout between phases through shared memory (one store,
//     one barrier, one load per value and phase) under an XOR swizzle that
//     keeps every access free of bank conflicts; no warp shuffles;
//   * butterflies on register pairs use the packed f32x2 add / subtract of
//     sm_100a (same IEEE rounding as scalar adds);
//   * Hadamard blocks of a size that is not a power of two are handled by
//     testing, per butterfly, whether both ends lie in one block;
//   * the input direction also finds the row's max |xr| (one reduction) and
//     writes either the fp16 operand of the tensor-core GEMM, xr 2^e with
//     max |xr| 2^e < 2^14, or the decode GEMV's operand X = round(xr 2^e) as
//     high / low bytes with its exact row sum (a second reduction), plus 2^-e.
#include <algorithm>

#include "glq_kernels.cuh"

namespace glq {

namespace {

constexpr int VPT = 16;  // values per thread

// block (offset, size) of the Hadamard decomposition containing column c
__device__ __forceinline__ int block_size_at(const RowsParams &p, int c, float *norm) {
    for (int i = 0; i < p.nblk; ++i)
        if (c >= p.blk_off[i] && c < p.blk_off[i] + p.blk_len[i]) {
            *norm = p.blk_norm[i];
            return p.blk_len[i];
        }
    *norm = 0.f;
    return 0;
}

// ---------------------------------------------------------------------------
// Layout of a row of 2^L words (9 <= L <= 14) in the butterfly phases.
//
// Phase q owns the position bits 4q .. 4q+3 (those below L).  In it a thread
// holds 16 values whose positions differ exactly in four "register" bits:
// the phase's own bits, filled up with the lowest other bits when fewer than
// four remain; the bits of the thread index give the other position bits in
// increasing order.  Phase 0 is the layout of the global loads and stores
// (16 consecutive values per thread); the later phases read and write the
// row through shared memory.
// ---------------------------------------------------------------------------

// Word of position p in shared memory: p with its bank bits (0..4) XORed by a
// linear function of bits 5..13.  The table was found by exhaustive check:
// with it, every access of the phases below (a warp's 32 lanes at one
// register index) meets 32 distinct banks for every L from 9 to 14.
__host__ __device__ constexpr uint32_t swz(uint32_t p) {
    constexpr uint32_t M[9] = {9u, 26u, 22u, 24u, 20u, 7u, 21u, 0u, 20u};
    uint32_t t = 0u;
    for (int k = 0; k < 9; ++k)
        if ((p >> (5 + k)) & 1u) t ^= M[k];
    return p ^ t;
}

// position bit of register bit r (0..3) in phase q
__host__ __device__ constexpr int reg_bit(int L, int q, int r) {
    const int na = (L - 4 * q) < 4 ? (L - 4 * q) : 4;
    if (r < na) return 4 * q + r;
    int k = r - na;
    for (int b = 0; b < L; ++b) {
        if (b >= 4 * q && b < 4 * q + na) continue;
        if (k == 0) return b;
        --k;
    }
    return 0;
}

// position bits of register index j (0..15) in phase q
__host__ __device__ constexpr uint32_t jpos(int L, int q, int j) {
    uint32_t p = 0u;
    for (int r = 0; r < 4; ++r)
        if ((j >> r) & 1) p |= 1u << reg_bit(L, q, r);
    return p;
}

// position bits given by thread index t (< 2^(L-4)) in phase q: around the
// four register bits 4q..4q+3, or, in a last phase with fill bits, above
// the fill bits
template <int L>
__device__ __forceinline__ uint32_t tpos(int q, uint32_t t) {
    const int na = (L - 4 * q) < 4 ? (L - 4 * q) : 4;
    if (na == 4) return (t & ((1u << (4 * q)) - 1u)) | ((t >> (4 * q)) << (4 * q + 4));
    return t << (4 - na);
}

// a value the compiler must treat as new on every use, so that loop-invariant
// shared-memory addresses are recomputed (one XOR) rather than kept live
__device__ __forceinline__ uint32_t opaque(uint32_t x) {
    uint32_t y;
    asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Two butterflies on value pairs: (a0, a1) <- (a0, a1) + (b0, b1) and
// (b0, b1) <- old (a0, a1) - (b0, b1), as packed f32x2 operations.
__device__ __forceinline__ void bfly2(float &a0, float &a1, float &b0, float &b1) {
    asm("{\n"
        " .reg .b64 A, B, S, D;\n"
        " mov.b64 A, {%0, %1};\n"
        " mov.b64 B, {%2, %3};\n"
        " add.rn.f32x2 S, A, B;\n"
        " sub.rn.f32x2 D, A, B;\n"
        " mov.b64 {%0, %1}, S;\n"
        " mov.b64 {%2, %3}, D;\n"
        "}\n"
        : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// The butterflies of phase Q on a thread's 16 values (register bit r of the
// index j pairs j with j | 2^r; bit 0 pairs neighbours, the other bits whole
// register pairs).  The butterfly of span 2^b between positions p and
// p + 2^b (bit b of p clear) belongs to the block transform iff both lie in
// one Hadamard block, i.e. iff the block holding p is larger than 2^b.
// Blocks are aligned powers of two in descending order, so the block of
// p < len has size 2^msb(p ^ len) and the test is (p ^ len) >> (b + 1) != 0;
// positions past the row hold zeros either way.  X = (the thread's position
// bits) ^ len; full: every test of the phase holds.
template <int L, int Q>
__device__ __forceinline__ void phase_stages(float v[VPT], uint32_t X, unsigned full) {
    constexpr int na = (L - 4 * Q) < 4 ? (L - 4 * Q) : 4;
    if (full) {
#pragma unroll
        for (int j = 0; j < VPT; j += 2) {
            const float a = v[j], c = v[j + 1];
            v[j] = a + c;
            v[j + 1] = a - c;
        }
#pragma unroll
        for (int r = 1; r < na; ++r)
#pragma unroll
            for (int j = 0; j < VPT; j += 2)
                if (((j >> r) & 1) == 0) {
                    const int k = j | (1 << r);
                    bfly2(v[j], v[j + 1], v[k], v[k + 1]);
                }
    } else {
#pragma unroll
        for (int r = 0; r < na; ++r)
#pragma unroll
            for (int j = 0; j < VPT; ++j)
                if (((j >> r) & 1) == 0) {
                    const int k = j | (1 << r);
                    // only the position bits above the span matter
                    if ((X >> (4 * Q + r + 1)) != (jpos(L, Q, j) >> (4 * Q + r + 1))) {
                        const float a = v[j], c = v[k];
                        v[j] = a + c;
                        v[k] = a - c;
                    }
                }
    }
}

// Phase Q >= 1: load the thread's 16 values of the phase from shared memory,
// apply its butterflies, store them back, then a CTA barrier.  Every thread
// reads and writes only its own 16 positions within a phase.
template <int L, int Q>
__device__ __forceinline__ void phase_pass(float v[VPT], float *srow, uint32_t base, uint32_t len, unsigned full) {
    const uint32_t b0 = opaque(base);
#pragma unroll
    for (int j = 0; j < VPT; ++j) v[j] = srow[b0 ^ swz(jpos(L, Q, j))];
    phase_stages<L, Q>(v, tpos<L>(Q, opaque(threadIdx.x)) ^ len, full);
    const uint32_t b1 = opaque(base);
#pragma unroll
    for (int j = 0; j < VPT; ++j) srow[b1 ^ swz(jpos(L, Q, j))] = v[j];
    __syncthreads();
}

// 16-byte asynchronous copy from global to shared memory; with src_bytes = 0
// nothing is read and the 16 bytes are zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// sign of value j (bit j of sb) applied to v
__device__ __forceinline__ float flip(float v, uint32_t sb, int j) {
    return __int_as_float(__float_as_int(v) ^ ((sb << (31 - j)) & 0x80000000u));
}

// Persistent over rows: a CTA transforms rows blockIdx.x, blockIdx.x +
// gridDim.x, ...  Each thread stages its raw input of the next row (16 fp16 /
// bf16 activations, or 16 fp32 partial sums of the first K split) with
// asynchronous copies into its own slots of a staging buffer while the
// current row is transformed.
template <bool IN, bool XQ, int L>
__global__ void __launch_bounds__(1 << (L - 4)) rht_rows_kernel(RowsParams p, int B) {
    constexpr int NPH = (L + 3) / 4;  // phases of (up to) four position bits
    constexpr int NCH = IN ? 2 : 4;   // 16-byte chunks of raw input per thread
    extern __shared__ __align__(16) float smem_rows[];
    float *srow = smem_rows;  // the row, 2^L words, swizzled
    const uint4 *stage = reinterpret_cast<const uint4 *>(smem_rows + (1 << L));
    __shared__ float s_red[2][32];  // per-warp row max, by row parity
    __shared__ int s_sum[2][32];    // per-warp sums of X, by row parity
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c0 = VPT * tid;  // first column of this thread
    const uint32_t len = (uint32_t)p.len;
    const int valid = max(0, min(VPT, p.len - c0));  // 16, 8 (last block of 8) or 0
    pdl_launch_dependents();
    int b = blockIdx.x;
    if (b < B && c0 < p.len) {  // warm L2 and the TLB before waiting on the producer
        if (IN) prefetch_l2(static_cast<const uint16_t *>(p.x) + (size_t)b * p.len + c0);
        else prefetch_l2(p.z + (size_t)b * p.z_ld + c0);  // the first split
    }

    // row-independent data of this thread
    float norm = 0.f;
    if (c0 < p.len) block_size_at(p, c0, &norm);
    const uint32_t sb = valid ? (p.sign_bits[c0 >> 5] >> (c0 & 31)) & 0xFFFFu : 0u;
    uint32_t base[NPH];
    unsigned full = 0u;
#pragma unroll
    for (int q = 0; q < NPH; ++q) {
        const uint32_t tp = tpos<L>(q, (uint32_t)tid);
        base[q] = swz(tp);
        const int top = (4 * q + 4 < L ? 4 * q + 4 : L);  // one past the phase's highest bit
        if (((tp ^ len) >> top) != 0u) full |= 1u << q;
    }
    // staging slots, swizzled so that the 16-byte reads of 8 consecutive
    // threads meet 8 distinct bank groups
    const uint32_t stage_sh = (uint32_t)__cvta_generic_to_shared(stage);
    auto slot = [&](int c) -> int {
        return IN ? 2 * tid + (c ^ ((tid >> 2) & 1)) : 4 * tid + (c ^ ((tid >> 1) & 3));
    };
    auto issue = [&](int row) {
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const bool ok = IN ? (8 * c < valid) : (4 * c < valid);
            const void *src;
            if (IN) src = static_cast<const uint16_t *>(p.x) + (size_t)row * p.len + (ok ? c0 + 8 * c : 0);
            else src = p.z + (size_t)row * p.z_ld + (ok ? c0 + 4 * c : 0);
            cp_async16(stage_sh + 16u * (uint32_t)slot(c), src, ok ? 16u : 0u);
        }
        cp_async_commit();
    };

    pdl_wait();  // the input comes from the previous kernel
    if (b < B) issue(b);
    for (int par = 0; b < B; b += gridDim.x, par ^= 1) {
        cp_async_wait_all();
        uint4 raw[NCH];
#pragma unroll
        for (int c = 0; c < NCH; ++c) raw[c] = stage[slot(c)];
        if (b + (int)gridDim.x < B) issue(b + gridDim.x);  // this thread's slots are free again
        float v[VPT];
        if (IN) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (p.x_bf16) {
                        v[8 * q + 2 * j] = __uint_as_float(w[j] << 16);
                        v[8 * q + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
                    } else {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[j]));
                        v[8 * q + 2 * j] = f.x;
                        v[8 * q + 2 * j + 1] = f.y;
                    }
                }
            }
            const uint32_t sbr = opaque(sb);  // sign masks rebuilt per row, not kept live
#pragma unroll
            for (int j = 0; j < VPT; ++j) v[j] = flip(v[j], sbr, j);
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[4 * q] = __uint_as_float(raw[q].x);
                v[4 * q + 1] = __uint_as_float(raw[q].y);
                v[4 * q + 2] = __uint_as_float(raw[q].z);
                v[4 * q + 3] = __uint_as_float(raw[q].w);
            }
            for (int sp = 1; sp < p.zsplits; ++sp) {  // further K-split partial sums, in split order
                const float4 *src = reinterpret_cast<const float4 *>(p.z + sp * p.zs + (size_t)b * p.z_ld + c0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (4 * q < valid) r = __ldcs(src + q);
                    v[4 * q] += r.x;
                    v[4 * q + 1] += r.y;
                    v[4 * q + 2] += r.z;
                    v[4 * q + 3] += r.w;
                }
            }
        }

        // the butterflies, phase by phase (phase 0 on the values as loaded)
        phase_stages<L, 0>(v, opaque((uint32_t)c0) ^ len, full & 1u);
        if (NPH > 1) {
            const uint32_t b0 = opaque(base[0]);
#pragma unroll
            for (int j = 0; j < VPT; ++j) srow[b0 ^ swz(jpos(L, 0, j))] = v[j];
            __syncthreads();
            if (NPH > 1) phase_pass<L, (NPH > 1 ? 1 : 0)>(v, srow, base[NPH > 1 ? 1 : 0], len, (full >> 1) & 1u);
            if (NPH > 2) phase_pass<L, (NPH > 2 ? 2 : 0)>(v, srow, base[NPH > 2 ? 2 : 0], len, (full >> 2) & 1u);
            if (NPH > 3) phase_pass<L, (NPH > 3 ? 3 : 0)>(v, srow, base[NPH > 3 ? 3 : 0], len, (full >> 3) & 1u);
            const uint32_t b1 = opaque(base[0]);
#pragma unroll
            for (int j = 0; j < VPT; ++j) v[j] = srow[b1 ^ swz(jpos(L, 0, j))];
        }

        if (IN) {
            // row max of |xr| = |v| norm (norm is one per thread: all 16 values share a block)
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) mx = fmaxf(mx, fabsf(v[j]));
            mx *= norm;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) s_red[par][warp] = mx;
            __syncthreads();
            // every warp reduces the per-warp maxima (one load per lane)
            float rowmax = lane < (int)(blockDim.x >> 5) ? s_red[par][lane] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) rowmax = fmaxf(rowmax, __shfl_xor_sync(0xffffffffu, rowmax, o));
            float scale = 1.f;
            if (rowmax > 0.f && isfinite(rowmax)) {
                int e;
                frexpf(rowmax, &e);  // rowmax < 2^e
                scale = ldexpf(1.f, 14 - e);
            }
            const float f = norm * scale;  // scale is a power of two: one rounding, as xr 2^e
            if (XQ) {  // decode GEMV operand: X = round(xr 2^e), bytes per 8-column group
                int sum = 0;
                if (c0 < p.len_pad) {
                    uint32_t hb[4] = {0u, 0u, 0u, 0u}, lb[4] = {0u, 0u, 0u, 0u};
                    uint32_t hx[8];
#pragma unroll
                    for (int j = 0; j < VPT; ++j) {
                        const int X = __float2int_rn(v[j] * f);
                        sum += X;
                        hb[j >> 2] |= (uint32_t)((X >> 8) & 0xFF) << (8 * (j & 3));
                        lb[j >> 2] |= (uint32_t)(X & 0xFF) << (8 * (j & 3));
                        const __half hX = __int2half_rn(X);
                        if (j & 1) hx[j >> 1] |= (uint32_t)__half_as_ushort(hX) << 16;
                        else hx[j >> 1] = __half_as_ushort(hX);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.xq + ((size_t)b * p.len_pad + c0) * 2);
                    dst[0] = make_uint4(hb[0], hb[1], lb[0], lb[1]);  // group c0 / 8
                    dst[1] = make_uint4(hb[2], hb[3], lb[2], lb[3]);  // group c0 / 8 + 1
                    if (p.xh) {
                        uint4 *dh = reinterpret_cast<uint4 *>(p.xh + (size_t)b * p.len_pad + c0);
                        dh[0] = make_uint4(hx[0], hx[1], hx[2], hx[3]);
                        dh[1] = make_uint4(hx[4], hx[5], hx[6], hx[7]);
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                if (lane == 0) s_sum[par][warp] = sum;
                __syncthreads();
                if (tid == 0) {
                    long long total = 0;
                    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += s_sum[par][w];
                    p.info[b] = glq_rowinfo{total, 1.f / scale, 0.f};
                }
            } else {
                if (c0 < p.len_pad) {  // padding columns [len, len_pad) hold zeros
                    uint32_t w[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const __half2 h2 = __floats2half2_rn(v[2 * j] * f, v[2 * j + 1] * f);
                        w[j] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.xh + (size_t)b * p.len_pad + c0);
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
                if (tid == 0) p.info[b] = glq_rowinfo{0, 1.f / scale, 0.f};
            }
        } else if (valid) {
            float y[VPT];
            const uint32_t sbr = opaque(sb);  // sign masks rebuilt per row, not kept live
#pragma unroll
            for (int j = 0; j < VPT; ++j) y[j] = flip(v[j] * norm, sbr, j);
            const size_t off = (size_t)b * p.len + c0;
            for (int q = 0; q < valid / 8; ++q) {
                const float *r = y + 8 * q;
                if (p.y_dtype == 2) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.y) + off + 8 * q);
                    dst[0] = make_float4(r[0], r[1], r[2], r[3]);
                    dst[1] = make_float4(r[4], r[5], r[6], r[7]);
                } else {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if (p.y_dtype == 1) {
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(r[2 * j], r[2 * j + 1]);
                            w[j] = *reinterpret_cast<const uint32_t *>(&h2);
                        } else {
                            const __half2 h2 = __floats2half2_rn(r[2 * j], r[2 * j + 1]);
                            w[j] = *reinterpret_cast<const uint32_t *>(&h2);
                        }
                    }
                    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.y) + off + 8 * q) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    }
    cp_async_wait_all();  // nothing may be in flight at exit (no copy is issued past the last row)
}

}  // namespace

bool rht_rows_supported(int len) { return len <= (1 << 14) && len >= 8; }

namespace {

int rows_log2(int cover) {
    int L = 9;  // at least one warp
    while ((1 << L) < cover) ++L;
    return L;
}

template <bool IN, bool XQ, int L>
cudaError_t launch_rows_t(const RowsParams &p, int B, cudaStream_t s, bool pdl) {
    const void *fn = (const void *)rht_rows_kernel<IN, XQ, L>;
    const int threads = 1 << (L - 4);
    // the row buffer and the staging buffer of the next row's raw input
    const size_t smem = (sizeof(float) << L) + (size_t)threads * (IN ? 32 : 64);
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    // persistent grid: every CTA that fits on the device at once, at most one
    // per row (SM count and occupancy queried once per device, not per call)
    constexpr int MAX_DEV = 64;
    static int sms_of[MAX_DEV] = {}, per_sm_of[MAX_DEV] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int sms = dev < MAX_DEV ? sms_of[dev] : 0, per_sm = dev < MAX_DEV ? per_sm_of[dev] : 0;
    if (sms <= 0 || per_sm <= 0) {
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
        if (e != cudaSuccess) return e;
        if (dev < MAX_DEV) {
            sms_of[dev] = sms;
            per_sm_of[dev] = per_sm;
        }
    }
    const int grid = (int)std::min<long long>((long long)B, (long long)std::max(1, sms) * std::max(1, per_sm));
    RowsParams q = p;
    int nrows = B;
    void *args[] = {&q, &nrows};
    return launch_ex(fn, dim3(grid), dim3(threads), smem, s, pdl, args);
}

// IN: input side; XQ: the decode operand (bytes of X) instead of fp16 xr 2^e
template <bool IN, bool XQ>
cudaError_t launch_rows_sel(const RowsParams &p, int B, cudaStream_t s, bool pdl) {
    const int cover = IN ? p.len_pad : p.len;
    switch (rows_log2(cover)) {
        case 9: return launch_rows_t<IN, XQ, 9>(p, B, s, pdl);
        case 10: return launch_rows_t<IN, XQ, 10>(p, B, s, pdl);
        case 11: return launch_rows_t<IN, XQ, 11>(p, B, s, pdl);
        case 12: return launch_rows_t<IN, XQ, 12>(p, B, s, pdl);
        case 13: return launch_rows_t<IN, XQ, 13>(p, B, s, pdl);
        case 14: return launch_rows_t<IN, XQ, 14>(p, B, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_rht_rows(const RowsParams &p, bool input, int B, cudaStream_t s, bool pdl) {
    if (B <= 0) return cudaErrorInvalidValue;
    if (!input) return launch_rows_sel<false, false>(p, B, s, pdl);
    return p.xq ? launch_rows_sel<true, true>(p, B, s, pdl) : launch_rows_sel<true, false>(p, B, s, pdl);
}

}  // namespace glq
