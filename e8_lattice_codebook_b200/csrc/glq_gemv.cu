// glq_gemv.cu -- decode-phase (B <= 16) codebook GEMV of the GLQ linear
// layer: z[b][r] = sum_k W^[r][k] xr[b][k] computed directly against the
// compressed indices, W never materialised (glq 0.5.1 PyPI page, "How it
// works" 4 and "Inference kernels": indices read from HBM, 8-D codewords
// gathered from an on-chip codebook, matmul accumulated against them;
// split over K with a fixed-order reduction, "Bit-exact determinism").
//
// Design (B200, sm_100a):
//   * persistent CTAs, one per SM, each holding the negation-folded nibble
//     codebook (4 B per entry, ~145 KB) in shared memory, loaded once per
//     launch with a bulk async copy; the copy and the first index loads are
//     issued before the programmatic-dependent-launch wait, so they overlap
//     the input RHT;
//   * a task is (band of 16 row tiles = 256 rows, split of the chunk range);
//     each warp owns one 16-row tile and streams its fragment-native index
//     stream with coalesced 128-bit non-allocating loads, 4 chunks ahead;
//   * each lane turns a 16-bit code into one whole codeword (fold, one
//     shared-memory word, two masks) that is exactly its two A registers of
//     the integer mma.m16n8k32 (u8 codeword bytes v = 2x + 6 times the high
//     (s8) and low (u8) bytes of the 16-bit activations); accumulation is
//     exact in int32, so the result does not depend on summation order;
//   * the 3 bpw residual stage (arbitrary fp16 table) uses mma.m16n8k16 on
//     fp16 operands with fp32 accumulation;
//   * per task, partial sums go to a workspace in fp64; the last CTA to
//     finish a band (atomic counter, no waiting) adds the splits in fixed
//     order and writes the band's final z.  When every CTA has one task and
//     a band's splits fit one thread-block cluster, each split stores its
//     partials into the shared memory of the CTA that owns that share of the
//     band (distributed shared memory), and after one cluster barrier every
//     CTA adds its share in the same fixed order (no global round trip, no
//     last arriver);
//   * small batches fuse both transforms (one launch per layer): each task
//     rotates, scales and quantises its own aligned column range of x in
//     shared memory (a Hadamard block of size N = 2^a S restricted to an
//     aligned range of S outputs is H_S applied to the 2^a-term signed fold
//     of the block), and the last band to finish a Hadamard block of m
//     transforms that block of z in shared memory and writes y.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "glq_kernels.cuh"

namespace cg = cooperative_groups;

namespace glq {

namespace {

constexpr uint32_t TABLE_WAIT_POLLS = 1u << 24;

struct Acc {
    int hi[2][4], lo[2][4];  // [n-tile][fragment]
};

template <int NT>
__device__ __forceinline__ void zero(Acc &a) {
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) a.hi[i][j] = a.lo[i][j] = 0;
}

// Shared addresses of the folded table: T[0] and T[-neg_base].
struct TableRef {
    uint32_t base, neg;
};

__device__ __forceinline__ TableRef table_ref(const uint32_t *T, FoldParams fold) {
    const uint32_t b = (uint32_t)__cvta_generic_to_shared(T);
    return TableRef{b, b - 4u * (uint32_t)fold.neg_base};
}

// One stage (one code per row) of one super-tile: codes of rows g and g+8.
// The A operands are 16 v (see table_a16), so the int32 sums are 16 sum v X:
// at most 16 * 12 * 255 * 32768 < 2^31 for the low bytes over the longest row.
template <int NT>
__device__ __forceinline__ void stage_int(TableRef T, FoldParams fold, LookupConsts kc, uint32_t codes,
                                          const uint4 &x0, const uint4 &x1, Acc &acc) {
    uint32_t a[4];
    table_a16(T.base, T.neg, codes & 0xFFFFu, (uint32_t)fold.nb, kc, a[0], a[2]);
    table_a16(T.base, T.neg, codes >> 16, (uint32_t)fold.nb, kc, a[1], a[3]);
    mma_u8s8(acc.hi[0], a, x0.x, x0.y);
    mma_u8u8(acc.lo[0], a, x0.z, x0.w);
    if (NT == 2) {
        mma_u8s8(acc.hi[NT - 1], a, x1.x, x1.y);
        mma_u8u8(acc.lo[NT - 1], a, x1.z, x1.w);
    }
}

// 16-byte load of activations: global (read-only path) or shared memory
template <bool XS>
__device__ __forceinline__ uint4 ld_x(const void *p) {
    if (XS) return *reinterpret_cast<const uint4 *>(p);
    return ldg_v4(p);
}

// One chunk (128 columns = 4 super-tiles of 32) of a warp's row tile: q1
// holds the primary codes, qr[k] those of 16-bit residual stage k, q8 the
// 8-bit stage's indices (odd bpw).
template <int BPW, int NT, bool XS>
__device__ __forceinline__ void process_chunk(TableRef T, const uint4 *R8, FoldParams fold, LookupConsts kc,
                                              const uint4 &q1, const uint4 (&qr)[Stages<BPW>::NA],
                                              const uint2 &q8, const uint4 *xq0, const uint4 *xq1,
                                              const __half *xh0, const __half *xh1, bool has0, bool has1,
                                              Acc &acc1, Acc (&accs)[Stages<BPW>::NA], float accr[2][4]) {
    constexpr int N16 = Stages<BPW>::N16;
    const uint32_t p1[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
        if (has0) x0 = ld_x<XS>(xq0 + 4 * s);
        if (NT == 2 && has1) x1 = ld_x<XS>(xq1 + 4 * s);
        stage_int<NT>(T, fold, kc, p1[s], x0, x1, acc1);
#pragma unroll
        for (int k = 0; k < N16; ++k) {
            const uint32_t pk[4] = {qr[k].x, qr[k].y, qr[k].z, qr[k].w};
            stage_int<NT>(T, fold, kc, pk[s], x0, x1, accs[k]);
        }
        if (Stages<BPW>::U8) {
            // bytes 2s (row g) and 2s+1 (row g+8) of the 8-byte payload
            const uint32_t word = (s < 2) ? q8.x : q8.y;
            const uint32_t sh = (s & 1) * 16;
            const uint4 ra = R8[(word >> sh) & 0xFFu];
            const uint4 rb = R8[(word >> (sh + 8)) & 0xFFu];
            const uint32_t lo[4] = {ra.x, rb.x, ra.y, rb.y};
            const uint32_t hi[4] = {ra.z, rb.z, ra.w, rb.w};
            uint4 h0 = make_uint4(0, 0, 0, 0), h1 = make_uint4(0, 0, 0, 0);
            if (has0) h0 = ld_x<XS>(xh0 + 32 * s);
            if (NT == 2 && has1) h1 = ld_x<XS>(xh1 + 32 * s);
            mma_16816(accr[0], lo, h0.x, h0.y);
            mma_16816(accr[0], hi, h0.z, h0.w);
            if (NT == 2) {
                mma_16816(accr[NT - 1], lo, h1.x, h1.y);
                mma_16816(accr[NT - 1], hi, h1.z, h1.w);
            }
        }
    }
}

// The index words of chunk slot i of every stage (fragment-native streams).
template <int BPW>
__device__ __forceinline__ void load_codes(const GemvParams &p, size_t i, uint4 &q1, uint4 (&qr)[Stages<BPW>::NA],
                                           uint2 &q8) {
    q1 = ldg_nc_v4(p.idx1 + i);
#pragma unroll
    for (int k = 0; k < Stages<BPW>::N16; ++k) qr[k] = ldg_nc_v4(p.idx16[k] + i);
    if (Stages<BPW>::U8) q8 = ldg_nc_v2(p.idx8 + i);
}

// sum v X of one accumulator pair from its 16 v sums (exact: a multiple of 16)
__device__ __forceinline__ double exact_sum(int hi, int lo) {
    return (double)((long long)hi * 256 + (long long)lo) * 0.0625;
}

// z of (token b, any row) from D = sum over splits of the partials:
// z = ws 2^-e (D - 6 corr_mult sum X) / 2.
__device__ __forceinline__ float finish_z(const GemvParams &p, int b, double D) {
    const glq_rowinfo info = p.info[b];
    const double corr = (double)GLQ_NIB_OFFSET * p.corr_mult * (double)info.sum_x;
    return (float)((D - corr) * (0.5 * (double)p.ws * (double)info.inv_scale));
}

// ---------------------------------------------------------------------------
// Fused transforms
// ---------------------------------------------------------------------------

struct TaskRow {  // per token, over the task's column range
    int sum_x;        // exact sum of X
    float inv_scale;  // 2^-e
};

// 8 activations (fp16 or bf16 bits) as float
__device__ __forceinline__ void unpack8_act(const uint4 &r, int bf16, float v[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (bf16) {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        } else {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[j]));
            v[2 * j] = f.x;
            v[2 * j + 1] = f.y;
        }
    }
}

// butterflies of spans 1, 2, 4 on 8 consecutive values (Sylvester order)
__device__ __forceinline__ void fwht8(float v[8]) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

// A run of one Hadamard transform within a row of a shared-memory buffer:
// elements [start, start + size), size a power of two >= 8, start a
// multiple of size; norm = 1/sqrt(size of the whole block).
struct Seg {
    int start, size;
    float norm;
};

// Butterflies of spans 8 .. size/2 on every segment of every row (rows of
// `ld` floats), the spans 1, 2, 4 being done already per 8-vector.  Spans up
// to 128 run in registers across the lanes of a warp (32 consecutive
// 8-vectors, shuffles); longer spans run in shared memory, one barrier per
// span.  Every thread of the CTA calls it; it ends with a barrier.
template <int THREADS>
__device__ void fwht_segments(float *u, int nrows, int ld, const Seg *segs, int nseg) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vrow = ld / 8, total = nrows * vrow;
    int smax = 0;
    for (int i = 0; i < nseg; ++i) smax = max(smax, segs[i].size);
    if (smax > 8) {
        for (int v0 = warp * 32; v0 < total; v0 += THREADS) {
            const int v = v0 + lane;
            const bool valid = v < total;
            const int row = valid ? v / vrow : 0;
            const int q = valid ? 8 * (v - row * vrow) : 0;
            int S = 0;
            for (int i = 0; i < nseg; ++i)
                if (q >= segs[i].start && q < segs[i].start + segs[i].size) S = segs[i].size;
            float r[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            float *src = u + (size_t)row * ld + q;
            if (valid && S > 8) {
                const float4 a = *reinterpret_cast<const float4 *>(src);
                const float4 c = *reinterpret_cast<const float4 *>(src + 4);
                r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
                r[4] = c.x; r[5] = c.y; r[6] = c.z; r[7] = c.w;
            }
#pragma unroll
            for (int k = 0; k < 5; ++k) {  // spans 8, 16, 32, 64, 128
                const int off = 1 << k;
                const bool act = valid && (8 << k) < S;
                const bool upper = (lane & off) != 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float o = __shfl_xor_sync(0xffffffffu, r[j], off);
                    if (act) r[j] = upper ? o - r[j] : r[j] + o;
                }
            }
            if (valid && S > 8) {
                *reinterpret_cast<float4 *>(src) = make_float4(r[0], r[1], r[2], r[3]);
                *reinterpret_cast<float4 *>(src + 4) = make_float4(r[4], r[5], r[6], r[7]);
            }
        }
    }
    __syncthreads();
    for (int h = 256; h < smax; h <<= 1) {
        for (int i = 0; i < nseg; ++i) {
            if (segs[i].size <= h) continue;
            const int pairs = segs[i].size >> 1;
            for (int e = threadIdx.x; e < nrows * pairs; e += THREADS) {
                const int row = e / pairs, q0 = e - row * pairs;
                float *r = u + (size_t)row * ld + segs[i].start + ((q0 / h) * 2 * h) + (q0 % h);
                const float a = r[0], c = r[h];
                r[0] = a + c;
                r[h] = a - c;
            }
        }
        __syncthreads();
    }
}

// Constant data of a task's fused input, fetched before the wait on the
// previous kernel: the S_in sign words of every Hadamard block the task's
// column range meets (a contiguous run of columns), into `sw` starting at
// word `*w0`.  Every thread calls it; ends with a barrier.
template <int THREADS>
__device__ void fused_input_signs(const GemvParams &p, int k0, int klen, uint32_t *sw, int *w0) {
    int lo = 1 << 30, hi = 0;
    for (int bi = 0; bi < p.nblk_n; ++bi) {
        const int o = p.blk_off_n[bi], N = p.blk_len_n[bi];
        if (max(k0, o) < min(k0 + klen, o + N)) {
            lo = min(lo, o);
            hi = max(hi, o + N);
        }
    }
    const int a = lo >> 5, e = (hi + 31) >> 5;  // at most n / 32 + 1 words
    for (int i = threadIdx.x; i < e - a; i += THREADS) sw[i] = __ldg(p.sin_bits + a + i);
    *w0 = a;
    __syncthreads();
}

// Warp-per-token tail of the input transform for the common task shape:
// the range [k0, k0 + 32V) (V = 4, 8 or 16) meets one Hadamard block of n,
// as an aligned part of it or as the whole block followed by padding past n.
// u holds the token's folded values f (positions past S, the range's
// columns inside the block, are not read: zeros).  Lane l holds positions
// l V .. l V + V - 1: spans below V in registers, V .. 16 V as shuffles, then
// the row max, the scale and X, with no CTA barrier.
template <int BPW, int V>
__device__ __forceinline__ void warp_transform(const GemvParams &p, int b, int N, int S, const float *u,
                                               uint4 *xs, __half *xhs, TaskRow *rows) {
    const int lane = threadIdx.x & 31;
    const int klen = 32 * V, p0 = lane * V;
    float v[V];
#pragma unroll
    for (int q = 0; q < V / 4; ++q) {
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p0 + 4 * q < S) r = *reinterpret_cast<const float4 *>(u + (size_t)b * klen + p0 + 4 * q);
        v[4 * q] = r.x;
        v[4 * q + 1] = r.y;
        v[4 * q + 2] = r.z;
        v[4 * q + 3] = r.w;
    }
    // a span applies iff it is below S (positions past S hold zeros)
#pragma unroll
    for (int h = 1; h < V; h <<= 1)
        if (h < S)
#pragma unroll
            for (int j = 0; j < V; ++j)
                if ((j & h) == 0) {
                    const float a = v[j], c = v[j + h];
                    v[j] = a + c;
                    v[j + h] = a - c;
                }
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        if ((V << k) >= S) break;
        const bool upper = (lane >> k) & 1;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, v[j], 1 << k);
            v[j] = upper ? o - v[j] : v[j] + o;
        }
    }
    const float nrm = __frsqrt_rn((float)N);
    float mx = 0.f;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        v[j] *= nrm;
        mx = fmaxf(mx, fabsf(v[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float scale = 1.f;
    if (mx > 0.f && isfinite(mx)) {
        int ex;
        frexpf(mx, &ex);
        scale = ldexpf(1.f, min(14 - ex, 126));  // scale and 1 / scale normal for the tiniest rows
    }
    int sum = 0;
    uint32_t hb[V / 4], lb[V / 4];
#pragma unroll
    for (int q = 0; q < V / 4; ++q) hb[q] = lb[q] = 0u;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const int X = __float2int_rn(v[j] * scale);
        sum += X;
        hb[j >> 2] |= (uint32_t)((X >> 8) & 0xFF) << (8 * (j & 3));
        lb[j >> 2] |= (uint32_t)(X & 0xFF) << (8 * (j & 3));
        if (Stages<BPW>::U8) xhs[(size_t)b * klen + p0 + j] = __int2half_rn(X);
    }
    // per 8-column group: 8 high bytes, then 8 low bytes
    uint32_t *xw = reinterpret_cast<uint32_t *>(xs + (size_t)b * (klen / 8));
#pragma unroll
    for (int q = 0; q < V / 4; ++q) {
        const int c4 = p0 / 4 + q;  // 4-column quarter of the range
        xw[(c4 >> 1) * 4 + (c4 & 1)] = hb[q];
        xw[(c4 >> 1) * 4 + 2 + (c4 & 1)] = lb[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
        rows[b].sum_x = sum;
        rows[b].inv_scale = 1.f / scale;
    }
}

// The task's activations for columns [k0, k0 + klen): xr = H_n (S_in x)
// restricted to the range, scaled per token by 2^e (max |xr| 2^e < 2^14 over
// the range), rounded to X and stored as the GEMV consumes it: xs[b][group]
// = 8 high bytes, 8 low bytes; xhs[b][col] = X as fp16 (3 bpw).  The range is
// aligned and a power-of-two multiple of 128 columns, so within each Hadamard
// block it meets it is either the whole block or an aligned part of size S
// of a block of size N: then xr = N^-1/2 H_S f with f[j] = sum over the
// N/S sub-blocks t of (-1)^popc(i t) (S_in x)[t S + j], i the part's index.
template <int BPW, int THREADS>
__device__ void fused_input(const GemvParams &p, int k0, int klen, uint4 *xs, __half *xhs, float *u,
                            TaskRow *rows, unsigned *s_max, Seg *segs, const uint32_t *sw, int w0) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int B = p.B, k1 = k0 + klen;
    // The warp-per-token tail (warp_transform) applies when the range meets
    // one Hadamard block, from the range's first column, and spans 128, 256
    // or 512 columns; the condition is the same in every thread.
    int wo = 0, wN = 0, wseg = 0;
    for (int bi = 0; bi < p.nblk_n; ++bi) {
        const int o = p.blk_off_n[bi], N = p.blk_len_n[bi];
        if (max(k0, o) < min(k1, o + N)) {
            wo = o;
            wN = N;
            ++wseg;
        }
    }
    const bool warp_tail = B <= THREADS / 32 && (klen == 128 || klen == 256 || klen == 512) && wseg == 1 &&
                           max(k0, wo) == k0;
    if (!warp_tail) {
        for (int e = tid; e < B * klen; e += THREADS) u[e] = 0.f;  // columns >= n stay zero
        if (tid < GLQ_DECODE_MAX_B) {
            s_max[tid] = 0u;
            rows[tid].sum_x = 0;
        }
        __syncthreads();
    }
    int nseg = 0;  // the task's segments (identical in every thread)
    for (int bi = 0; bi < p.nblk_n; ++bi) {
        const int o = p.blk_off_n[bi], N = p.blk_len_n[bi];
        const int lo = max(k0, o), hi = min(k1, o + N);
        if (lo >= hi) continue;
        if (tid == 0) segs[nseg] = Seg{lo - k0, hi - lo, __frsqrt_rn((float)N)};
        ++nseg;
        const int S = hi - lo;  // N or an aligned part of it
        const int A = N / S, ihi = (lo - o) / S, nv = S / 8;
        const int items = B * nv;
        int G = 1;  // lanes sharing one 8-column vector (split over the fold terms)
        while (G < 32 && 2 * G <= A && items * 2 * G <= THREADS) G *= 2;
        for (int it0 = 0; it0 < items * G; it0 += THREADS) {
            const int it = it0 + tid;
            const bool valid = it < items * G;
            const int grp = it & (G - 1), item = it / G;
            const int b = valid ? item / nv : 0, v = valid ? item - b * nv : 0;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (valid) {
                // four terms per round: their loads are all in flight before any is used
                for (int jh0 = grp; jh0 < A; jh0 += 4 * G) {
                    uint4 r[4];
                    uint32_t flip[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int jh = jh0 + q * G;
                        const int col = o + jh * S + 8 * v;
                        r[q] = make_uint4(0, 0, 0, 0);
                        flip[q] = 0u;
                        if (jh < A) {
                            r[q] = ldg_v4(static_cast<const uint16_t *>(p.x) + (size_t)b * p.n + col);
                            const uint32_t sb = (sw[(col >> 5) - w0] >> (col & 31)) & 0xFFu;
                            flip[q] = sb ^ ((__popc(ihi & jh) & 1) ? 0xFFu : 0u);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float xv[8];
                        unpack8_act(r[q], p.x_bf16, xv);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[j] += ((flip[q] >> j) & 1u) ? -xv[j] : xv[j];
                    }
                }
            }
            // fixed-order reduction over the G lanes of a vector
            for (int off = 1; off < G; off <<= 1)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
            if (valid && grp == 0) {
                if (!warp_tail) fwht8(acc);
                float *dst = u + (size_t)b * klen + (lo - k0) + 8 * v;
                *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                *reinterpret_cast<float4 *>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
        }
    }
    __syncthreads();
    if (warp_tail) {
        const int S = min(k1, wo + wN) - k0;  // klen, or the whole block followed by padding
        const int warp = tid >> 5;
        if (warp < B) {
            if (klen == 128) warp_transform<BPW, 4>(p, warp, wN, S, u, xs, xhs, rows);
            else if (klen == 256) warp_transform<BPW, 8>(p, warp, wN, S, u, xs, xhs, rows);
            else warp_transform<BPW, 16>(p, warp, wN, S, u, xs, xhs, rows);
        }
        __syncthreads();
        return;
    }
    fwht_segments<THREADS>(u, B, klen, segs, nseg);
    // normalise per block, row max per token
    const int nvec = klen / 8;
    for (int e = tid; e < B * nvec; e += THREADS) {
        const int b = e / nvec, v = e - b * nvec;
        float nrm = 0.f;
        for (int i = 0; i < nseg; ++i)
            if (8 * v >= segs[i].start && 8 * v < segs[i].start + segs[i].size) nrm = segs[i].norm;
        float *r = u + (size_t)b * klen + 8 * v;
        float mx = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            r[j] *= nrm;
            mx = fmaxf(mx, fabsf(r[j]));
        }
        atomicMax(s_max + b, __float_as_uint(mx));
    }
    __syncthreads();
    // X = round(xr 2^e), interleaved bytes, exact sum
    for (int e = tid; e < B * nvec; e += THREADS) {
        const int b = e / nvec, v = e - b * nvec;
        const float rowmax = __uint_as_float(s_max[b]);
        float scale = 1.f;
        if (rowmax > 0.f && isfinite(rowmax)) {
            int ex;
            frexpf(rowmax, &ex);
            scale = ldexpf(1.f, min(14 - ex, 126));  // scale and 1 / scale normal for the tiniest rows
        }
        const float *r = u + (size_t)b * klen + 8 * v;
        uint32_t hb[2] = {0u, 0u}, lb[2] = {0u, 0u};
        int sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int X = __float2int_rn(r[j] * scale);
            sum += X;
            hb[j >> 2] |= (uint32_t)((X >> 8) & 0xFF) << (8 * (j & 3));
            lb[j >> 2] |= (uint32_t)(X & 0xFF) << (8 * (j & 3));
            if (Stages<BPW>::U8) xhs[(size_t)b * klen + 8 * v + j] = __int2half_rn(X);
        }
        xs[(size_t)b * nvec + v] = make_uint4(hb[0], hb[1], lb[0], lb[1]);
        atomicAdd(&rows[b].sum_x, sum);
        if (v == 0) rows[b].inv_scale = 1.f / scale;
    }
    (void)lane;
    __syncthreads();
}

// y for Hadamard block `blk` of m, all tokens: the block's z (complete in
// global memory) is transformed in shared memory `buf` (B x N floats).
template <int THREADS>
__device__ void fused_output(const GemvParams &p, int blk, float *buf) {
    const int o = p.blk_off_m[blk], N = p.blk_len_m[blk], B = p.B;
    const int nvec = N / 8;
    for (int e = threadIdx.x; e < B * nvec; e += THREADS) {
        const int b = e / nvec, v = e - b * nvec;
        const float4 *zp = reinterpret_cast<const float4 *>(p.z + (size_t)b * p.m_pad + o + 8 * v);
        const float4 a = __ldcg(zp), c = __ldcg(zp + 1);
        float r[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
        fwht8(r);
        float *dst = buf + (size_t)b * N + 8 * v;
        *reinterpret_cast<float4 *>(dst) = make_float4(r[0], r[1], r[2], r[3]);
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(r[4], r[5], r[6], r[7]);
    }
    __syncthreads();
    const Seg seg{0, N, 0.f};
    fwht_segments<THREADS>(buf, B, N, &seg, 1);
    const float nrm = __frsqrt_rn((float)N);
    for (int e = threadIdx.x; e < B * nvec; e += THREADS) {
        const int b = e / nvec, v = e - b * nvec;
        const int col = o + 8 * v;
        const uint32_t sb = (p.sout_bits[col >> 5] >> (col & 31)) & 0xFFu;
        const float *r = buf + (size_t)b * N + 8 * v;
        float y[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = ((sb >> j) & 1u) ? -(r[j] * nrm) : r[j] * nrm;
        const size_t off = (size_t)b * p.m + col;
        if (p.y_dtype == 2) {  // fp32
            float4 *yp = reinterpret_cast<float4 *>(static_cast<float *>(p.y) + off);
            yp[0] = make_float4(y[0], y[1], y[2], y[3]);
            yp[1] = make_float4(y[4], y[5], y[6], y[7]);
        } else {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (p.y_dtype == 1) {  // bf16
                    const __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
                    w[j] = *reinterpret_cast<const uint32_t *>(&h);
                } else {
                    const __half2 h = __floats2half2_rn(y[2 * j], y[2 * j + 1]);
                    w[j] = *reinterpret_cast<const uint32_t *>(&h);
                }
            }
            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.y) + off) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

template <int BPW, int NT, bool FIN, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) gemv_kernel(GemvParams p) {
    constexpr int THREADS = WARPS * 32;
    constexpr int BAND_ROWS = WARPS * GLQ_ROW_TILE;
    extern __shared__ __align__(16) uint4 smem_u4[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int s_last;
    __shared__ TaskRow s_rows[GLQ_DECODE_MAX_B];
    __shared__ unsigned s_max[GLQ_DECODE_MAX_B];
    __shared__ int s_pending[GLQ_MAX_BLOCKS];
    __shared__ Seg s_segs[GLQ_MAX_BLOCKS];
    __shared__ uint32_t s_sign[GLQ_RHT_MAX_N / 32 + 2];  // fused input: S_in words of the task's blocks
    __shared__ int s_sign_w0;
    __shared__ int s_npending;
    uint32_t *T = reinterpret_cast<uint32_t *>(smem_u4);
    const TableRef tref = table_ref(T, p.fold);
    uint4 *R8 = smem_u4 + p.table_words / 4;
    // fused input: [xs: B x klen/8 uint4][xhs: B x klen halves (3 bpw)][u: B x klen floats]
    const int klen_max = min(p.cps, p.KC) * GLQ_CHUNK_K;
    uint4 *xs = R8 + (Stages<BPW>::U8 ? 256 : 0);
    __half *xhs = reinterpret_cast<__half *>(xs + (size_t)p.B * klen_max / 8);
    float *ubuf = reinterpret_cast<float *>(xhs + (Stages<BPW>::U8 ? (size_t)p.B * klen_max : 0));
    // cluster reduction: the partial sums of this CTA's share of the band,
    // [split][share] (fp64), stored by every split of the cluster
    double *spart = reinterpret_cast<double *>(reinterpret_cast<char *>(smem_u4) + p.spart_off);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int ntasks = p.bands * p.splits;

    // 1. codebook into shared memory (constant data: before the PDL wait)
    if (tid == 0) {
        mbar_init(&bar, 1);
        s_npending = 0;
    }
    __syncthreads();
    if (tid == 0) {
        const uint32_t tbytes = (uint32_t)p.table_words * 4u;
        const uint32_t rbytes = Stages<BPW>::U8 ? 256u * 16u : 0u;
        mbar_expect_tx(&bar, tbytes + rbytes);
        const uint32_t piece = 32768u;
        for (uint32_t off = 0; off < tbytes; off += piece) {
            const uint32_t len = tbytes - off < piece ? tbytes - off : piece;
            bulk_g2s(reinterpret_cast<char *>(T) + off, reinterpret_cast<const char *>(p.table) + off,
                     len, &bar);
        }
        if (Stages<BPW>::U8) bulk_g2s(R8, p.tab8, rbytes, &bar);
    }
    pdl_launch_dependents();

    // 2. index loads of the first task (constant data: before the PDL wait)
    constexpr int NA = Stages<BPW>::NA;
    uint4 r1[GEMV_PREFETCH], rq[GEMV_PREFETCH][NA];
    uint2 r8[GEMV_PREFETCH];
    int task = blockIdx.x;
    int rt = 0, c0 = 0, c1 = 0;
    auto task_geom = [&](int tk) {
        const int band = tk / p.splits, split = tk - band * p.splits;
        rt = band * WARPS + warp;
        c0 = split * p.cps;
        c1 = min(p.KC, c0 + p.cps);
    };
    auto prefetch = [&]() {
        const size_t base = ((size_t)rt * p.KC) * 32 + lane;
#pragma unroll
        for (int i = 0; i < GEMV_PREFETCH; ++i) {
            if (rt < p.RT && c0 + i < c1) load_codes<BPW>(p, base + (size_t)(c0 + i) * 32, r1[i], rq[i], r8[i]);
        }
    };
    if (task < ntasks) {
        task_geom(task);
        prefetch();
        // The rest of the first task's index range (constant data) into L2
        // now, so that the chunks the loop reads after the wait hit L2
        // instead of paying a DRAM round trip each (short tasks, where the
        // one-chunk register prefetch cannot cover the latency).
        if (FIN) {
            fused_input_signs<THREADS>(p, c0 * GLQ_CHUNK_K, (c1 - c0) * GLQ_CHUNK_K, s_sign, &s_sign_w0);
            // the columns of x the first task folds: Hadamard blocks met by its range
            const int lo = s_sign_w0 * 32;
            const int hi = min(p.n, lo + (int)(sizeof(s_sign) / 4) * 32);
            for (int b = 0; b < p.B; ++b)
                for (int col = lo + 64 * tid; col < hi; col += 64 * THREADS)  // 128-byte lines of bf16 / fp16
                    prefetch_l2(static_cast<const uint16_t *>(p.x) + (size_t)b * p.n + col);
        }
    }

    // 3. activations (and row info) come from the previous kernel; with the
    // input transform fused, the codebook copy keeps landing meanwhile
    pdl_wait();
    auto wait_table = [&]() {  // every thread calls it; the verdict is the CTA's
        const bool ok = __syncthreads_and(mbar_wait_bounded(&bar, 0, TABLE_WAIT_POLLS) ? 1 : 0) != 0;
        if (ok) return true;
        if (tid == 0) atomicOr(p.err, GLQ_DEVERR_TIMEOUT);
        mbar_wait_bounded(&bar, 0, TABLE_WAIT_POLLS);  // let the copy land before exiting
        if (p.clu) cg::this_cluster().sync();  // leaving early: still take the reduction's cluster barrier
        return false;
    };
    if (!FIN && !wait_table()) return;

    const bool has0 = g < p.B, has1 = (g + 8) < p.B;
    const size_t xq_row = (size_t)p.n_pad / 8;  // uint4 (one group) per 8 columns
    const uint4 *xq0 = FIN ? nullptr : reinterpret_cast<const uint4 *>(p.xq) + (size_t)g * xq_row + t;
    const uint4 *xq1 = FIN ? nullptr : reinterpret_cast<const uint4 *>(p.xq) + (size_t)(g + 8) * xq_row + t;
    const __half *xh0 = (!FIN && p.xh) ? p.xh + (size_t)g * p.n_pad + 8 * t : nullptr;
    const __half *xh1 = (!FIN && p.xh) ? p.xh + (size_t)(g + 8) * p.n_pad + 8 * t : nullptr;

    for (bool first = true; task < ntasks; task += gridDim.x, first = false) {
        if (!first) {
            task_geom(task);
            prefetch();
        }
        const int band = task / p.splits, split = task - band * p.splits;
        const int klen = (c1 - c0) * GLQ_CHUNK_K;
        if (FIN) {
            __syncthreads();  // the previous task's activations and row info are no longer read
            if (!first) fused_input_signs<THREADS>(p, c0 * GLQ_CHUNK_K, klen, s_sign, &s_sign_w0);
            fused_input<BPW, THREADS>(p, c0 * GLQ_CHUNK_K, klen, xs, xhs, ubuf, s_rows, s_max, s_segs, s_sign,
                                      s_sign_w0);
            if (first && !wait_table()) return;  // the CTA's common verdict: all threads return
        }
        Acc acc1, accs[NA];
        zero<NT>(acc1);
#pragma unroll
        for (int k = 0; k < NA; ++k) zero<NT>(accs[k]);
        float accr[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};

        if (rt < p.RT) {
            const size_t base = ((size_t)rt * p.KC + c0) * 32 + lane;
            size_t q_next = base + GEMV_PREFETCH * 32;  // slot of the next chunk to load
            const uint4 *px0, *px1;
            const __half *ph0, *ph1;
            if (FIN) {  // the task's range in shared memory, row stride klen
                px0 = xs + (size_t)g * (klen / 8) + t;
                px1 = xs + (size_t)(g + 8) * (klen / 8) + t;
                ph0 = Stages<BPW>::U8 ? xhs + (size_t)g * klen + 8 * t : nullptr;
                ph1 = Stages<BPW>::U8 ? xhs + (size_t)(g + 8) * klen + 8 * t : nullptr;
            } else {
                px0 = xq0 + (size_t)c0 * GLQ_GROUPS_PER_CHUNK;
                px1 = xq1 + (size_t)c0 * GLQ_GROUPS_PER_CHUNK;
                ph0 = xh0 ? xh0 + (size_t)c0 * GLQ_CHUNK_K : nullptr;
                ph1 = xh1 ? xh1 + (size_t)c0 * GLQ_CHUNK_K : nullptr;
            }
            int ahead = c0 + GEMV_PREFETCH;
            for (int c = c0; c < c1; c += GEMV_PREFETCH) {
#pragma unroll
                for (int i = 0; i < GEMV_PREFETCH; ++i) {
                    if (c + i < c1) {
                        uint4 q1 = r1[i], qr[NA];
                        uint2 q8 = r8[i];
#pragma unroll
                        for (int k = 0; k < NA; ++k) qr[k] = rq[i][k];
                        if (ahead < c1) load_codes<BPW>(p, q_next, r1[i], rq[i], r8[i]);
                        q_next += 32;
                        ++ahead;
                        process_chunk<BPW, NT, FIN>(tref, R8, p.fold, p.kc, q1, qr, q8, px0, px1, ph0, ph1, has0,
                                                    has1, acc1, accs, accr);
                        px0 += GLQ_GROUPS_PER_CHUNK;
                        px1 += GLQ_GROUPS_PER_CHUNK;
                        if (Stages<BPW>::U8) {
                            ph0 += GLQ_CHUNK_K;
                            ph1 += GLQ_CHUNK_K;
                        }
                    }
                }
            }
            // lane (g, t) holds rows g, g+8 and batch columns nt*8 + 2t, 2t+1
            const int row0 = rt * GLQ_ROW_TILE + g;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int b = nt * 8 + 2 * t + (j & 1);
                    const int row = row0 + (j >> 1) * 8;
                    if (b < p.B) {
                        double D = exact_sum(acc1.hi[nt][j], acc1.lo[nt][j]);
#pragma unroll
                        for (int k = 0; k < Stages<BPW>::N16; ++k)
                            D += p.rs16_d[k] * exact_sum(accs[k].hi[nt][j], accs[k].lo[nt][j]);
                        if (Stages<BPW>::U8) D += p.rs8_d * (double)accr[nt][j];
                        if (FIN) {  // this range's own scale and sum: a partial of x . w
                            D = (D - (double)GLQ_NIB_OFFSET * p.corr_mult * (double)s_rows[b].sum_x) *
                                (0.5 * (double)s_rows[b].inv_scale);
                        }
                        if (p.splits == 1) {
                            p.z[(size_t)b * p.m_pad + row] = FIN ? (float)(D * (double)p.ws) : finish_z(p, b, D);
                        } else if (p.clu) {
                            // to the cluster CTA that owns element (b, row) of the band, slot `split`
                            const int rows_b = min(BAND_ROWS, p.m_pad - band * BAND_ROWS);
                            const int per = (rows_b * p.B + p.clu - 1) / p.clu;
                            const int e = b * rows_b + (row - band * BAND_ROWS), owner = e / per;
                            cg::this_cluster().map_shared_rank(spart, owner)[split * per + (e - owner * per)] = D;
                        } else {
                            __stcg(p.partials + ((size_t)split * p.B + b) * p.m_pad + row, D);
                        }
                    }
                }
            }
        }

        // 4. band completion: the last split to finish reduces the band.  The
        // CTA barrier orders every thread's partial stores before thread 0's
        // release-acquire increment; the barrier after it hands the acquire to
        // the threads that read the other CTAs' partials.
        bool band_done = true;
        if (p.splits > 1 && p.clu) {
            // one task per CTA; the cluster's CTAs are the band's splits, rank =
            // split.  The band's (token, row) elements are dealt out in
            // contiguous shares; every split has stored its partial of each
            // element into the owner's shared memory, slot `split`.
            cg::cluster_group cluster = cg::this_cluster();
            cluster.sync();  // all partials are in their owners' shared memory
            const int S = p.clu, rank = (int)cluster.block_rank();
            const int r_base = band * BAND_ROWS;
            const int rows = min(BAND_ROWS, p.m_pad - r_base);
            const int total = rows * p.B, per = (total + S - 1) / S;
            const int e0 = rank * per, e1 = min(total, e0 + per);
            for (int e = e0 + tid; e < e1; e += THREADS) {
                const int b = e / rows, row = e - b * rows;
                double D = 0.0;
                for (int sp = 0; sp < S; ++sp) D += spart[sp * per + (e - e0)];  // fixed order
                p.z[(size_t)b * p.m_pad + r_base + row] = FIN ? (float)(D * (double)p.ws) : finish_z(p, b, D);
            }
        } else if (p.splits > 1) {
            __syncthreads();
            if (tid == 0) {
                const unsigned prev = atom_add_acq_rel_gpu(&p.counters[band], 1u);
                s_last = prev == (unsigned)(p.splits - 1);
            }
            __syncthreads();
            band_done = s_last;
            if (band_done) {
                const int r_base = band * BAND_ROWS;
                const int rows = min(BAND_ROWS, p.m_pad - r_base);
                for (int e = tid; e < rows * p.B; e += THREADS) {
                    const int b = e / rows, row = r_base + (e - b * rows);
                    double D = 0.0;
                    for (int s = 0; s < p.splits; ++s)  // fixed order
                        D += __ldcg(p.partials + ((size_t)s * p.B + b) * p.m_pad + row);
                    p.z[(size_t)b * p.m_pad + row] = FIN ? (float)(D * (double)p.ws) : finish_z(p, b, D);
                }
                if (tid == 0) p.counters[band] = 0u;
            }
        }
        // 5. output blocks: the band whose z completes a Hadamard block of m
        // queues that block's transform for the end of this CTA's tasks
        if (p.fuse_out && band_done) {
            __syncthreads();  // the band's z is written
            if (tid == 0) {
                __threadfence();
                const int r0 = band * BAND_ROWS, r1 = min(r0 + BAND_ROWS, p.m);
                for (int bi = 0; bi < p.nblk_m; ++bi) {
                    const int o = p.blk_off_m[bi], N = p.blk_len_m[bi];
                    if (r0 < o + N && o < r1) {
                        const unsigned prev = atom_add_acq_rel_gpu(&p.blk_cnt[bi], 1u);
                        if (prev == (unsigned)(p.blk_bands[bi] - 1)) {
                            s_pending[s_npending++] = bi;
                            p.blk_cnt[bi] = 0u;
                        }
                    }
                }
            }
        }
        __syncthreads();  // s_last and the shared activations are reused by the next task
    }
    if (p.fuse_out) {
        __syncthreads();
        const int np = s_npending;
        // the table is no longer needed: its shared memory holds the block
        for (int i = 0; i < np; ++i) {
            fused_output<THREADS>(p, s_pending[i], reinterpret_cast<float *>(smem_u4));
            __syncthreads();
        }
    }
}

template <int BPW, int NT, bool FIN, int WARPS = gemv_warps(NT, BPW)>
cudaError_t launch_t(const GemvParams &p, int grid, cudaStream_t s, bool pdl) {
    const size_t smem = gemv_launch_smem_bytes(p, BPW, FIN, WARPS);
    // raised once per device to the largest the library launches with (never
    // lowered: captured graphs replay against the attribute value at replay time)
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = once_per_device(configured, [] {
        return cudaFuncSetAttribute(gemv_kernel<BPW, NT, FIN, WARPS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)GEMV_SMEM_LIMIT);
    });
    if (e != cudaSuccess) return e;
    if (smem > GEMV_SMEM_LIMIT) return cudaErrorInvalidValue;
    if (p.fuse_out) {  // the output block is transformed in the table's shared memory
        for (int bi = 0; bi < p.nblk_m; ++bi)
            if ((size_t)p.B * p.blk_len_m[bi] * sizeof(float) > smem) return cudaErrorInvalidValue;
    }
    GemvParams q = p;
    void *args[] = {&q};
    if (p.clu > 1) {
        if (grid != p.bands * p.splits || p.clu != p.splits) return cudaErrorInvalidValue;
        static std::atomic<uint64_t> nonportable{0};  // clusters above 8 CTAs
        e = once_per_device(nonportable, [] {
            return cudaFuncSetAttribute(gemv_kernel<BPW, NT, FIN, WARPS>,
                                        cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        });
        if (e != cudaSuccess) return e;
        return launch_ex((const void *)gemv_kernel<BPW, NT, FIN, WARPS>, dim3(grid), dim3(WARPS * 32), smem, s,
                         pdl, args, p.clu);
    }
    return launch_ex((const void *)gemv_kernel<BPW, NT, FIN, WARPS>, dim3(grid), dim3(WARPS * 32), smem, s,
                     pdl, args);
}

// Largest number of clusters of `csize` CTAs of this kernel that can be
// resident at once (0 if the cluster does not fit).
template <int BPW, int NT, bool FIN, int WARPS = gemv_warps(NT, BPW)>
int max_clusters_t(int csize, size_t smem) {
    const void *fn = (const void *)gemv_kernel<BPW, NT, FIN, WARPS>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMV_SMEM_LIMIT) != cudaSuccess ||
        cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

}  // namespace

// Split of the chunk range so that (bands x splits) tasks spread over the
// persistent grid with the least makespan (in chunks per CTA), with a
// charge per task for the band reduction (`charge` chunks when split).
GemvPlan plan_gemv(int RT, int KC, int num_sms, int warps, bool pow2, int max_cps, int max_splits, double charge) {
    GemvPlan pl{};
    pl.bands = (RT + warps - 1) / warps;
    int best_cps = 0;
    double best = 1e30;
    // candidate chunk counts per split: every count that populates all its
    // splits, or the powers of two (the last split may be short)
    for (int cps = 1; cps <= (pow2 ? 2 * KC : KC); cps = pow2 ? 2 * cps : cps + 1) {
        const int s = (KC + cps - 1) / cps;
        if (!pow2 && (KC + s - 1) / s != cps) continue;
        if (cps > max_cps || s > max_splits) continue;
        const long long tasks = (long long)pl.bands * s;
        const long long waves = (tasks + num_sms - 1) / num_sms;
        const int work = cps < KC ? cps : KC;
        const double cost = (double)waves * (work + (s > 1 ? charge : 0.0)) + 0.02 * s;
        if (cost < best) {
            best = cost;
            best_cps = cps;
        }
        if (s == 1) break;
    }
    if (best_cps == 0) {  // nothing within the bounds: the fewest splits the bound allows
        best_cps = 1;
        while ((KC + best_cps - 1) / best_cps > max_splits) best_cps = pow2 ? 2 * best_cps : best_cps + 1;
    }
    pl.cps = best_cps;
    pl.splits = (KC + best_cps - 1) / best_cps;
    const long long tasks = (long long)pl.bands * pl.splits;
    pl.grid = (int)(tasks < num_sms ? tasks : num_sms);
    return pl;
}

size_t gemv_smem_bytes(int table_words, int bpw) {
    return (size_t)table_words * 4 + (stage8(bpw) ? 256 * 16 : 0);
}

size_t gemv_launch_smem_bytes(const GemvParams &p, int bpw, bool fin, int warps) {
    const size_t base = fin ? gemv_fused_smem_bytes(p.table_words, bpw, p.B, std::min(p.cps, p.KC) * GLQ_CHUNK_K)
                            : gemv_smem_bytes(p.table_words, bpw);
    return p.clu ? std::max(base, p.spart_off + gemv_cluster_partials_bytes(warps, p.B)) : base;
}

size_t gemv_cluster_partials_bytes(int warps, int B) {
    // splits x ceil(rows x B / splits) slots, splits <= 16
    return ((size_t)warps * GLQ_ROW_TILE * B + 16) * sizeof(double);
}

// The kernel variant of (BPW, token tiles, fused input, warps) the launcher
// selects, and its resident-cluster count.
template <int BPW>
int max_clusters_sel(int nt, bool fin, int warps, int csize, size_t smem) {
    if (fin) return nt == 1 ? max_clusters_t<BPW, 1, true>(csize, smem) : max_clusters_t<BPW, 2, true>(csize, smem);
    if (BPW <= 4 && nt == 1 && warps == GEMV_WIDE_WARPS)
        return max_clusters_t<BPW, 1, false, (BPW <= 4 ? GEMV_WIDE_WARPS : gemv_warps(1, BPW))>(csize, smem);
    return nt == 1 ? max_clusters_t<BPW, 1, false>(csize, smem) : max_clusters_t<BPW, 2, false>(csize, smem);
}

int gemv_max_clusters(int bpw, int nt, bool fin, int warps, int csize, size_t smem) {
    // memoised per device, kernel, cluster size and shared-memory size
    // (host-side, under a lock: layers may be created from several threads)
    struct Key {
        int dev, bpw, nt, fin, warps, csize;
        size_t smem;
        int n;
    };
    static Key cache[64];
    static int ncache = 0;
    static std::mutex lock;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> guard(lock);
    for (int i = 0; i < ncache; ++i) {
        const Key &k = cache[i];
        if (k.dev == dev && k.bpw == bpw && k.nt == nt && k.fin == (int)fin && k.warps == warps &&
            k.csize == csize && k.smem == smem)
            return k.n;
    }
    int n = 0;
    switch (bpw) {
        case 2: n = max_clusters_sel<2>(nt, fin, warps, csize, smem); break;
        case 3: n = max_clusters_sel<3>(nt, fin, warps, csize, smem); break;
        case 4: n = max_clusters_sel<4>(nt, fin, warps, csize, smem); break;
        case 5: n = max_clusters_sel<5>(nt, fin, warps, csize, smem); break;
        case 6: n = max_clusters_sel<6>(nt, fin, warps, csize, smem); break;
        case 7: n = max_clusters_sel<7>(nt, fin, warps, csize, smem); break;
        case 8: n = max_clusters_sel<8>(nt, fin, warps, csize, smem); break;
        default: n = 0;
    }
    if (ncache < 64) cache[ncache++] = Key{dev, bpw, nt, (int)fin, warps, csize, smem, n};
    return n;
}

size_t gemv_fused_smem_bytes(int table_words, int bpw, int B, int klen) {
    // the table is a multiple of 4 words, so the activation area is 16-byte aligned
    return gemv_smem_bytes(table_words, bpw) + (size_t)B * klen * (2 + (stage8(bpw) ? 2 : 0) + 4);
}

template <int BPW, bool FIN>
cudaError_t launch_bpw(const GemvParams &p, int grid, cudaStream_t s, bool pdl) {
    const bool two = p.B > 8;
    if (BPW <= 4 && !FIN && !two && p.warps == GEMV_WIDE_WARPS)
        return launch_t<BPW, 1, false, (BPW <= 4 ? GEMV_WIDE_WARPS : gemv_warps(1, BPW))>(p, grid, s, pdl);
    if (p.warps != gemv_warps(two ? 2 : 1, BPW)) return cudaErrorInvalidValue;
    return two ? launch_t<BPW, 2, FIN>(p, grid, s, pdl) : launch_t<BPW, 1, FIN>(p, grid, s, pdl);
}

template <bool FIN>
cudaError_t launch_sel(const GemvParams &p, int bpw, int grid, cudaStream_t s, bool pdl) {
    switch (bpw) {
        case 2: return launch_bpw<2, FIN>(p, grid, s, pdl);
        case 3: return launch_bpw<3, FIN>(p, grid, s, pdl);
        case 4: return launch_bpw<4, FIN>(p, grid, s, pdl);
        case 5: return launch_bpw<5, FIN>(p, grid, s, pdl);
        case 6: return launch_bpw<6, FIN>(p, grid, s, pdl);
        case 7: return launch_bpw<7, FIN>(p, grid, s, pdl);
        case 8: return launch_bpw<8, FIN>(p, grid, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemv(const GemvParams &p, int bpw, int grid, cudaStream_t s, bool pdl, bool fused_in) {
    return fused_in ? launch_sel<true>(p, bpw, grid, s, pdl) : launch_sel<false>(p, bpw, grid, s, pdl);
}

}  // namespace glq
