// glq_rht_rows.cu -- the input and output randomized Hadamard transforms,
// xr = H_n (S_in x) and y = S_out (H_m z), for rows of up to 16384 values: all
// of the tensor-core (many-token) path, the decode output stage, and the
// decode input stage when it is not fused into the GEMV.  H is block-diagonal
// over the binary decomposition of the size, each block a Sylvester-ordered
// FWHT normalised by 1/sqrt(block) (glq 0.5.1 PyPI page, "How it works" 2 and
// "Bit widths": block-diagonal FHT for sizes that are not powers of two;
// GLQ v0.3.2 release notes, input_rht / output_rht).
//
// Design (B200): throughput over many rows, bound by the per-value
// instruction count rather than by DRAM.  A persistent grid of CTAs
// transforms one row at a time per CTA, with the next row already streaming
// into a shared-memory staging buffer (16-byte asynchronous copies):
//   * a row of up to 2^L values (9 <= L <= 14) is held 16 values per thread;
//     the butterflies run in registers, four position bits per phase, and the
//     row changes layout between phases through shared memory (one store,
//     one barrier, one load per value and phase); no warp shuffles;
//   * the row sits in shared memory under the padded layout word(p) = p +
//     (p >> 5), which is additive over disjoint position bits, so every
//     access is a per-thread base plus an immediate offset; which position
//     bits the lanes of a warp own in each phase is chosen so that their
//     words fall in 32 distinct banks;
//   * the stages of a Hadamard transform commute, so the last phase carries
//     the lowest position bits along as "fill" and writes its values straight
//     to global memory in runs of consecutive columns;
//   * the output side alternates two row buffers, so that no barrier protects
//     a buffer from the next row; the input side keeps one (its row-max
//     reduction already separates rows), which at 2^14 values lets two
//     1024-thread CTAs share an SM;
//   * butterflies and the norm use the packed f32x2 add / subtract / multiply
//     of sm_100a (same IEEE rounding as scalar operations); signs are XOR
//     masks on packed 16-bit words where the data is 16-bit;
//   * Hadamard blocks of a size that is not a power of two are handled by
//     testing, per butterfly, whether both ends lie in one block; the block
//     norm 1/sqrt(block) is applied on load, where a thread's 16 values share
//     one block;
//   * the input direction also finds the row's max |xr| (one reduction) and
//     writes either the fp16 operand of the tensor-core GEMM, xr 2^e with
//     max |xr| 2^e < 2^14, or the decode GEMV's operand X = round(xr 2^e) as
//     high / low bytes with its exact row sum (a second reduction), plus 2^-e;
//     the decode operand needs 8 consecutive columns per thread, so that
//     variant returns the row to the load layout first and applies the norm
//     there, as one product with the power-of-two scale.
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
// the phase's own bits, filled up with the lowest position bits when fewer
// than four remain.  The 32 lanes of a warp give five further position bits
// and the warp index the rest, in increasing order.  The lane bits are chosen
// per phase so that their word offsets under word(p) = p + (p >> 5) are 1, 2,
// 4, 8 and 16 modulo 32 in some order: bits 0..4 weigh 2^b and bits 5..9 weigh
// 2^b + 2^(b-5), i.e. 2^(b-5) modulo 32.
//   phase 0 (bits 0..3):      lanes on bits 4..8 (16 consecutive values per
//                             thread: the layout of the global loads);
//   phase 1 (bits 4..7):      lanes on bits 0..3 and 9 (bit 8 when L = 9,
//                             which leaves one two-way bank conflict);
//   a full later phase:       lanes on bits 0..4;
//   a last phase with f fill bits 0..f-1: lanes on bits f..f+4.
// ---------------------------------------------------------------------------

__host__ __device__ constexpr uint32_t word_of(uint32_t p) { return p + (p >> 5); }

// shared-memory words of one row buffer (a multiple of 4: 16-byte aligned)
__host__ __device__ constexpr int row_words(int L) { return (1 << L) + (1 << (L - 5)); }

// position bits of phase q that are butterflied (the rest of the four are fill)
__host__ __device__ constexpr int phase_na(int L, int q) { return (L - 4 * q) < 4 ? (L - 4 * q) : 4; }

// position bit of register bit r (0..3) in phase q
__host__ __device__ constexpr int reg_bit(int L, int q, int r) {
    return r < phase_na(L, q) ? 4 * q + r : r - phase_na(L, q);
}

// position bits of register index j (0..15) in phase q
__host__ __device__ constexpr uint32_t jpos(int L, int q, int j) {
    uint32_t p = 0u;
    for (int r = 0; r < 4; ++r)
        if ((j >> r) & 1) p |= 1u << reg_bit(L, q, r);
    return p;
}

// position bit of lane bit i (0..4) in phase q
__host__ __device__ constexpr int lane_bit(int L, int q, int i) {
    if (q == 0) return 4 + i;
    if (q == 1) return i < 4 ? i : (L >= 10 ? 9 : 8);
    const int f = 4 - phase_na(L, q);
    return f + i;
}

__host__ __device__ constexpr bool is_reg_or_lane_bit(int L, int q, int b) {
    for (int r = 0; r < 4; ++r)
        if (reg_bit(L, q, r) == b) return true;
    for (int i = 0; i < 5; ++i)
        if (lane_bit(L, q, i) == b) return true;
    return false;
}

// position bit of thread-index bit s (0 .. L-5): lanes first, then the warp
// index on the remaining bits in increasing order
__host__ __device__ constexpr int thread_bit(int L, int q, int s) {
    if (s < 5) return lane_bit(L, q, s);
    int k = s - 5;
    for (int b = 0; b < L; ++b) {
        if (is_reg_or_lane_bit(L, q, b)) continue;
        if (k == 0) return b;
        --k;
    }
    return 0;
}

// The thread-index bits of phase q as runs that land on consecutive position
// bits: run i moves len[i] bits from src[i] to dst[i].  Built at compile
// time, so that tpos is one shift and mask per run.
struct TposRuns {
    int n;
    int src[10], dst[10], len[10];
};

__host__ __device__ constexpr TposRuns tpos_runs(int L, int q) {
    TposRuns r{};
    int s = 0;
    while (s < L - 4) {
        int n = 1;
        while (s + n < L - 4 && thread_bit(L, q, s + n) == thread_bit(L, q, s) + n) ++n;
        r.src[r.n] = s;
        r.dst[r.n] = thread_bit(L, q, s);
        r.len[r.n] = n;
        ++r.n;
        s += n;
    }
    return r;
}

// position bits given by thread index t (< 2^(L-4)) in phase q
template <int L, int Q>
__device__ __forceinline__ uint32_t tpos(uint32_t t) {
    constexpr TposRuns R = tpos_runs(L, Q);
    uint32_t p = 0u;
#pragma unroll
    for (int i = 0; i < 10; ++i)
        if (i < R.n) p |= ((t >> R.src[i]) & ((1u << R.len[i]) - 1u)) << R.dst[i];
    return p;
}

// a value the compiler must treat as new on every use, so that loop-invariant
// shared-memory addresses and masks are recomputed rather than kept live
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

// (a0, a1) *= s as one packed f32x2 multiply (IEEE rounding, as two scalar ones)
__device__ __forceinline__ void mul2(float &a0, float &a1, float s) {
    asm("{\n"
        " .reg .b64 A, S, D;\n"
        " mov.b64 A, {%0, %1};\n"
        " mov.b64 S, {%2, %2};\n"
        " mul.rn.f32x2 D, A, S;\n"
        " mov.b64 {%0, %1}, D;\n"
        "}\n"
        : "+f"(a0), "+f"(a1)
        : "f"(s));
}

// Sign bits of two 16-bit values packed in word u (0..7) of a thread, laid
// out as bit u (low half) and bit u + 16 (high half) of m: the XOR mask that
// flips those halves' sign bits.
__device__ __forceinline__ uint32_t half2_sign_mask(uint32_t m, int u) {
    return (m << (15 - u)) & 0x80008000u;
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
        // only the position bits above the span matter; for r >= 1 the
        // neighbours j and j + 1 differ in a bit below the span, so one test
        // covers a packed pair of butterflies
#pragma unroll
        for (int j = 0; j < VPT; j += 2)
            if ((X >> (4 * Q + 1)) != (jpos(L, Q, j) >> (4 * Q + 1))) {
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
                    if ((X >> (4 * Q + r + 1)) != (jpos(L, Q, j) >> (4 * Q + r + 1)))
                        bfly2(v[j], v[j + 1], v[k], v[k + 1]);
                }
    }
}

// Phase Q >= 1 (not the last): load the thread's 16 values of the phase
// from shared memory, apply its butterflies, store them back, then a CTA
// barrier.  Every thread reads and writes only its own 16 positions within a
// phase.
template <int L, int Q>
__device__ __forceinline__ void phase_pass(float v[VPT], float *srow, uint32_t base, uint32_t len, unsigned full) {
    const float *r = srow + opaque(base);
#pragma unroll
    for (int j = 0; j < VPT; ++j) v[j] = r[word_of(jpos(L, Q, j))];
    phase_stages<L, Q>(v, tpos<L, Q>(opaque(threadIdx.x)) ^ len, full);
    float *w = srow + opaque(base);
#pragma unroll
    for (int j = 0; j < VPT; ++j) w[word_of(jpos(L, Q, j))] = v[j];
    __syncthreads();
}

// R consecutive output values (R = 1, 2, 4, 8) of one run, converted and
// stored with one vector store per 16 bytes: DT 0 fp16, 1 bf16, 2 fp32.
// 16-bit pairs (R >= 2) get their sign bits flipped by half2_sign_mask(m,
// u0 + k) for word k; single values and fp32 arrive with their signs.
template <int R, int DT>
__device__ __forceinline__ void store_run(void *dst, const float *r, uint32_t m, int u0) {
    if constexpr (DT == 2) {
        float *d = static_cast<float *>(dst);
        if constexpr (R == 1) {
            d[0] = r[0];
        } else if constexpr (R == 2) {
            *reinterpret_cast<float2 *>(d) = make_float2(r[0], r[1]);
        } else {
#pragma unroll
            for (int k = 0; k < R; k += 4)
                *reinterpret_cast<float4 *>(d + k) = make_float4(r[k], r[k + 1], r[k + 2], r[k + 3]);
        }
    } else if constexpr (R == 1) {
        const uint16_t h = DT == 1 ? __bfloat16_as_ushort(__float2bfloat16_rn(r[0]))
                                      : __half_as_ushort(__float2half_rn(r[0]));
        *static_cast<uint16_t *>(dst) = h;
    } else {
        uint32_t w[R / 2];
#pragma unroll
        for (int k = 0; k < R / 2; ++k) {
            if constexpr (DT == 1) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(r[2 * k], r[2 * k + 1]);
                w[k] = *reinterpret_cast<const uint32_t *>(&h2);
            } else {
                const __half2 h2 = __floats2half2_rn(r[2 * k], r[2 * k + 1]);
                w[k] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            w[k] ^= half2_sign_mask(m, u0 + k);
        }
        if constexpr (R == 2) *static_cast<uint32_t *>(dst) = w[0];
        else if constexpr (R == 4) *static_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
        else *static_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
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
// DT: the output dtype of the output direction (0 fp16, 1 bf16, 2 fp32)
template <bool IN, bool XQ, int L, int DT>
__global__ void __launch_bounds__(1 << (L - 4), L >= 14 ? (IN && !XQ ? 2 : 0) : (1024 >> (L - 4))) rht_rows_kernel(RowsParams p, int B) {
    constexpr int NPH = (L + 3) / 4;  // phases of (up to) four position bits
    constexpr int QL = NPH - 1;       // the last phase
    constexpr int NAL = phase_na(L, QL), RUN = 1 << (4 - NAL);  // its butterflied bits; run of fill values
    constexpr int NCH = IN ? 2 : 4;   // 16-byte chunks of raw input per thread
    constexpr int WORDS = row_words(L);
    // Row buffers: the output direction alternates two, so that no barrier
    // protects a buffer from the next row; the input direction needs one,
    // since its max reduction already puts a barrier between the last
    // phase's loads and the next row's stores.
    constexpr int NBUF = IN ? 1 : 2;
    constexpr bool PACKED_OUT = !IN && DT != 2 && RUN >= 2;  // output signs on packed 16-bit words
    extern __shared__ __align__(16) float smem_rows[];  // [NBUF][WORDS] row buffers, then the staging slots
    const uint4 *stage = reinterpret_cast<const uint4 *>(smem_rows + NBUF * WORDS);
    __shared__ float s_red[2][32];  // per-warp row max, by row parity
    __shared__ int s_sum[2][32];    // per-warp sums of X, by row parity
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c0 = VPT * tid;  // first column of this thread in the load layout (phase 0)
    const uint32_t len = (uint32_t)p.len;
    const int valid = max(0, min(VPT, p.len - c0));  // 16, 8 (last block of 8) or 0
    pdl_launch_dependents();
    int b = blockIdx.x;
    if (b < B && c0 < p.len) {  // warm L2 and the TLB before waiting on the producer
        if (IN) prefetch_l2(static_cast<const uint16_t *>(p.x) + (size_t)b * p.len + c0);
        else prefetch_l2(p.z + (size_t)b * p.z_ld + c0);  // the first split
    }

    // row-independent data of this thread
    float norm = 0.f;  // of the block holding its 16 load-layout columns
    if (c0 < p.len) block_size_at(p, c0, &norm);
    // signs as XOR masks: input, S_in of the 16 load-layout columns per
    // packed word (word u = columns 2u, 2u + 1); output, S_out of the last
    // phase's 16 positions, per value (bit j) or per packed 16-bit word
    uint32_t smask = 0u;
    if (IN) {
        const uint32_t sb = valid ? (p.sign_bits[c0 >> 5] >> (c0 & 31)) & 0xFFFFu : 0u;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            smask |= ((sb >> (2 * u)) & 1u) << u | ((sb >> (2 * u + 1)) & 1u) << (u + 16);
    } else {
        const uint32_t tl = tpos<L, QL>((uint32_t)tid);
        uint32_t sbj = 0u;
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const uint32_t pj = tl | jpos(L, QL, j);
            if (pj < len) sbj |= ((p.sign_bits[pj >> 5] >> (pj & 31)) & 1u) << j;
        }
        if (PACKED_OUT) {
#pragma unroll
            for (int j0 = 0; j0 < (1 << NAL); ++j0)
#pragma unroll
                for (int w = 0; w < RUN / 2; ++w) {
                    const int u = j0 * (RUN / 2) + w;
                    smask |= ((sbj >> (j0 + ((2 * w) << NAL))) & 1u) << u |
                             ((sbj >> (j0 + ((2 * w + 1) << NAL))) & 1u) << (u + 16);
                }
        } else {
            smask = sbj;
        }
    }
    uint32_t base[NPH];  // word of the thread's position bits, per phase
    unsigned full = 0u;  // per phase: every butterfly of the thread lies within one block
    {
        uint32_t tp[NPH];
        tp[0] = tpos<L, 0>((uint32_t)tid);
        if (NPH > 1) tp[NPH > 1 ? 1 : 0] = tpos<L, (NPH > 1 ? 1 : 0)>((uint32_t)tid);
        if (NPH > 2) tp[NPH > 2 ? 2 : 0] = tpos<L, (NPH > 2 ? 2 : 0)>((uint32_t)tid);
        if (NPH > 3) tp[NPH > 3 ? 3 : 0] = tpos<L, (NPH > 3 ? 3 : 0)>((uint32_t)tid);
#pragma unroll
        for (int q = 0; q < NPH; ++q) {
            base[q] = word_of(tp[q]);
            const int top = (4 * q + 4 < L ? 4 * q + 4 : L);  // one past the phase's highest bit
            if (((tp[q] ^ len) >> top) != 0u) full |= 1u << q;
        }
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
        float *srow = smem_rows + (NBUF == 2 ? par * WORDS : 0);
        cp_async_wait_all();
        uint4 raw[NCH];
#pragma unroll
        for (int c = 0; c < NCH; ++c) raw[c] = stage[slot(c)];
        if (b + (int)gridDim.x < B) issue(b + gridDim.x);  // this thread's slots are free again
        // the block norm now (all but the decode operand, which scales once at the end)
        float v[VPT];
        if (IN) {
            const uint32_t sm = opaque(smask);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t ws = w[j] ^ half2_sign_mask(sm, 4 * q + j);  // S_in on the raw halves
                    if (p.x_bf16) {
                        v[8 * q + 2 * j] = __uint_as_float(ws << 16);
                        v[8 * q + 2 * j + 1] = __uint_as_float(ws & 0xFFFF0000u);
                    } else {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&ws));
                        v[8 * q + 2 * j] = f.x;
                        v[8 * q + 2 * j + 1] = f.y;
                    }
                }
            }
            if (!XQ) {
#pragma unroll
                for (int j = 0; j < VPT; j += 2) mul2(v[j], v[j + 1], norm);
            }
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
#pragma unroll
            for (int j = 0; j < VPT; j += 2) mul2(v[j], v[j + 1], norm);
        }

        // the butterflies, phase by phase (phase 0 on the values as loaded)
        phase_stages<L, 0>(v, opaque((uint32_t)c0) ^ len, full & 1u);
        {
            float *w = srow + opaque(base[0]);
#pragma unroll
            for (int j = 0; j < VPT; ++j) w[word_of(jpos(L, 0, j))] = v[j];
            __syncthreads();
        }
        if (NPH > 2) phase_pass<L, (NPH > 2 ? 1 : 0)>(v, srow, base[NPH > 2 ? 1 : 0], len, (full >> 1) & 1u);
        if (NPH > 3) phase_pass<L, (NPH > 3 ? 2 : 0)>(v, srow, base[NPH > 3 ? 2 : 0], len, (full >> 2) & 1u);
        {  // the last phase
            const float *r = srow + opaque(base[QL]);
#pragma unroll
            for (int j = 0; j < VPT; ++j) v[j] = r[word_of(jpos(L, QL, j))];
            phase_stages<L, QL>(v, tpos<L, QL>(opaque(threadIdx.x)) ^ len, (full >> QL) & 1u);
        }

        if (XQ) {
            // back to the load layout (8 consecutive columns per group), then
            // X = round(xr 2^e) with the norm and the scale as one product
            {
                float *w = srow + opaque(base[QL]);
#pragma unroll
                for (int j = 0; j < VPT; ++j) w[word_of(jpos(L, QL, j))] = v[j];
                __syncthreads();
                const float *r = srow + opaque(base[0]);
#pragma unroll
                for (int j = 0; j < VPT; ++j) v[j] = r[word_of(jpos(L, 0, j))];
            }
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) mx = fmaxf(mx, fabsf(v[j]));
            mx *= norm;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) s_red[par][warp] = mx;
            __syncthreads();
            float rowmax = lane < (int)(blockDim.x >> 5) ? s_red[par][lane] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) rowmax = fmaxf(rowmax, __shfl_xor_sync(0xffffffffu, rowmax, o));
            float scale = 1.f;
            if (rowmax > 0.f && isfinite(rowmax)) {
                int e;
                frexpf(rowmax, &e);  // rowmax < 2^e
                scale = ldexpf(1.f, min(14 - e, 126));  // scale and 1 / scale normal for the tiniest rows
            }
            const float f = norm * scale;  // scale is a power of two: one rounding, as xr 2^e
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
            continue;
        }

        // the last phase's values, straight to global memory: runs of RUN
        // consecutive columns (the fill bits), one run per real register index
        const uint32_t tl = tpos<L, QL>(opaque(threadIdx.x));
        if (IN) {  // fp16 xr 2^e; padding columns [len, len_pad) hold zeros
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) mx = fmaxf(mx, fabsf(v[j]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) s_red[par][warp] = mx;
            __syncthreads();
            float rowmax = lane < (int)(blockDim.x >> 5) ? s_red[par][lane] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) rowmax = fmaxf(rowmax, __shfl_xor_sync(0xffffffffu, rowmax, o));
            float scale = 1.f;
            if (rowmax > 0.f && isfinite(rowmax)) {
                int e;
                frexpf(rowmax, &e);  // rowmax < 2^e
                scale = ldexpf(1.f, min(14 - e, 126));  // scale and 1 / scale normal for the tiniest rows
            }
            __half *xrow = p.xh + (size_t)b * p.len_pad;
#pragma unroll
            for (int j0 = 0; j0 < (1 << NAL); ++j0) {
                const uint32_t pj = tl | jpos(L, QL, j0);
                if (pj < (uint32_t)p.len_pad) {
                    float r[RUN];
#pragma unroll
                    for (int k = 0; k < RUN; ++k) r[k] = v[j0 + (k << NAL)] * scale;  // exact: a power of two
                    store_run<RUN, 0>(xrow + pj, r, 0u, 0);
                }
            }
            if (tid == 0) p.info[b] = glq_rowinfo{0, 1.f / scale, 0.f};
        } else {
            const uint32_t sm = opaque(smask);
            constexpr size_t esz = DT == 2 ? 4 : 2;
            char *yrow = static_cast<char *>(p.y) + (size_t)b * p.len * esz;
#pragma unroll
            for (int j0 = 0; j0 < (1 << NAL); ++j0) {
                const uint32_t pj = tl | jpos(L, QL, j0);
                if (pj < len) {
                    float r[RUN];
#pragma unroll
                    for (int k = 0; k < RUN; ++k)
                        r[k] = PACKED_OUT ? v[j0 + (k << NAL)] : flip(v[j0 + (k << NAL)], sm, j0 + (k << NAL));
                    store_run<RUN, DT>(yrow + pj * esz, r, PACKED_OUT ? sm : 0u, j0 * (RUN / 2));
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

template <bool IN, bool XQ, int L, int DT>
cudaError_t launch_rows_t(const RowsParams &p, int B, cudaStream_t s, bool pdl) {
    const void *fn = (const void *)rht_rows_kernel<IN, XQ, L, DT>;
    const int threads = 1 << (L - 4);
    // the row buffers (two on the output side) and the staging buffer of the
    // next row's raw input
    const size_t smem = (IN ? 1 : 2) * sizeof(float) * (size_t)row_words(L) + (size_t)threads * (IN ? 32 : 64);
    static std::atomic<uint64_t> configured{0};  // devices set
    cudaError_t e = once_per_device(configured, [fn, smem] {
        return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    // persistent grid: every CTA that fits on the device at once, at most one
    // per row (SM count and occupancy queried once per device, not per call)
    constexpr int MAX_DEV = 64;
    static int sms_of[MAX_DEV] = {}, per_sm_of[MAX_DEV] = {};
    int dev = 0;
    e = cudaGetDevice(&dev);
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
template <bool IN, bool XQ, int DT>
cudaError_t launch_rows_sel(const RowsParams &p, int B, cudaStream_t s, bool pdl) {
    const int cover = IN ? p.len_pad : p.len;
    switch (rows_log2(cover)) {
        case 9: return launch_rows_t<IN, XQ, 9, DT>(p, B, s, pdl);
        case 10: return launch_rows_t<IN, XQ, 10, DT>(p, B, s, pdl);
        case 11: return launch_rows_t<IN, XQ, 11, DT>(p, B, s, pdl);
        case 12: return launch_rows_t<IN, XQ, 12, DT>(p, B, s, pdl);
        case 13: return launch_rows_t<IN, XQ, 13, DT>(p, B, s, pdl);
        case 14: return launch_rows_t<IN, XQ, 14, DT>(p, B, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_rht_rows(const RowsParams &p, bool input, int B, cudaStream_t s, bool pdl) {
    if (B <= 0) return cudaErrorInvalidValue;
    if (!input) {
        switch (p.y_dtype) {
            case 0: return launch_rows_sel<false, false, 0>(p, B, s, pdl);
            case 1: return launch_rows_sel<false, false, 1>(p, B, s, pdl);
            case 2: return launch_rows_sel<false, false, 2>(p, B, s, pdl);
            default: return cudaErrorInvalidValue;
        }
    }
    if (p.xq) return launch_rows_sel<true, true, 0>(p, B, s, pdl);
    if (!p.butterfly && rht_in_mma_supported(p)) return launch_rht_in_mma(p, B, s, pdl);
    return launch_rows_sel<true, false, 0>(p, B, s, pdl);
}

}  // namespace glq
