// glq_rht_mma.cu -- the input randomized Hadamard transform of the
// tensor-core (many-token) path on the tensor pipe: xr = H_n (S_in x) for
// rows of 512 .. 16384 values whose length is a multiple of 256, written as
// the fp16 operand of the prefill GEMM, xr 2^e, with 2^-e per row.  H is
// block-diagonal over the binary decomposition of n, each block a
// Sylvester-ordered Hadamard normalised by 1/sqrt(block) (glq 0.5.1 PyPI
// page, "How it works" 2 and "Bit widths"; GLQ v0.3.2 release notes,
// input_rht).
//
// Design (B200).  The butterfly kernel for these rows is bound by shared
// memory traffic (each of its three layout changes moves 8 bytes per value).
// Here the Hadamard is applied as 16 x 16 matrices on the warp tensor cores,
// four position bits per product, so that a row crosses shared memory once
// between its two halves:
//   * a row of 2^L positions is cut into tiles of 256 (16 x 16); the Hadamard
//     over a tile's bits 4-7 is one m16n8k16 product pair with the data as
//     the B operand (loaded by ldmatrix.trans from 16-byte units of 8
//     consecutive positions), and its fp32 result, rounded to fp16, is
//     already the A operand of the product over bits 0-3 (no data movement);
//   * rows of 2^13 and 2^14 positions add one or two fp32 butterflies
//     between the 4 tiles a warp holds (position bits 8, 9);
//   * the tile is stored (stmatrix) into a row buffer and read back
//     (ldmatrix.trans) along the remaining (up to four) position bits, whose
//     Hadamard is one more product pair with the data as the B operand;
//   * the results go through an output buffer to 16-byte coalesced stores;
//   * every buffer is addressed in 16-byte units under an XOR swizzle of
//     position bits into the bank-group bits, chosen so that each 8-lane
//     phase of every ldmatrix / stmatrix and of the copies meets 8 distinct
//     bank groups;
//   * the matrices carry +-2^-k (exact in fp16 and bf16); what the block
//     norm still needs (a power of sqrt2: the cross butterflies are
//     unnormalised, a product over an odd count of active bits carries
//     2^-ceil(a/2)) is an fp32 multiply before the next rounding to fp16;
//   * the prescale 2^e comes from the row's max |x| (max |x| 2^e in
//     [2^7, 2^8)), so that every intermediate, bounded by ||x||_2 2^e <=
//     2^7 max |x| 2^e, stays below 2^15; the first product runs on the raw
//     16-bit inputs (bf16 or fp16 kind), with the scale inside its matrix
//     for bf16 (2^(e-2), so that its fp32 result cannot overflow) and
//     applied to its fp32 result for fp16;
//   * values are rounded to fp16 three times (after the first product,
//     after the second product and the cross butterflies, and after the
//     last product) instead of the butterfly kernel's once;
//   * a persistent CTA of up to 16 warps works on three rows at once as a
//     software pipeline (stage A of one row, stage B of the previous one, the
//     copy-out of the one before: independent work between two barriers,
//     with row and output buffers alternating by row parity), one CTA
//     barrier per row; the next rows' raw inputs stream into a ring of three
//     staging buffers (16-byte asynchronous copies); below 2^14 positions
//     CTAs of at most 8 warps, two or more per SM.
#include <algorithm>

#include "glq_kernels.cuh"

namespace glq {

namespace {

// ---------------------------------------------------------------------------
// Plan of a row of 2^L positions (9 <= L <= 14).
//   stage A: bits 0-7 of each 256-position tile (two products), plus C =
//            max(0, L - 12) cross-tile bits 8 .. 8 + C - 1 (fp32 butterflies
//            between the 2^C tiles of a warp);
//   stage B: the remaining bits 8 + C .. L - 1 (1 to 4 of them) as the k bits
//            of one product, filled up to four with already transformed bits
//            7, 6, 5, 4 (identity there);
//   warps:   2^(L-8) / T, each taking T tiles per stage: 4 from L = 13 (16
//            warps, one CTA per SM at L = 14; 8 warps, two CTAs per SM at
//            L = 13), else 2 (2^(L-9) warps, two or more CTAs per SM).
//            Measured at L = 14 (B200, 2048 rows of 14336): 32 warps of 2
//            tiles (the cross bits split between the stages) executed 1.5x
//            the instructions; 8 warps of 8 tiles (241 registers) executed
//            26 % fewer but, with 8 warps on the SM, issued in 41 % of the
//            cycles instead of 59 % and took longer (44.4 against 42.8 us).
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int mma_cross(int L) { return L > 12 ? L - 12 : 0; }
__host__ __device__ constexpr int mma_tpw(int L) { return L >= 13 ? 4 : 2; }
__host__ __device__ constexpr int mma_warps(int L) { return (1 << (L - 8)) / mma_tpw(L); }
// CTAs per SM the launch bounds ask for (registers): one 16-warp CTA at
// 2^14 positions, else at least two
__host__ __device__ constexpr int mma_min_ctas(int L) { return L >= 14 ? 1 : 2; }
__host__ __device__ constexpr int mma_real_b(int L) { return L - 8 - mma_cross(L); }

// position bit of stage-B k bit i (0..3)
__host__ __device__ constexpr int kb_bit(int L, int i) {
    return i < mma_real_b(L) ? 8 + mma_cross(L) + i : 7 - (i - mma_real_b(L));
}

// position bit of stage-B tile-index bit j: the bits 4 .. L-1 that are not k
// bits, in increasing order
__host__ __device__ constexpr int tileb_bit(int L, int j) {
    int k = 0;
    for (int b = 4; b < L; ++b) {
        bool is_k = false;
        for (int i = 0; i < 4; ++i)
            if (kb_bit(L, i) == b) is_k = true;
        if (is_k) continue;
        if (k == j) return b;
        ++k;
    }
    return 0;
}

// positions of stage-B k index k (0..15) and of stage-B tile index tb
__host__ __device__ constexpr uint32_t kb_pos(int L, int k) {
    uint32_t p = 0u;
    for (int i = 0; i < 4; ++i)
        if ((k >> i) & 1) p |= 1u << kb_bit(L, i);
    return p;
}
__host__ __device__ constexpr uint32_t tileb_pos(int L, int tb) {
    uint32_t p = 0u;
    for (int j = 0; j < L - 8; ++j)
        if ((tb >> j) & 1) p |= 1u << tileb_bit(L, j);
    return p;
}

// Slots (16-byte units) of position p in the three buffers.  The unit of p
// is p >> 3; its bank group is the unit's low three bits (position bits
// 3-5), into which higher position bits are XORed:
//   staging S:   bit 6 -> group bit 0        (stage-A loads vary bits 4-6,
//                                              the copies bits 3-5);
//   row buffer R: bit 6 -> group bit 0, k bits 0,1,2 of stage B -> group
//                bits 2,1,0 (one term dropped when that k bit is bit 6)
//                                             (stage-A stores vary bits 4-6,
//                                              stage-B loads the k bits 0-2);
//   output O:    k bits 0,1,2 -> group bits 2,1,0 (stage-B stores vary the k
//                                              bits 0-2, the copy-out bits 3-5).
// All three are linear over GF(2): slot(p ^ q) = slot(p) ^ slot(q).
__host__ __device__ constexpr uint32_t slot_s(uint32_t p) { return (p >> 3) ^ ((p >> 6) & 1u); }
__host__ __device__ constexpr uint32_t slot_r(int L, uint32_t p) {
    uint32_t f = (p >> 6) & 1u;
    for (int i = 0; i < 3; ++i)
        if (kb_bit(L, i) != 6) f ^= ((p >> kb_bit(L, i)) & 1u) << (2 - i);
    return (p >> 3) ^ f;
}
__host__ __device__ constexpr uint32_t slot_o(int L, uint32_t p) {
    uint32_t f = 0u;
    for (int i = 0; i < 3; ++i) f ^= ((p >> kb_bit(L, i)) & 1u) << (2 - i);
    return (p >> 3) ^ f;
}

// the butterfly on bit b between p (bit b clear) and p + 2^b lies within one
// Hadamard block of a row of len (blocks: aligned powers of two, descending)
__host__ __device__ constexpr bool bfly_active(uint32_t p, int b, uint32_t len) {
    return p < len && ((p ^ len) >> (b + 1)) != 0u;
}

// S_in of a warp's stage-A fragments, one bit per 16-bit value: register q
// of the warp's tile i at bit 4 (i & 3) + q (low half) or 16 + 4 (i & 3) + q
// (high half) of word i >> 2; sign_xor gives the mask that flips register q
// of tile i (the fp16 / bf16 sign bits 15 and 31)
__host__ __device__ constexpr int mma_sign_words(int L) { return (mma_tpw(L) + 3) / 4; }
__host__ __device__ constexpr int sign_bit_of(int i, int q, int h) { return 16 * h + 4 * (i & 3) + q; }
__host__ __device__ constexpr uint32_t sign_xor(uint32_t w, int i, int q) {
    return (w << (15 - (4 * (i & 3) + q))) & 0x80008000u;
}

// ---------------------------------------------------------------------------
// warp-level matrix instructions
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
}
// d = A B (zero accumulator); A 16 x 16 row-major fragment, B 16 x 8 column
// fragment; BF16: both operands bf16, else both fp16
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    const float z = 0.f;
    if constexpr (BF16) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%10, %10, %10, %10};\n"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
    } else {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%10, %10, %10, %10};\n"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
    }
}
// two fp32 values rounded to fp16 and packed (lo in the low half)
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__host__ __device__ inline int popc32(uint32_t v) {
#ifdef __CUDA_ARCH__
    return __popc(v);
#else
    return __builtin_popcount(v);
#endif
}

// Lane addressing of the x4 matrix loads and stores: lane l gives the row
// address of row l & 7 of matrix l >> 3.
//   stage A (tiles of bits 0-7): matrix bit 0 -> position bit 7, matrix bit
//     1 -> bit 3 (the second n-tile), row -> bits 4-6;
//   stage B: matrix bit 0 -> k bit 3, matrix bit 1 -> bit 3, row -> k bits 0-2.
__host__ __device__ constexpr uint32_t offa_of(int lane) {
    return ((uint32_t)(lane & 7) << 4) | ((uint32_t)((lane >> 3) & 1) << 7) | ((uint32_t)(lane >> 4) << 3);
}
__host__ __device__ constexpr uint32_t offb_of(int L, int lane) {
    return kb_pos(L, (lane & 7) + 8 * ((lane >> 3) & 1)) | ((uint32_t)(lane >> 4) << 3);
}
// position of half h of register q of lane l after the stage-A load
// (ldmatrix.trans: row 2t + h of matrix q, element gq) in the tile at base
__host__ __device__ constexpr uint32_t frag_pos(uint32_t base, int lane, int q, int h) {
    return base + offa_of(8 * q + 2 * (lane & 3) + h) + (uint32_t)(lane >> 2);
}

__device__ __forceinline__ void cp_async16_mma(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_mma() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_mma() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// the stage-B matrix entry (row j, col k) as fp16 bits, and its row's
// remaining norm factor: the butterflies on the real stage-B bits that are
// active for row j's block, scaled by 2^-ceil(a/2) for a active bits
template <int L>
__host__ __device__ inline uint32_t mb_active(int j, uint32_t len) {
    const uint32_t pj = kb_pos(L, j);
    uint32_t am = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (i < mma_real_b(L) && bfly_active(pj & ~(1u << kb_bit(L, i)), kb_bit(L, i), len)) am |= 1u << i;
    return am;
}
__host__ __device__ inline uint32_t mag_of_count(int a) {
    return a == 0 ? 0x3C00u : (a <= 2 ? 0x3800u : 0x3400u);  // 1, 1/2, 1/4 in fp16
}
template <int L>
__host__ __device__ inline uint32_t mb_half(int j, int k, uint32_t len) {
    const uint32_t am = mb_active<L>(j, len);
    if (((uint32_t)(j ^ k) & ~am) & 15u) return 0u;
    return mag_of_count(popc32(am)) | ((uint32_t)(popc32((uint32_t)(j & k) & am) & 1) << 15);
}
// remaining norm factor of stage-B row j: its product carries 2^-ceil(a/2)
// for a active bits, the block norm asks 2^(-a/2): sqrt2 for an odd a
template <int L>
__host__ __device__ inline float stageb_norm(int j, uint32_t len) {
    return (popc32(mb_active<L>(j, len)) & 1) ? 1.41421356237309515f : 1.f;
}
// remaining norm factor of the cross bits of the stage-A tile at base
template <int L>
__host__ __device__ inline float cross_norm(uint32_t base, uint32_t len) {
    int cact = 0;
    for (int cb = 0; cb < mma_cross(L); ++cb)
        if (bfly_active(base & ~(1u << (8 + cb)), 8 + cb, len)) ++cact;
    return cact == 0 ? 1.f : (cact == 1 ? 0.707106781186547524f : 0.5f);
}

// Fragments of a 16 x 16 matrix of 16-bit entries e(j, k) (row j, col k)
// in the m16n8k16 register layouts, lane l = 4 gq + t:
//   A (row-major): words (gq, 2t | 2t+1), (gq+8, 2t | 2t+1), (gq, 2t+8 | 2t+9),
//                  (gq+8, 2t+8 | 2t+9);
//   B (column n-tile nt): words (2t | 2t+1, gq + 8 nt), (2t+8 | 2t+9, gq + 8 nt);
// the first entry of each pair in the low half.
template <class E>
__host__ __device__ inline void a_frag(int lane, const E &e, uint32_t (&a)[4]) {
    const int gq = lane >> 2, t = lane & 3;
    a[0] = e(gq, 2 * t) | e(gq, 2 * t + 1) << 16;
    a[1] = e(gq + 8, 2 * t) | e(gq + 8, 2 * t + 1) << 16;
    a[2] = e(gq, 2 * t + 8) | e(gq, 2 * t + 9) << 16;
    a[3] = e(gq + 8, 2 * t + 8) | e(gq + 8, 2 * t + 9) << 16;
}
template <class E>
__host__ __device__ inline void b_frag(int lane, int nt, const E &e, uint32_t (&b)[2]) {
    const int gq = lane >> 2, t = lane & 3;
    b[0] = e(2 * t, gq + 8 * nt) | e(2 * t + 1, gq + 8 * nt) << 16;
    b[1] = e(2 * t + 8, gq + 8 * nt) | e(2 * t + 9, gq + 8 * nt) << 16;
}
// H16 scaled by a power of two: entry mag (16-bit bits) with the sign
// (-1)^popcount(j & k)
struct Had16 {
    uint32_t mag;
    __host__ __device__ uint32_t operator()(int j, int k) const {
        return mag | ((uint32_t)(popc32((uint32_t)(j & k)) & 1) << 15);
    }
};
// the stage-B matrix of a row of len
template <int L>
struct StageB {
    uint32_t len;
    __host__ __device__ uint32_t operator()(int j, int k) const { return mb_half<L>(j, k, len); }
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ void sts128_zero(uint32_t addr) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(addr), "r"(0u) : "memory");
}

// The kernel's per-unit and per-tile slot constants, evaluated at compile
// time (the swizzles are linear: a thread's or a warp's slot XOR these):
//   s_k, o_k: staging / output slot of unit k T (the thread's k-th unit);
//   ra_i:     row-buffer slot of the warp's stage-A tile i;
//   rb_i, ob_i: row-buffer / output slot of the warp's stage-B tile i.
template <int L>
struct MmaTables {
    uint32_t s_k[mma_tpw(L)], o_k[mma_tpw(L)], ra_i[mma_tpw(L)], rb_i[mma_tpw(L)], ob_i[mma_tpw(L)];
};
template <int L>
__host__ __device__ constexpr MmaTables<L> mma_tables() {
    MmaTables<L> t{};
    constexpr int T = 32 * mma_warps(L);
    for (int k = 0; k < mma_tpw(L); ++k) {
        t.s_k[k] = slot_s((uint32_t)(k * T) << 3);
        t.o_k[k] = slot_o(L, (uint32_t)(k * T) << 3);
        t.ra_i[k] = slot_r(L, (uint32_t)k << 8);
        t.rb_i[k] = slot_r(L, tileb_pos(L, k));
        t.ob_i[k] = slot_o(L, tileb_pos(L, k));
    }
    return t;
}

constexpr int MMA_NS = 3;  // staging ring: a CTA's rows j, j + 1, j + 2 in flight

// shared memory of one CTA: the staging ring, two row buffers, two output
// buffers (224 KB at 2^14 positions)
__host__ __device__ constexpr size_t mma_smem_bytes(int L) { return (size_t)(MMA_NS + 4) * ((size_t)2 << L); }

// butterflies (a, b) <- (a + b, a - b) and products on value pairs, as
// scalar fp32 operations (the packed f32x2 forms measured slower here: they
// tie the pairs to adjacent registers)
__device__ __forceinline__ void bfly_f2(float &a0, float &a1, float &b0, float &b1) {
    const float x0 = a0, x1 = a1;
    a0 = x0 + b0;
    a1 = x1 + b1;
    b0 = x0 - b0;
    b1 = x1 - b1;
}
__device__ __forceinline__ void mul_f2(float &a0, float &a1, float s0, float s1) {
    a0 *= s0;
    a1 *= s1;
}

// per 16-bit half, the larger magnitude of m and v (one native max; sign
// bits arbitrary; a NaN half of v is ignored, as fmaxf does)
template <bool BF16>
__device__ __forceinline__ uint32_t absmax2(uint32_t m, uint32_t v) {
    uint32_t d;
    if constexpr (BF16) asm("max.xorsign.abs.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(m), "r"(v));
    else asm("max.xorsign.abs.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(m), "r"(v));
    return d;
}

// The prescale exponent e of a row whose largest magnitude has the 16-bit
// bits h (bf16 or fp16, sign clear): with h < 2^E as a value, e = 8 - E, so
// that max |x| 2^e lies in [2^7, 2^8); 0 for a zero, infinite or NaN row;
// clamped to [-124, 126].  Integer operations on the bits: a normal value
// with biased exponent E_b is below 2^(E_b - bias + 1), a subnormal one
// m 2^(1 - bias - mbits) below 2^(bitlength(m) + 1 - bias - mbits).
template <bool BF16>
__host__ __device__ inline int prescale_exp(uint32_t h) {
    constexpr int MB = BF16 ? 7 : 10, BIAS = BF16 ? 127 : 15, EMAX = BF16 ? 255 : 31;
    const int eb = (int)(h >> MB);
    const uint32_t m = h & ((1u << MB) - 1u);
    if (h == 0u || eb == EMAX) return 0;
    int E;
    if (eb > 0) {
        E = eb - BIAS + 1;
    } else {
        int bl = 0;
        while ((m >> bl) != 0u) ++bl;  // bit length of the subnormal significand
        E = bl + 1 - BIAS - MB;
    }
    const int e = 8 - E;
    return e < -124 ? -124 : (e > 126 ? 126 : e);
}

// Persistent over rows: a CTA transforms rows blockIdx.x, blockIdx.x +
// gridDim.x, ...; the raw inputs of the next two rows stream into the
// staging ring meanwhile, and the rows go through a three-deep software
// pipeline with one CTA barrier per row.
template <int L, bool BF16>
__global__ void __launch_bounds__(32 * mma_warps(L), mma_min_ctas(L)) rht_in_mma_kernel(RowsParams p, int B) {
    constexpr int W = mma_warps(L), T = 32 * W, TPW = mma_tpw(L), C = mma_cross(L);
    constexpr uint32_t BUF = 2u << L;  // bytes of one row buffer (16-bit values)
    constexpr MmaTables<L> K = mma_tables<L>();
    // a row has TPW * T units of 8 positions: a thread copies units tid + k T, k < TPW
    extern __shared__ __align__(128) uint8_t smem_mma[];
    __shared__ uint32_t s_max[2][W];
    const uint32_t sb = (uint32_t)__cvta_generic_to_shared(smem_mma);
    const uint32_t R0 = sb + MMA_NS * BUF, O0 = R0 + 2 * BUF;  // two row buffers, two output buffers
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gq = lane >> 2;
    const uint32_t len = (uint32_t)p.len;
    const int units = p.len >> 3;
    pdl_launch_dependents();

    // ---- per-lane constants (the layer's, not the row's)
    // H16 as the A operand of the first product (the input's dtype; its
    // magnitude, set per row, carries the prescale for bf16 inputs), H16 / 4
    // as the B operand (fp16, two n-tiles) of the second; the stage-B matrix
    uint32_t a1s[4], b2[2][2], aB[4];
    a_frag(lane, Had16{0u}, a1s);  // signs only
    b_frag(lane, 0, Had16{0x3400u}, b2[0]);
    b_frag(lane, 1, Had16{0x3400u}, b2[1]);
    a_frag(lane, StageB<L>{len}, aB);
    // the stage-B rows' remaining norms
    const float corr0 = stageb_norm<L>(gq, len), corr1 = stageb_norm<L>(gq + 8, len);
    // this warp's stage-A tiles: their signs, slots and the cross bits'
    // remaining norm
    const uint32_t offA = offa_of(lane), offB = offb_of(L, lane);
    const uint32_t lS = slot_s(offA) * 16u, lRa = slot_r(L, offA);
    const uint32_t lRb = slot_r(L, offB), lOb = slot_o(L, offB);
    // (tile i of the warp: its slots are the warp's first tile's XOR a
    // constant, the swizzles being linear and the tile bits disjoint)
    // S_in of the warp's stage-A fragments (sign_bit_of)
    uint32_t sgn[mma_sign_words(L)] = {};
    float fA[TPW];
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
        const uint32_t base = (uint32_t)(warp * TPW + i) << 8;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t lo = frag_pos(base, lane, q, 0), hi = frag_pos(base, lane, q, 1);
            const uint32_t slo = lo < len ? (p.sign_bits[lo >> 5] >> (lo & 31)) & 1u : 0u;
            const uint32_t shi = hi < len ? (p.sign_bits[hi >> 5] >> (hi & 31)) & 1u : 0u;
            sgn[i >> 2] |= slo << sign_bit_of(i, q, 0) | shi << sign_bit_of(i, q, 1);
        }
        fA[i] = cross_norm<L>(base, len);
    }
    const uint32_t wA = slot_r(L, (uint32_t)(warp * TPW) << 8) ^ lRa;
    const uint32_t wB = slot_r(L, tileb_pos(L, warp * TPW)) ^ lRb;
    const uint32_t wO = slot_o(L, tileb_pos(L, warp * TPW)) ^ lOb;
    // this thread's units tid + k T in the staging and output buffers (the
    // swizzles are linear and tid, k T have disjoint bits)
    const uint32_t uS = slot_s((uint32_t)tid << 3), uO = slot_o(L, (uint32_t)tid << 3);
    // units past the row stay zero: in the staging ring (the stage-A loads
    // read them), and in both row buffers (stage A skips those tiles, stage
    // B reads them: with weight zero, which a stale NaN would not respect)
#pragma unroll
    for (int k = 0; k < TPW; ++k)
        if (tid + k * T >= units) {
#pragma unroll
            for (int s = 0; s < MMA_NS; ++s) sts128_zero(sb + s * BUF + (uS ^ K.s_k[k]) * 16u);
            const uint32_t ur = slot_r(L, (uint32_t)(tid + k * T) << 3);
            sts128_zero(R0 + ur * 16u);
            sts128_zero(R0 + BUF + ur * 16u);
        }

    pdl_wait();  // x, xh and info are shared with the neighbouring kernels
    // this CTA's rows: blockIdx.x + j gridDim.x, j < nmine
    const int nmine = blockIdx.x < B ? (B - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto row_of = [&](int j) { return (int)blockIdx.x + j * (int)gridDim.x; };
    auto issue = [&](int j, int slot) {  // copies of the CTA's row j into staging slot j % 3
        if (j < nmine) {
            const char *src = static_cast<const char *>(p.x) + (size_t)row_of(j) * p.len * 2;
            const uint32_t dst = sb + slot * BUF;
#pragma unroll
            for (int k = 0; k < TPW; ++k) {
                const int u = tid + k * T;
                if (u < units) cp_async16_mma(dst + (uS ^ K.s_k[k]) * 16u, src + (size_t)u * 16);
            }
        }
        cp_async_commit_mma();
    };
    // row max |x| of the CTA's row j over this thread's own copies (as the
    // magnitude bits), per warp into s_max[j & 1]
    auto row_max = [&](int j, int slot) {
        const uint32_t src = sb + slot * BUF;
        uint4 v[TPW];
#pragma unroll
        for (int k = 0; k < TPW; ++k)
            v[k] = tid + k * T < units ? lds128(src + (uS ^ K.s_k[k]) * 16u)
                                       : make_uint4(0u, 0u, 0u, 0u);
        uint32_t mx = 0u;
#pragma unroll
        for (int k = 0; k < TPW; ++k) {
            mx = absmax2<BF16>(mx, v[k].x);
            mx = absmax2<BF16>(mx, v[k].y);
            mx = absmax2<BF16>(mx, v[k].z);
            mx = absmax2<BF16>(mx, v[k].w);
        }
        mx &= 0x7FFF7FFFu;  // magnitudes: as integers, in the order of the values
        mx = __reduce_max_sync(0xffffffffu, max(mx & 0xFFFFu, mx >> 16));
        if (lane == 0) s_max[j & 1][warp] = mx;
    };
    issue(0, 0);
    issue(1, 1);
    if (nmine > 0) {
        cp_async_wait_mma<MMA_NS - 2>();
        row_max(0, 0);
    }
    __syncthreads();

    // Software pipeline over the CTA's rows: phase j runs the copy-out of row
    // j - 2, stage B of row j - 1, stage A of row j and the row max of row
    // j + 1 (independent work, buffers alternating by row parity), then one
    // CTA barrier.
    for (int j = 0, ring = 0; j < nmine + 2; ++j, ring = ring == MMA_NS - 1 ? 0 : ring + 1) {  // ring = j % 3
        const int ring1 = ring == MMA_NS - 1 ? 0 : ring + 1, ring2 = ring1 == MMA_NS - 1 ? 0 : ring1 + 1;
        // ---- copy-out of row j - 2: 16-byte coalesced stores
        if (j >= 2) {
            const uint32_t Ob = O0 + (j & 1) * BUF;
            uint4 *dst = reinterpret_cast<uint4 *>(p.xh + (size_t)row_of(j - 2) * p.len_pad);
#pragma unroll
            for (int k0 = 0; k0 < TPW; k0 += 2) {  // two units in flight at a time
                uint4 v[2];
#pragma unroll
                for (int k = k0; k < k0 + 2; ++k)
                    if (tid + k * T < units) v[k - k0] = lds128(Ob + (uO ^ K.o_k[k]) * 16u);
#pragma unroll
                for (int k = k0; k < k0 + 2; ++k)
                    if (tid + k * T < units) dst[tid + k * T] = v[k - k0];
            }
        }
        // ---- stage B of row j - 1: the remaining bits, one product per tile
        // (row-buffer positions past the row hold zeros)
        if (j >= 1 && j - 1 < nmine) {
            const uint32_t Rb = R0 + ((j - 1) & 1) * BUF, Ob = O0 + ((j - 1) & 1) * BUF;
            uint32_t rb[TPW][4];
#pragma unroll
            for (int i = 0; i < TPW; ++i) ldsm_x4_trans(Rb + 16u * (wB ^ K.rb_i[i]), rb[i]);
            float d[TPW][2][4];
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
                mma16816<false>(d[i][0], aB, rb[i][0], rb[i][1]);
                mma16816<false>(d[i][1], aB, rb[i][2], rb[i][3]);
            }
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    mul_f2(d[i][nt][0], d[i][nt][1], corr0, corr0);
                    mul_f2(d[i][nt][2], d[i][nt][3], corr1, corr1);
                }
                stsm_x4(Ob + 16u * (wO ^ K.ob_i[i]), pack_h2(d[i][0][0], d[i][0][1]), pack_h2(d[i][0][2], d[i][0][3]),
                        pack_h2(d[i][1][0], d[i][1][1]), pack_h2(d[i][1][2], d[i][1][3]));
            }
        }
        // ---- stage A of row j: bits 4-7, then 0-3, of each tile; then the
        // cross bits (tiles past the row are skipped: zero inputs, and the
        // butterflies never pair them with a tile of the row)
        if (j < nmine) {
            const int e = prescale_exp<BF16>(__reduce_max_sync(0xffffffffu, lane < W ? s_max[j & 1][lane] : 0u));
            if (tid == 0) p.info[row_of(j)] = glq_rowinfo{0, __int_as_float((127 - e) << 23), 0.f};
            issue(j + 2, ring2);  // into the slot stage A of row j - 1 read
            // first product: bf16, H16 2^(e-2) (exact, and its fp32 result
            // cannot overflow); fp16, H16 / 4 and the scale 2^e on the result
            const uint32_t m1 = BF16 ? (uint32_t)(125 + e) << 7 : 0x3400u;
            const float scale = __int_as_float((127 + e) << 23);
            uint32_t a1[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) a1[q] = a1s[q] | m1 | m1 << 16;
            const uint32_t Sb = sb + ring * BUF, Rb = R0 + (j & 1) * BUF;
            // (each tile's fragments loaded while the previous tile computes)
            auto real = [&](int i) { return ((uint32_t)(warp * TPW + i) << 8) < len; };
            uint32_t rn[4];
            if (real(0)) ldsm_x4_trans(Sb + ((uint32_t)(warp * TPW) << 9) + lS, rn);
            float d2[TPW][2][4];
#pragma unroll
            for (int i = 0; i < TPW; ++i) {
                uint32_t r[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) r[q] = rn[q] ^ sign_xor(sgn[i >> 2], i, q);  // S_in
                if (i + 1 < TPW && real(i + 1))
                    ldsm_x4_trans(Sb + ((uint32_t)(warp * TPW + i + 1) << 9) + lS, rn);
                if (real(i)) {
                    float d1[2][4];
                    mma16816<BF16>(d1[0], a1, r[0], r[1]);
                    mma16816<BF16>(d1[1], a1, r[2], r[3]);
                    if constexpr (!BF16) {
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            mul_f2(d1[nt][0], d1[nt][1], scale, scale);
                            mul_f2(d1[nt][2], d1[nt][3], scale, scale);
                        }
                    }
                    const uint32_t a2[4] = {pack_h2(d1[0][0], d1[0][1]), pack_h2(d1[0][2], d1[0][3]),
                                            pack_h2(d1[1][0], d1[1][1]), pack_h2(d1[1][2], d1[1][3])};
                    mma16816<false>(d2[i][0], a2, b2[0][0], b2[0][1]);
                    mma16816<false>(d2[i][1], a2, b2[1][0], b2[1][1]);
                }
            }
#pragma unroll
            for (int cb = 0; cb < C; ++cb)
#pragma unroll
                for (int a = 0; a < TPW; ++a)
                    if (!((a >> cb) & 1) && bfly_active((uint32_t)(warp * TPW + a) << 8, 8 + cb, len)) {
                        const int z = a | (1 << cb);
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            bfly_f2(d2[a][nt][0], d2[a][nt][1], d2[z][nt][0], d2[z][nt][1]);
                            bfly_f2(d2[a][nt][2], d2[a][nt][3], d2[z][nt][2], d2[z][nt][3]);
                        }
                    }
#pragma unroll
            for (int i = 0; i < TPW; ++i)
                if (((uint32_t)(warp * TPW + i) << 8) < len) {
                    if (C > 0) {
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            mul_f2(d2[i][nt][0], d2[i][nt][1], fA[i], fA[i]);
                            mul_f2(d2[i][nt][2], d2[i][nt][3], fA[i], fA[i]);
                        }
                    }
                    stsm_x4(Rb + 16u * (wA ^ K.ra_i[i]), pack_h2(d2[i][0][0], d2[i][0][1]),
                            pack_h2(d2[i][0][2], d2[i][0][3]), pack_h2(d2[i][1][0], d2[i][1][1]),
                            pack_h2(d2[i][1][2], d2[i][1][3]));
                }
        }
        // ---- the row max of row j + 1 (this thread's copies of it are done)
        if (j + 1 < nmine) {
            cp_async_wait_mma<MMA_NS - 2>();
            row_max(j + 1, ring1);
        }
        __syncthreads();
    }
    cp_async_wait_mma<0>();  // nothing in flight at exit
}

template <int L, bool BF16>
cudaError_t launch_mma_t(const RowsParams &p, int B, cudaStream_t s, bool pdl) {
    const void *fn = (const void *)rht_in_mma_kernel<L, BF16>;
    constexpr int threads = 32 * mma_warps(L);
    const size_t smem = mma_smem_bytes(L);
    static std::atomic<uint64_t> configured{0};  // devices set
    cudaError_t e = once_per_device(configured, [fn, smem] {
        return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
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

template <bool BF16>
cudaError_t launch_mma_sel(const RowsParams &p, int B, cudaStream_t s, bool pdl) {
    int L = 9;
    while ((1 << L) < p.len) ++L;
    switch (L) {
        case 9: return launch_mma_t<9, BF16>(p, B, s, pdl);
        case 10: return launch_mma_t<10, BF16>(p, B, s, pdl);
        case 11: return launch_mma_t<11, BF16>(p, B, s, pdl);
        case 12: return launch_mma_t<12, BF16>(p, B, s, pdl);
        case 13: return launch_mma_t<13, BF16>(p, B, s, pdl);
        case 14: return launch_mma_t<14, BF16>(p, B, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool rht_in_mma_supported(const RowsParams &p) {
    return !p.xq && p.len == p.len_pad && p.len % 256 == 0 && p.len >= 512 && p.len <= (1 << 14);
}

cudaError_t launch_rht_in_mma(const RowsParams &p, int B, cudaStream_t s, bool pdl) {
    if (B <= 0 || !rht_in_mma_supported(p)) return cudaErrorInvalidValue;
    return p.x_bf16 ? launch_mma_sel<true>(p, B, s, pdl) : launch_mma_sel<false>(p, B, s, pdl);
}

}  // namespace glq
