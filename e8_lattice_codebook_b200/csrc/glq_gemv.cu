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
//     launch with a bulk async copy before the programmatic-dependent-launch
//     wait, so it overlaps the input RHT;
//   * a task is (band of 16 row tiles = 256 rows, split of the chunk range);
//     each warp owns one 16-row tile and streams its fragment-native index
//     stream with coalesced 128-bit non-allocating loads, 4 chunks ahead;
//   * each lane turns a 16-bit code into one whole 8-D codeword (fold,
//     one shared-memory word, one AND per coordinate pair giving exact fp16
//     subnormals) and feeds it straight into the A fragment of
//     mma.m16n8k16 (fp16 x fp16 -> fp32); the batch (<= 8 or <= 16 tokens)
//     is the N dimension;
//   * the residual stage accumulates separately and is scaled once;
//   * partial sums per split go to a workspace, reduced in fixed order by
//     the output-RHT kernel (no atomics: bitwise reproducible).
#include "glq_kernels.cuh"

namespace glq {

namespace {

constexpr uint32_t TABLE_WAIT_POLLS = 1u << 24;

template <int BPW, int NT>
__device__ __forceinline__ void process_chunk(const uint32_t *T, const uint4 *R8, FoldParams fold,
                                              uint4 q1, uint4 q2, const __half *xrow0,
                                              const __half *xrow1, bool has0, bool has1,
                                              float acc1[NT][4], float acc2[NT][4]) {
    const uint32_t p1[4] = {q1.x, q1.y, q1.z, q1.w};
    const uint32_t p2[4] = {q2.x, q2.y, q2.z, q2.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint4 xb0 = make_uint4(0, 0, 0, 0), xb1 = make_uint4(0, 0, 0, 0);
        if (has0) xb0 = ldg_v4(xrow0 + 32 * s);
        if (NT == 2 && has1) xb1 = ldg_v4(xrow1 + 32 * s);

        uint32_t ha[4], hb[4];
        unpack_sub(table_word(T, p1[s] & 0xFFFFu, fold), ha);
        unpack_sub(table_word(T, p1[s] >> 16, fold), hb);
        {
            const uint32_t lo[4] = {ha[0], hb[0], ha[1], hb[1]};
            const uint32_t hi[4] = {ha[2], hb[2], ha[3], hb[3]};
            mma_16816(acc1[0], lo, xb0.x, xb0.y);
            mma_16816(acc1[0], hi, xb0.z, xb0.w);
            if (NT == 2) {
                mma_16816(acc1[NT - 1], lo, xb1.x, xb1.y);
                mma_16816(acc1[NT - 1], hi, xb1.z, xb1.w);
            }
        }
        if (BPW == 4) {
            // two codes per 32-bit word: row g in the low half, row g+8 high
            unpack_sub(table_word(T, p2[s] & 0xFFFFu, fold), ha);
            unpack_sub(table_word(T, p2[s] >> 16, fold), hb);
            const uint32_t lo[4] = {ha[0], hb[0], ha[1], hb[1]};
            const uint32_t hi[4] = {ha[2], hb[2], ha[3], hb[3]};
            mma_16816(acc2[0], lo, xb0.x, xb0.y);
            mma_16816(acc2[0], hi, xb0.z, xb0.w);
            if (NT == 2) {
                mma_16816(acc2[NT - 1], lo, xb1.x, xb1.y);
                mma_16816(acc2[NT - 1], hi, xb1.z, xb1.w);
            }
        } else if (BPW == 3) {
            // bytes 2s (row g) and 2s+1 (row g+8) of the 8-byte payload
            uint32_t word = (s < 2) ? q2.x : q2.y;
            uint32_t sh = (s & 1) * 16;
            uint4 ra = R8[(word >> sh) & 0xFFu];
            uint4 rb = R8[(word >> (sh + 8)) & 0xFFu];
            const uint32_t lo[4] = {ra.x, rb.x, ra.y, rb.y};
            const uint32_t hi[4] = {ra.z, rb.z, ra.w, rb.w};
            mma_16816(acc2[0], lo, xb0.x, xb0.y);
            mma_16816(acc2[0], hi, xb0.z, xb0.w);
            if (NT == 2) {
                mma_16816(acc2[NT - 1], lo, xb1.x, xb1.y);
                mma_16816(acc2[NT - 1], hi, xb1.z, xb1.w);
            }
        }
    }
}

template <int BPW>
__device__ __forceinline__ uint4 load_q2(const void *idx2, size_t i) {
    if (BPW == 4) return ldg_nc_v4(reinterpret_cast<const uint4 *>(idx2) + i);
    if (BPW == 3) {
        uint2 v = ldg_nc_v2(reinterpret_cast<const uint2 *>(idx2) + i);
        return make_uint4(v.x, v.y, 0, 0);
    }
    return make_uint4(0, 0, 0, 0);
}

template <int BPW, int NT>
__global__ void __launch_bounds__(GEMV_WARPS * 32, 1) gemv_kernel(GemvParams p) {
    extern __shared__ __align__(16) uint4 smem_u4[];
    __shared__ __align__(8) uint64_t bar;
    uint32_t *T = reinterpret_cast<uint32_t *>(smem_u4);
    uint4 *R8 = smem_u4 + p.table_words / 4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;

    // 1. codebook into shared memory (constant data: before the PDL wait)
    if (tid == 0) mbar_init(&bar, 1);
    __syncthreads();
    if (tid == 0) {
        uint32_t tbytes = (uint32_t)p.table_words * 4u;
        uint32_t rbytes = BPW == 3 ? 256u * 16u : 0u;
        mbar_expect_tx(&bar, tbytes + rbytes);
        const uint32_t piece = 32768u;
        for (uint32_t off = 0; off < tbytes; off += piece) {
            uint32_t len = tbytes - off < piece ? tbytes - off : piece;
            bulk_g2s(reinterpret_cast<char *>(T) + off, reinterpret_cast<const char *>(p.table) + off,
                     len, &bar);
        }
        if (BPW == 3) bulk_g2s(R8, p.res8, rbytes, &bar);
    }
    pdl_launch_dependents();
    bool ok = mbar_wait_bounded(&bar, 0, TABLE_WAIT_POLLS);
    if (!ok) {
        if (tid == 0) atomicOr(p.err, GLQ_DEVERR_TIMEOUT);
        mbar_wait_bounded(&bar, 0, TABLE_WAIT_POLLS);  // let the copy land before exiting
        return;
    }

    // 2. activations come from the input-RHT kernel
    pdl_wait();

    const int ntasks = p.bands * p.splits;
    for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
        const int band = task / p.splits, split = task - band * p.splits;
        const int rt = band * GEMV_WARPS + warp;
        if (rt >= p.RT) continue;
        const int c0 = split * p.cps;
        const int c1 = min(p.KC, c0 + p.cps);
        if (c0 >= c1) continue;

        float acc1[NT][4], acc2[NT][4];
#pragma unroll
        for (int i = 0; i < NT; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc1[i][j] = acc2[i][j] = 0.f;

        const size_t base = ((size_t)rt * p.KC) * 32 + lane;
        const bool has0 = g < p.B, has1 = (g + 8) < p.B;
        const __half *x0 = p.xr + (size_t)g * p.n_pad + 8 * t;
        const __half *x1 = p.xr + (size_t)(g + 8) * p.n_pad + 8 * t;

        uint4 r1[GEMV_PREFETCH], r2[GEMV_PREFETCH];
#pragma unroll
        for (int i = 0; i < GEMV_PREFETCH; ++i) {
            if (c0 + i < c1) {
                r1[i] = ldg_nc_v4(p.idx1 + base + (size_t)(c0 + i) * 32);
                r2[i] = load_q2<BPW>(p.idx2, base + (size_t)(c0 + i) * 32);
            }
        }
        for (int c = c0; c < c1; c += GEMV_PREFETCH) {
#pragma unroll
            for (int i = 0; i < GEMV_PREFETCH; ++i) {
                const int cc = c + i;
                if (cc < c1) {
                    uint4 q1 = r1[i], q2 = r2[i];
                    if (cc + GEMV_PREFETCH < c1) {
                        r1[i] = ldg_nc_v4(p.idx1 + base + (size_t)(cc + GEMV_PREFETCH) * 32);
                        r2[i] = load_q2<BPW>(p.idx2, base + (size_t)(cc + GEMV_PREFETCH) * 32);
                    }
                    const size_t xo = (size_t)cc * GLQ_CHUNK_K;
                    process_chunk<BPW, NT>(T, R8, p.fold, q1, q2, x0 + xo, x1 + xo, has0, has1, acc1,
                                           acc2);
                }
            }
        }

        // 3. partial sums: lane (g, t) holds rows g, g+8 and batch columns
        // nt*8 + 2t, 2t+1
        const int row0 = rt * GLQ_ROW_TILE + g;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int b = nt * 8 + 2 * t + (j & 1);
                const int row = row0 + (j >> 1) * 8;
                if (b < p.B) {
                    float v = acc1[nt][j];
                    if (BPW > 2) v = fmaf(p.rs_acc, acc2[nt][j], v);
                    p.partials[((size_t)split * p.B + b) * p.m_pad + row] = v;
                }
            }
        }
    }
}

template <int BPW, int NT>
cudaError_t launch_t(const GemvParams &p, int grid, cudaStream_t s, bool pdl) {
    size_t smem = gemv_smem_bytes(p.table_words, BPW);
    // raised once to the largest table the library accepts (never lowered:
    // captured graphs replay against the attribute value at replay time)
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemv_kernel<BPW, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)gemv_smem_bytes(GLQ_TABLE_MAX_WORDS, BPW));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    GemvParams q = p;
    void *args[] = {&q};
    return launch_ex((const void *)gemv_kernel<BPW, NT>, dim3(grid), dim3(GEMV_WARPS * 32), smem, s,
                     pdl, args);
}

}  // namespace

size_t gemv_smem_bytes(int table_words, int bpw) {
    return (size_t)table_words * 4 + (bpw == 3 ? 256 * 16 : 0);
}

cudaError_t launch_gemv(const GemvParams &p, int bpw, int grid, cudaStream_t s, bool pdl) {
    const bool two = p.B > 8;
    switch (bpw) {
        case 2: return two ? launch_t<2, 2>(p, grid, s, pdl) : launch_t<2, 1>(p, grid, s, pdl);
        case 3: return two ? launch_t<3, 2>(p, grid, s, pdl) : launch_t<3, 1>(p, grid, s, pdl);
        case 4: return two ? launch_t<4, 2>(p, grid, s, pdl) : launch_t<4, 1>(p, grid, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace glq
