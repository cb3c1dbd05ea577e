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
//     order and writes the band's final z.
#include "glq_kernels.cuh"

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

// One stage (one code per row) of one super-tile: codes of rows g and g+8.
template <int NT>
__device__ __forceinline__ void stage_int(const uint32_t *T, FoldParams fold, uint32_t codes,
                                          const uint4 &x0, const uint4 &x1, Acc &acc) {
    const uint32_t wg = table_word(T, codes & 0xFFFFu, fold);
    const uint32_t wg8 = table_word(T, codes >> 16, fold);
    const uint32_t a[4] = {nib_lo(wg), nib_lo(wg8), nib_hi(wg), nib_hi(wg8)};
    mma_u8s8(acc.hi[0], a, x0.x, x0.y);
    mma_u8u8(acc.lo[0], a, x0.z, x0.w);
    if (NT == 2) {
        mma_u8s8(acc.hi[NT - 1], a, x1.x, x1.y);
        mma_u8u8(acc.lo[NT - 1], a, x1.z, x1.w);
    }
}

template <int BPW, int NT>
__device__ __forceinline__ void process_chunk(const uint32_t *T, const uint4 *R8, FoldParams fold,
                                              const uint4 &q1, const uint4 &q2, const uint4 *xq0,
                                              const uint4 *xq1, const __half *xh0, const __half *xh1,
                                              bool has0, bool has1, Acc &acc1, Acc &acc2,
                                              float accr[2][4]) {
    const uint32_t p1[4] = {q1.x, q1.y, q1.z, q1.w};
    const uint32_t p2[4] = {q2.x, q2.y, q2.z, q2.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
        if (has0) x0 = ldg_v4(xq0 + 4 * s);
        if (NT == 2 && has1) x1 = ldg_v4(xq1 + 4 * s);
        stage_int<NT>(T, fold, p1[s], x0, x1, acc1);
        if (BPW == 4) stage_int<NT>(T, fold, p2[s], x0, x1, acc2);
        if (BPW == 3) {
            // bytes 2s (row g) and 2s+1 (row g+8) of the 8-byte payload
            const uint32_t word = (s < 2) ? q2.x : q2.y;
            const uint32_t sh = (s & 1) * 16;
            const uint4 ra = R8[(word >> sh) & 0xFFu];
            const uint4 rb = R8[(word >> (sh + 8)) & 0xFFu];
            const uint32_t lo[4] = {ra.x, rb.x, ra.y, rb.y};
            const uint32_t hi[4] = {ra.z, rb.z, ra.w, rb.w};
            uint4 h0 = make_uint4(0, 0, 0, 0), h1 = make_uint4(0, 0, 0, 0);
            if (has0) h0 = ldg_v4(xh0 + 32 * s);
            if (NT == 2 && has1) h1 = ldg_v4(xh1 + 32 * s);
            mma_16816(accr[0], lo, h0.x, h0.y);
            mma_16816(accr[0], hi, h0.z, h0.w);
            if (NT == 2) {
                mma_16816(accr[NT - 1], lo, h1.x, h1.y);
                mma_16816(accr[NT - 1], hi, h1.z, h1.w);
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

__device__ __forceinline__ double exact_sum(int hi, int lo) {
    return (double)((long long)hi * 256 + (long long)lo);
}

// z of (token b, any row) from D = sum over splits of the partials:
// z = ws 2^-e (D - 6 corr_mult sum X) / 2.
__device__ __forceinline__ float finish_z(const GemvParams &p, int b, double D) {
    const glq_rowinfo info = p.info[b];
    const double corr = (double)GLQ_NIB_OFFSET * p.corr_mult * (double)info.sum_x;
    return (float)((D - corr) * (0.5 * (double)p.ws * (double)info.inv_scale));
}

template <int BPW, int NT>
__global__ void __launch_bounds__(gemv_warps(NT) * 32, 1) gemv_kernel(GemvParams p) {
    constexpr int WARPS = gemv_warps(NT);
    constexpr int BAND_ROWS = WARPS * GLQ_ROW_TILE;
    extern __shared__ __align__(16) uint4 smem_u4[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int s_last;
    uint32_t *T = reinterpret_cast<uint32_t *>(smem_u4);
    uint4 *R8 = smem_u4 + p.table_words / 4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int ntasks = p.bands * p.splits;

    // 1. codebook into shared memory (constant data: before the PDL wait)
    if (tid == 0) mbar_init(&bar, 1);
    __syncthreads();
    if (tid == 0) {
        const uint32_t tbytes = (uint32_t)p.table_words * 4u;
        const uint32_t rbytes = BPW == 3 ? 256u * 16u : 0u;
        mbar_expect_tx(&bar, tbytes + rbytes);
        const uint32_t piece = 32768u;
        for (uint32_t off = 0; off < tbytes; off += piece) {
            const uint32_t len = tbytes - off < piece ? tbytes - off : piece;
            bulk_g2s(reinterpret_cast<char *>(T) + off, reinterpret_cast<const char *>(p.table) + off,
                     len, &bar);
        }
        if (BPW == 3) bulk_g2s(R8, p.res8, rbytes, &bar);
    }
    pdl_launch_dependents();

    // 2. index loads of the first task (constant data: before the PDL wait)
    uint4 r1[GEMV_PREFETCH], r2[GEMV_PREFETCH];
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
            if (rt < p.RT && c0 + i < c1) {
                r1[i] = ldg_nc_v4(p.idx1 + base + (size_t)(c0 + i) * 32);
                r2[i] = load_q2<BPW>(p.idx2, base + (size_t)(c0 + i) * 32);
            }
        }
    };
    if (task < ntasks) {
        task_geom(task);
        prefetch();
    }

    const bool ok = mbar_wait_bounded(&bar, 0, TABLE_WAIT_POLLS);
    if (!ok) {
        if (tid == 0) atomicOr(p.err, GLQ_DEVERR_TIMEOUT);
        mbar_wait_bounded(&bar, 0, TABLE_WAIT_POLLS);  // let the copy land before exiting
        return;
    }
    // 3. activations and row info come from the input-RHT kernel
    pdl_wait();

    const bool has0 = g < p.B, has1 = (g + 8) < p.B;
    const size_t xq_row = (size_t)p.n_pad / 8;  // uint4 (one group) per 8 columns
    const uint4 *xq0 = reinterpret_cast<const uint4 *>(p.xq) + (size_t)g * xq_row + t;
    const uint4 *xq1 = reinterpret_cast<const uint4 *>(p.xq) + (size_t)(g + 8) * xq_row + t;
    const __half *xh0 = p.xh ? p.xh + (size_t)g * p.n_pad + 8 * t : nullptr;
    const __half *xh1 = p.xh ? p.xh + (size_t)(g + 8) * p.n_pad + 8 * t : nullptr;

    for (bool first = true; task < ntasks; task += gridDim.x, first = false) {
        if (!first) {
            task_geom(task);
            prefetch();
        }
        const int band = task / p.splits, split = task - band * p.splits;
        Acc acc1, acc2;
        zero<NT>(acc1);
        zero<NT>(acc2);
        float accr[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};

        if (rt < p.RT) {
            const size_t base = ((size_t)rt * p.KC + c0) * 32 + lane;
            const uint4 *pq1 = p.idx1 + base + GEMV_PREFETCH * 32;  // next chunk to load
            const size_t q2_off = base + GEMV_PREFETCH * 32;
            const uint4 *px0 = xq0 + (size_t)c0 * GLQ_GROUPS_PER_CHUNK;
            const uint4 *px1 = xq1 + (size_t)c0 * GLQ_GROUPS_PER_CHUNK;
            const __half *ph0 = xh0 ? xh0 + (size_t)c0 * GLQ_CHUNK_K : nullptr;
            const __half *ph1 = xh1 ? xh1 + (size_t)c0 * GLQ_CHUNK_K : nullptr;
            int ahead = c0 + GEMV_PREFETCH;
            for (int c = c0; c < c1; c += GEMV_PREFETCH) {
#pragma unroll
                for (int i = 0; i < GEMV_PREFETCH; ++i) {
                    if (c + i < c1) {
                        const uint4 q1 = r1[i], q2 = r2[i];
                        if (ahead < c1) {
                            r1[i] = ldg_nc_v4(pq1);
                            r2[i] = load_q2<BPW>(p.idx2, q2_off + (size_t)(ahead - c0 - GEMV_PREFETCH) * 32);
                        }
                        pq1 += 32;
                        ++ahead;
                        process_chunk<BPW, NT>(T, R8, p.fold, q1, q2, px0, px1, ph0, ph1, has0, has1, acc1,
                                               acc2, accr);
                        px0 += GLQ_GROUPS_PER_CHUNK;
                        px1 += GLQ_GROUPS_PER_CHUNK;
                        if (BPW == 3) {
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
                        if (BPW == 4) D += p.rs_d * exact_sum(acc2.hi[nt][j], acc2.lo[nt][j]);
                        if (BPW == 3) D += p.rs_d * (double)accr[nt][j];
                        if (p.splits == 1) {
                            p.z[(size_t)b * p.m_pad + row] = finish_z(p, b, D);
                        } else {
                            __stcg(p.partials + ((size_t)split * p.B + b) * p.m_pad + row, D);
                        }
                    }
                }
            }
        }
        if (p.splits == 1) continue;

        // 4. band completion: the last split to finish reduces the band.  The
        // CTA barrier orders every thread's partial stores before thread 0's
        // release-acquire increment; the barrier after it hands the acquire to
        // the threads that read the other CTAs' partials.
        __syncthreads();
        if (tid == 0) {
            const unsigned prev = atom_add_acq_rel_gpu(&p.counters[band], 1u);
            s_last = prev == (unsigned)(p.splits - 1);
        }
        __syncthreads();
        if (s_last) {
            const int r_base = band * BAND_ROWS;
            const int rows = min(BAND_ROWS, p.m_pad - r_base);
            for (int e = tid; e < rows * p.B; e += WARPS * 32) {
                const int b = e / rows, row = r_base + (e - b * rows);
                double D = 0.0;
                for (int s = 0; s < p.splits; ++s)  // fixed order
                    D += __ldcg(p.partials + ((size_t)s * p.B + b) * p.m_pad + row);
                p.z[(size_t)b * p.m_pad + row] = finish_z(p, b, D);
            }
            if (tid == 0) p.counters[band] = 0u;
        }
        __syncthreads();  // s_last is reused by the next task
    }
}

template <int BPW, int NT>
cudaError_t launch_t(const GemvParams &p, int grid, cudaStream_t s, bool pdl) {
    const size_t smem = gemv_smem_bytes(p.table_words, BPW);
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
    return launch_ex((const void *)gemv_kernel<BPW, NT>, dim3(grid), dim3(gemv_warps(NT) * 32), smem, s,
                     pdl, args);
}

}  // namespace

// Split of the chunk range so that (bands x splits) tasks spread over the
// persistent grid with the least makespan (in chunks per CTA), with a small
// charge per task for the band reduction.
GemvPlan plan_gemv(int RT, int KC, int num_sms, int warps) {
    GemvPlan pl{};
    pl.bands = (RT + warps - 1) / warps;
    int best_s = 1;
    double best = 1e30;
    for (int s = 1; s <= KC; ++s) {
        const int cps = (KC + s - 1) / s;
        const int used = (KC + cps - 1) / cps;  // splits actually populated
        if (used != s) continue;
        const long long tasks = (long long)pl.bands * s;
        const long long waves = (tasks + num_sms - 1) / num_sms;
        const double cost = (double)waves * (cps + (s > 1 ? 0.5 : 0.0)) + 0.02 * s;
        if (cost < best) {
            best = cost;
            best_s = s;
        }
    }
    pl.splits = best_s;
    pl.cps = (KC + best_s - 1) / best_s;
    const long long tasks = (long long)pl.bands * pl.splits;
    pl.grid = (int)(tasks < num_sms ? tasks : num_sms);
    return pl;
}

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
