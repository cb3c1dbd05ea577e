// glq_prefill.cu -- prefill (B > 16 tokens) GEMM of the GLQ linear layer on
// the 5th-generation tensor cores: z[b][r] = sum_k W^[r][k] xr[b][k]
// (glq 0.5.1 PyPI page, "Inference kernels": a tensor-core path for B >= 2
// that matmuls against codebook-reconstructed weights without materialising
// W in memory).
//
// Design (B200, sm_100a), one CTA per SM, persistent over output tiles of
// 128 weight rows x 512 tokens:
//   * warp 0 loads activation tiles (256 tokens x 64 columns, fp16, 128-byte
//     swizzle) with TMA;
//   * warps 2-5 are the dequantising producer: for each 64-column step they
//     read the 16-bit codes of the tile's 128 rows, gather the fp16 codewords
//     from the L2-resident folded codebook, form c = cb1 + rs cb2 and write
//     each 8-weight group as one 16-byte chunk of the swizzled K-major A
//     operand in shared memory;
//   * warp 1 issues tcgen05.mma (kind::f16, M = 128 rows, N = 256 tokens,
//     K = 16) into two TMEM accumulators (512 columns), so every dequantised
//     W step serves 512 tokens;
//   * warps 2-5 then drain TMEM (tcgen05.ld), apply ws * 2^-e per token and
//     store z (fp32).
// Stages are handed over with mbarriers (TMA transaction bytes, producer
// arrivals, tcgen05.commit); every wait is bounded and a timeout aborts the
// CTA with an error flag instead of hanging.
#include "glq_kernels.cuh"
#include "glq_sm100.cuh"

namespace glq {

namespace {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BN = 256;       // tokens per accumulator (MMA N)
constexpr int NACC = 2;       // accumulators per tile (512 tokens)
constexpr int BK = 64;        // columns per stage (one 128-byte swizzle row of fp16)
constexpr int STAGES = 2;
constexpr int W_BYTES = BM * BK * 2;              // 16 KB
constexpr int X_BYTES = BN * BK * 2;              // 32 KB
constexpr int STAGE_BYTES = W_BYTES + NACC * X_BYTES;  // 80 KB
constexpr int THREADS = 192;  // 6 warps
constexpr uint64_t WAIT_NS = 2000000000ull;  // wait limit, ns (2 s)

__device__ __forceinline__ uint4 ldg_nc_u4(const uint4 *p) { return ldg_v4(p); }

__device__ __forceinline__ uint4 neg_h8(uint4 v) {
    v.x ^= 0x80008000u;
    v.y ^= 0x80008000u;
    v.z ^= 0x80008000u;
    v.w ^= 0x80008000u;
    return v;
}

// fp16 codeword of a folded code from the global folded fp16 table.
__device__ __forceinline__ uint4 codeword(const uint4 *tab, uint32_t e, FoldParams f) {
    const bool neg = e >= (uint32_t)f.nb;
    const uint4 v = ldg_nc_u4(tab + (neg ? e - (uint32_t)f.neg_base : e));
    return neg ? neg_h8(v) : v;
}

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t s, uint32_t b, uint32_t a) {  // s * b + a
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(s), "r"(b), "r"(a));
    return r;
}

__device__ __forceinline__ uint4 hfma8(uint32_t rs2, uint4 b, uint4 a) {  // rs * b + a, 8 lanes
    return make_uint4(hfma2_bits(rs2, b.x, a.x), hfma2_bits(rs2, b.y, a.y), hfma2_bits(rs2, b.z, a.z),
                      hfma2_bits(rs2, b.w, a.w));
}

// Dequantise the W tile (BM rows x BK columns) of (row tile rtile, step kb)
// into `wt` (swizzled K-major, 128-byte rows).  Producer thread p (0..127)
// covers rows (g, g+8) of 16-row tile p/16 and lanes t = 2 tp, 2 tp + 1 of
// the fragment-native index stream (p = 16 rt_l + 8 tp + g).
template <int BPW>
__device__ __forceinline__ void dequant_tile(const PrefillParams &p, int rtile, int kb, uint8_t *wt, int pt) {
    const int rt_l = pt >> 4, tp = (pt >> 3) & 1, g = pt & 7;
    const int rt = rtile * (BM / GLQ_ROW_TILE) + rt_l;
    const int kc = kb >> 1, h = kb & 1;
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
        const int t = 2 * tp + tt;
        uint2 c1 = make_uint2(0, 0), c2 = make_uint2(0, 0);
        uint32_t c2b = 0;
        const bool live = rt < p.RT;
        if (live) {
            const size_t slot = ((size_t)rt * p.KC + kc) * 32 + 4 * g + t;
            c1 = *(reinterpret_cast<const uint2 *>(p.idx1 + slot) + h);
            if (BPW == 4) c2 = *(reinterpret_cast<const uint2 *>(reinterpret_cast<const uint4 *>(p.idx2) + slot) + h);
            if (BPW == 3) c2b = *(reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint2 *>(p.idx2) + slot) + h);
        }
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2) {
            const uint32_t w1 = s2 ? c1.y : c1.x;
            const uint32_t w2 = s2 ? c2.y : c2.x;
            const int gl = 4 * s2 + t;  // group within the 64-column step
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                uint4 cw = make_uint4(0, 0, 0, 0);
                if (live) {
                    cw = codeword(p.cb_f16, hi ? (w1 >> 16) : (w1 & 0xFFFFu), p.fold);
                    if (BPW == 4) {
                        const uint4 r = codeword(p.cb_f16, hi ? (w2 >> 16) : (w2 & 0xFFFFu), p.fold);
                        cw = hfma8(p.rs_h2, r, cw);
                    } else if (BPW == 3) {
                        const uint32_t i2 = (c2b >> (8 * (2 * s2 + hi))) & 0xFFu;
                        cw = hfma8(p.rs_h2, ldg_nc_u4(p.res8 + i2), cw);
                    }
                }
                const int row = rt_l * GLQ_ROW_TILE + g + 8 * hi;
                *reinterpret_cast<uint4 *>(wt + row * 128 + ((gl ^ (row & 7)) << 4)) = cw;
            }
        }
    }
}

template <int BPW>
__global__ void __launch_bounds__(THREADS, 1) prefill_kernel(const __grid_constant__ CUtensorMap xmap,
                                                              PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    // x_full: TMA bytes landed; w_full: the 4 producer warps wrote W;
    // empty: the MMAs of the stage finished (tcgen05.commit).
    __shared__ __align__(8) uint64_t x_full[STAGES], w_full[STAGES], empty_bar[STAGES], acc_full, acc_empty,
        mma_done;
    __shared__ uint32_t tmem_holder;
    __shared__ volatile int abort_flag;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KB = p.KC * 2;  // 64-column steps

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&w_full[s], 4);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, 4);
        mbar_init(&mma_done, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        sm100::prefetch_tensormap(&xmap);
    }
    if (warp == 1) {
        sm100::tmem_alloc(&tmem_holder, 512);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem_base = tmem_holder;
    pdl_launch_dependents();
    pdl_wait();  // activations and row info come from the input RHT

    auto fail = [&]() {
        atomicOr(p.err, GLQ_DEVERR_TIMEOUT);
        abort_flag = 1;
    };

    uint32_t it = 0;        // pipeline step counter (stage, phase)
    uint32_t tcount = 0;    // tiles done by this CTA (accumulator phase)
    int32_t last_load = -1; // TMA thread: last step it issued
    for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++tcount) {
        const int rtile = tile / p.tiles_tok, ttile = tile - rtile * p.tiles_tok;
        const int tok0 = ttile * (BN * NACC);
        // accumulators with at least one live token
        const int na = min(NACC, (p.B - tok0 + BN - 1) / BN);
        if (warp == 0) {
            if (lane == 0) {
                for (int kb = 0; kb < KB && !abort_flag; ++kb) {
                    const uint32_t s = (it + kb) % STAGES, use = (it + kb) / STAGES;
                    if (!sm100::mbar_wait(&empty_bar[s], (use & 1) ^ 1, WAIT_NS)) {
                        fail();
                        break;
                    }
                    uint8_t *st = smem + s * STAGE_BYTES;
                    mbar_expect_tx(&x_full[s], na * X_BYTES);
                    for (int a = 0; a < na; ++a)
                        sm100::tma_load_2d(st + W_BYTES + a * X_BYTES, &xmap, &x_full[s], kb * BK, tok0 + a * BN);
                    last_load = (int32_t)(it + kb);
                }
            }
        } else if (warp == 1) {
            if (lane == 0) {
                const uint32_t idesc = sm100::idesc_f16_f32(BM, BN);
                if (!sm100::mbar_wait(&acc_empty, (tcount & 1) ^ 1, WAIT_NS)) fail();
                sm100::tc_fence_after();
                for (int kb = 0; kb < KB && !abort_flag; ++kb) {
                    const uint32_t s = (it + kb) % STAGES, use = (it + kb) / STAGES;
                    if (!sm100::mbar_wait(&x_full[s], use & 1, WAIT_NS) ||
                        !sm100::mbar_wait(&w_full[s], use & 1, WAIT_NS)) {
                        fail();
                        break;
                    }
                    sm100::tc_fence_after();
                    uint8_t *st = smem + s * STAGE_BYTES;
                    const uint64_t adesc = sm100::smem_desc_sw128(st);
                    for (int a = 0; a < na; ++a) {
                        const uint64_t bdesc = sm100::smem_desc_sw128(st + W_BYTES + a * X_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            sm100::mma_f16_ss(tmem_base + a * BN, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                              (kb | kk) != 0);
                    }
                    sm100::mma_commit(&empty_bar[s]);
                }
                sm100::mma_commit(&acc_full);
            }
        } else {
            // producer: dequantise W steps
            const int pt = tid - 64;
            for (int kb = 0; kb < KB && !abort_flag; ++kb) {
                const uint32_t s = (it + kb) % STAGES, use = (it + kb) / STAGES;
                if (!sm100::mbar_wait(&empty_bar[s], (use & 1) ^ 1, WAIT_NS)) {
                    fail();
                    break;
                }
                dequant_tile<BPW>(p, rtile, kb, smem + s * STAGE_BYTES, pt);
                sm100::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&w_full[s]);
            }
            // epilogue: TMEM lanes of this warp's quadrant -> z rows
            const int q = warp & 3;
            const int row = rtile * BM + 32 * q + lane;
            const bool ok = !abort_flag && sm100::mbar_wait(&acc_full, tcount & 1, WAIT_NS);
            if (!ok && !abort_flag) fail();
            sm100::tc_fence_after();
            if (ok) {
                for (int a = 0; a < na; ++a) {
                    for (int c = 0; c < BN / 16; ++c) {
                        uint32_t r[16];
                        sm100::tmem_ld16(tmem_base + ((uint32_t)(32 * q) << 16) + a * BN + c * 16, r);
                        sm100::tmem_wait_ld();
                        const int tb = tok0 + a * BN + c * 16;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int tok = tb + j;
                            if (tok < p.B && row < p.m_pad)
                                p.z[(size_t)tok * p.m_pad + row] =
                                    __uint_as_float(r[j]) * p.ws * p.info[tok].inv_scale;
                        }
                    }
                }
            }
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&acc_empty);
        }
        it += KB;
        if (abort_flag) break;
    }
    // Drain what may still be in flight after an abort: the TMA thread waits
    // for its last load of each stage, the MMA thread for all its MMAs.
    if (warp == 0 && lane == 0 && abort_flag) {
        for (int32_t i = max(0, last_load - (STAGES - 1)); i <= last_load; ++i)
            sm100::mbar_wait(&x_full[i % STAGES], (uint32_t)(i / STAGES) & 1, WAIT_NS);
    }
    if (warp == 1 && lane == 0) {
        sm100::mma_commit(&mma_done);
        sm100::mbar_wait(&mma_done, 0, WAIT_NS);
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace

size_t prefill_smem_bytes() { return (size_t)STAGES * STAGE_BYTES + 1024; }

int prefill_tile_tokens() { return BN * NACC; }

cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &xmap, int grid, cudaStream_t s, bool pdl) {
    const size_t smem = prefill_smem_bytes();
    const void *fn = p.bpw == 4 ? (const void *)prefill_kernel<4>
                                : (p.bpw == 3 ? (const void *)prefill_kernel<3> : (const void *)prefill_kernel<2>);
    static bool configured[5] = {false, false, false, false, false};
    if (!configured[p.bpw]) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured[p.bpw] = true;
    }
    PrefillParams q = p;
    CUtensorMap m = xmap;
    void *args[] = {&m, &q};
    return launch_ex(fn, dim3(grid), dim3(THREADS), smem, s, pdl, args);
}

}  // namespace glq
