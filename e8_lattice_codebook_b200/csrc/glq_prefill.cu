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
//   * warp 1 issues tcgen05.mma (kind::f16, M = 128 rows, N = 256 tokens,
//     K = 16) into two TMEM accumulators (512 columns), so every dequantised
//     W step serves 512 tokens;
//   * warps 2-5 are the dequantising producer: for each 64-column step they
//     read the 16-bit codes of the tile's 128 rows, gather the fp16 codewords
//     from the L2-resident table (indexed by folded code), form
//     c = cb1 + rs cb2 and write each 8-weight group as one 16-byte chunk of
//     the swizzled K-major A operand in shared memory.  The gathers of step
//     k+1 and the code loads of step k+2 are in flight while step k is
//     stored, so each step waits on at most one memory round trip;
//   * warps 6-9 drain each accumulator as soon as its last MMA completes
//     (tcgen05.ld), apply ws * 2^-e per token and store z (fp32), while the
//     producer already works on the next tile.
// Stages are handed over with mbarriers (TMA transaction bytes, producer
// arrivals, tcgen05.commit); every wait is bounded in time and a timeout
// aborts the CTA with an error flag instead of hanging.
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
constexpr int THREADS = 320;  // 10 warps: TMA, MMA, 4 producer, 4 epilogue
constexpr uint64_t WAIT_NS = 2000000000ull;  // wait limit, ns (2 s)

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t s, uint32_t b, uint32_t a) {  // s * b + a
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(s), "r"(b), "r"(a));
    return r;
}

__device__ __forceinline__ uint4 hfma8(uint32_t rs2, uint4 b, uint4 a) {  // rs * b + a, 8 lanes
    return make_uint4(hfma2_bits(rs2, b.x, a.x), hfma2_bits(rs2, b.y, a.y), hfma2_bits(rs2, b.z, a.z),
                      hfma2_bits(rs2, b.w, a.w));
}

// Producer thread pt (0..127) of a W step: rows (g, g + 8) of 16-row tile
// rt_l = pt / 16, lanes t = 2 tp, 2 tp + 1 of the fragment-native index
// stream (pt = 16 rt_l + 8 tp + g).  Its 8 groups are i = 4 tt + 2 s2 + hi:
// row 16 rt_l + g + 8 hi, group 4 s2 + t of the step, t = 2 tp + tt.
struct StepCodes {
    uint2 c1[2];     // primary codes, words s = 2h, 2h + 1 of lanes t
    uint2 c2[2];     // 4 bpw residual codes
    uint32_t c3[2];  // 3 bpw residual bytes
};

template <int BPW>
__device__ __forceinline__ void load_codes(const PrefillParams &p, size_t slot0, int kb, bool live, StepCodes &c) {
    const int kc = kb >> 1, h = kb & 1;
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
        const size_t slot = slot0 + (size_t)kc * 32 + tt;
        c.c1[tt] = live ? __ldg(reinterpret_cast<const uint2 *>(p.idx1 + slot) + h) : make_uint2(0, 0);
        if (BPW == 4)
            c.c2[tt] = live ? __ldg(reinterpret_cast<const uint2 *>(reinterpret_cast<const uint4 *>(p.idx2) + slot) + h)
                            : make_uint2(0, 0);
        if (BPW == 3)
            c.c3[tt] = live ? __ldg(reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint2 *>(p.idx2) + slot) + h)
                            : 0u;
    }
}

struct StepWords {
    uint4 a[8];  // primary codewords
    uint4 b[8];  // residual codewords
};

template <int BPW>
__device__ __forceinline__ void issue_gathers(const PrefillParams &p, const StepCodes &c, bool live, StepWords &w) {
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int i = 4 * tt + 2 * s2 + hi;
                const uint32_t w1 = s2 ? c.c1[tt].y : c.c1[tt].x;
                w.a[i] = live ? __ldg(p.cb_f16 + (hi ? (w1 >> 16) : (w1 & 0xFFFFu))) : make_uint4(0, 0, 0, 0);
                if (BPW == 4) {
                    const uint32_t w2 = s2 ? c.c2[tt].y : c.c2[tt].x;
                    w.b[i] = live ? __ldg(p.cb_f16 + (hi ? (w2 >> 16) : (w2 & 0xFFFFu))) : make_uint4(0, 0, 0, 0);
                } else if (BPW == 3) {
                    const uint32_t i2 = (c.c3[tt] >> (8 * (2 * s2 + hi))) & 0xFFu;
                    w.b[i] = live ? __ldg(p.res8 + i2) : make_uint4(0, 0, 0, 0);
                }
            }
}

template <int BPW>
__device__ __forceinline__ void store_step(const PrefillParams &p, const StepWords &w, uint8_t *wt, int rt_l, int tp,
                                           int g) {
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int i = 4 * tt + 2 * s2 + hi;
                const uint4 cw = BPW == 2 ? w.a[i] : hfma8(p.rs_h2, w.b[i], w.a[i]);
                const int row = rt_l * GLQ_ROW_TILE + g + 8 * hi;
                const int gl = 4 * s2 + 2 * tp + tt;
                *reinterpret_cast<uint4 *>(wt + row * 128 + ((gl ^ (row & 7)) << 4)) = cw;
            }
}

template <int BPW>
__global__ void __launch_bounds__(THREADS, 1) prefill_kernel(const __grid_constant__ CUtensorMap xmap,
                                                              PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    // x_full: TMA bytes landed; w_full: the 4 producer warps wrote W;
    // empty: the MMAs of the stage finished (tcgen05.commit);
    // acc_full / acc_empty: accumulator a computed / drained.
    __shared__ __align__(8) uint64_t x_full[STAGES], w_full[STAGES], empty_bar[STAGES], acc_full[NACC],
        acc_empty[NACC], mma_done;
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
        for (int a = 0; a < NACC; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
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
    // live accumulators of a tile (tokens tok0 .. tok0 + 512)
    auto live_acc = [&](int tok0) { return min(NACC, (p.B - tok0 + BN - 1) / BN); };

    if (warp == 0) {
        // ---------------- TMA producer of the activation tiles ----------------
        if (lane == 0) {
            uint32_t it = 0;
            int32_t last_load = -1;
            for (int tile = blockIdx.x; tile < p.ntiles && !abort_flag; tile += gridDim.x) {
                const int ttile = tile % p.tiles_tok;
                const int tok0 = ttile * (BN * NACC), na = live_acc(tok0);
                for (int kb = 0; kb < KB && !abort_flag; ++kb, ++it) {
                    const uint32_t s = it % STAGES, use = it / STAGES;
                    if (!sm100::mbar_wait(&empty_bar[s], (use & 1) ^ 1, WAIT_NS)) {
                        fail();
                        break;
                    }
                    uint8_t *st = smem + s * STAGE_BYTES;
                    mbar_expect_tx(&x_full[s], na * X_BYTES);
                    for (int a = 0; a < na; ++a)
                        sm100::tma_load_2d(st + W_BYTES + a * X_BYTES, &xmap, &x_full[s], kb * BK, tok0 + a * BN);
                    last_load = (int32_t)it;
                }
            }
            if (abort_flag)  // let the copies in flight land before the CTA exits
                for (int32_t i = max(0, last_load - (STAGES - 1)); i <= last_load; ++i)
                    sm100::mbar_wait(&x_full[i % STAGES], (uint32_t)(i / STAGES) & 1, WAIT_NS);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = sm100::idesc_f16_f32(BM, BN);
            uint32_t it = 0, acc_use[NACC] = {0, 0};
            for (int tile = blockIdx.x; tile < p.ntiles && !abort_flag; tile += gridDim.x) {
                const int ttile = tile % p.tiles_tok;
                const int na = live_acc(ttile * (BN * NACC));
                for (int kb = 0; kb < KB && !abort_flag; ++kb, ++it) {
                    const uint32_t s = it % STAGES, use = it / STAGES;
                    if (!sm100::mbar_wait(&x_full[s], use & 1, WAIT_NS) ||
                        !sm100::mbar_wait(&w_full[s], use & 1, WAIT_NS)) {
                        fail();
                        break;
                    }
                    sm100::tc_fence_after();
                    uint8_t *st = smem + s * STAGE_BYTES;
                    const uint64_t adesc = sm100::smem_desc_sw128(st);
                    for (int a = 0; a < na; ++a) {
                        if (kb == 0) {  // the epilogue must have drained this accumulator
                            if (!sm100::mbar_wait(&acc_empty[a], (acc_use[a] & 1) ^ 1, WAIT_NS)) {
                                fail();
                                break;
                            }
                            sm100::tc_fence_after();
                        }
                        const uint64_t bdesc = sm100::smem_desc_sw128(st + W_BYTES + a * X_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            sm100::mma_f16_ss(tmem_base + a * BN, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                              (kb | kk) != 0);
                        if (kb == KB - 1) sm100::mma_commit(&acc_full[a]);
                    }
                    sm100::mma_commit(&empty_bar[s]);
                }
                for (int a = 0; a < na; ++a) ++acc_use[a];
            }
            sm100::mma_commit(&mma_done);  // every MMA of this CTA has completed
            sm100::mbar_wait(&mma_done, 0, WAIT_NS);
        }
    } else if (warp < 6) {
        // ---------------- dequantising producer of the W tiles ----------------
        const int pt = tid - 64;
        const int rt_l = pt >> 4, tp = (pt >> 3) & 1, g = pt & 7;
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < p.ntiles && !abort_flag; tile += gridDim.x) {
            const int rtile = tile / p.tiles_tok;
            const int rt = rtile * (BM / GLQ_ROW_TILE) + rt_l;
            const bool live = rt < p.RT;
            const size_t slot0 = (size_t)rt * p.KC * 32 + 4 * g + 2 * tp;
            StepCodes codes;
            StepWords words;
            load_codes<BPW>(p, slot0, 0, live, codes);
            issue_gathers<BPW>(p, codes, live, words);
            if (KB > 1) load_codes<BPW>(p, slot0, 1, live, codes);
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const uint32_t s = it % STAGES, use = it / STAGES;
                if (abort_flag || !sm100::mbar_wait(&empty_bar[s], (use & 1) ^ 1, WAIT_NS)) {
                    if (!abort_flag) fail();
                    break;
                }
                store_step<BPW>(p, words, smem + s * STAGE_BYTES, rt_l, tp, g);
                sm100::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&w_full[s]);
                if (kb + 1 < KB) issue_gathers<BPW>(p, codes, live, words);
                if (kb + 2 < KB) load_codes<BPW>(p, slot0, kb + 2, live, codes);
            }
        }
    } else {
        // ---------------- epilogue: TMEM -> z ----------------
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        uint32_t acc_use[NACC] = {0, 0};
        for (int tile = blockIdx.x; tile < p.ntiles && !abort_flag; tile += gridDim.x) {
            const int rtile = tile / p.tiles_tok, ttile = tile - rtile * p.tiles_tok;
            const int tok0 = ttile * (BN * NACC), na = live_acc(tok0);
            const int row = rtile * BM + 32 * q + lane;
            for (int a = 0; a < na; ++a) {
                if (abort_flag || !sm100::mbar_wait(&acc_full[a], acc_use[a] & 1, WAIT_NS)) {
                    if (!abort_flag) fail();
                    break;
                }
                sm100::tc_fence_after();
                for (int c = 0; c < BN / 16; ++c) {
                    uint32_t r[16];
                    sm100::tmem_ld16(tmem_base + ((uint32_t)(32 * q) << 16) + a * BN + c * 16, r);
                    sm100::tmem_wait_ld();
                    const int tb = tok0 + a * BN + c * 16;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int tok = tb + j;
                        if (tok < p.B && row < p.m_pad)
                            p.z[(size_t)tok * p.m_pad + row] = __uint_as_float(r[j]) * p.ws * p.info[tok].inv_scale;
                    }
                }
                sm100::tc_fence_before();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&acc_empty[a]);
                ++acc_use[a];
            }
        }
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
