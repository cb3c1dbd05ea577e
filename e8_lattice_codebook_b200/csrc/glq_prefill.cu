// glq_prefill.cu -- prefill (B > 16 tokens) GEMM of the GLQ linear layer on
// the 5th-generation tensor cores: z[b][r] = sum_k W^[r][k] xr[b][k]
// (glq 0.5.1 PyPI page, "Inference kernels": a tensor-core path for B >= 2
// that matmuls against codebook-reconstructed weights without materialising
// W in memory).
//
// Design (B200, sm_100a): persistent clusters of two CTAs (one per SM)
// share each tcgen05 MMA (cta_group::2, M = 256 = 128 rows per CTA,
// N = 256 tokens = 128 per CTA, K = 16), over output tiles of 256 weight rows
// x 512 tokens (two TMEM accumulators of 256 columns in each CTA; the tiles
// of a last partial wave as two half tiles of 256 tokens each), with a
// four-stage ring of 64-column steps (48 KB per CTA: its 128 rows of W and
// its 2 x 128 tokens of x):
//   * warp 0 of each CTA loads its half of the activations with TMA (128
//     tokens x 64 columns, fp16, 128-byte swizzle), completing on the first
//     CTA's barrier;
//   * warps 2-9 (dequantising producer) gather the fp16 codewords of the
//     CTA's 128 rows x 64 columns from the L2-resident table (16 bytes per
//     codeword, indexed by folded code), form c = cb1 + rs cb2 and write the
//     swizzled K-major A tile, then arrive on the first CTA's barrier; the
//     gathers of the next step and the code loads of the next chunk are in
//     flight while the current step is stored;
//   * warp 1 of the first CTA issues the pair's MMAs and commits to both
//     CTAs' barriers;
//   * warps 10-13 and 14-17 drain accumulators 0 and 1 with tcgen05.ld as
//     soon as the tile's last MMA completes and store z = acc ws 2^-e (fp32);
//     each accumulator is released on its own.  Items of one accumulator
//     (half tiles) alternate between the two, so that one is drained while
//     the next item's MMAs fill the other.
// Every wait is bounded (4e9 SM clock cycles, about 2 s); a timeout sets the
// layer's error flag, lets in-flight TMA loads and MMAs land, frees TMEM and
// returns.
#include <cmath>

#include "glq_kernels.cuh"
#include "glq_sm100.cuh"

namespace glq {

namespace {

constexpr int BM = 128;        // weight rows per CTA (the pair's MMA has M = 256)
constexpr int BN = 256;        // tokens per accumulator (the pair's MMA has N = 256)
constexpr int BNH = BN / 2;    // tokens per accumulator loaded by one CTA
constexpr int NACC = 2;        // accumulators per tile (512 tokens)
constexpr int BK = 64;         // columns per stage (one 128-byte swizzle row of fp16)
constexpr int STAGES = 4;
constexpr int W_BYTES = BM * BK * 2;                       // 16 KB
constexpr int X_BYTES = BNH * BK * 2;                      // 16 KB per accumulator
constexpr int STAGE_BYTES = W_BYTES + NACC * X_BYTES;     // 48 KB
constexpr int PRODUCER_WARPS = 8;                         // fused variant only
constexpr int EPI_WARPS = 8;                               // four per accumulator
// warp roles: 0 TMA, 1 MMA, [2-9 dequantising producer,] then the epilogue
__host__ __device__ constexpr int epi_warp0(bool mat) { return mat ? 2 : 2 + PRODUCER_WARPS; }
__host__ __device__ constexpr int threads_of(bool mat) { return (epi_warp0(mat) + EPI_WARPS) * 32; }  // 320 / 576
constexpr uint64_t WAIT_CYCLES = 4000000000ull;           // wait limit: 4e9 SM cycles (about 2 s)

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t s, uint32_t b, uint32_t a) {  // s * b + a
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(s), "r"(b), "r"(a));
    return r;
}

__device__ __forceinline__ uint4 hfma8(uint32_t rs2, uint4 b, uint4 a) {  // rs * b + a, 8 lanes
    return make_uint4(hfma2_bits(rs2, b.x, a.x), hfma2_bits(rs2, b.y, a.y), hfma2_bits(rs2, b.z, a.z),
                      hfma2_bits(rs2, b.w, a.w));
}

// MAT: W was dequantised into an fp16 matrix first; both operands are
// loaded by TMA and there is no producer.  Otherwise the producer warps
// rebuild each W step from the codes.
template <int BPW, bool MAT>
__global__ void __launch_bounds__(threads_of(MAT), 1) prefill_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                      const __grid_constant__ CUtensorMap wmap,
                                                                      PrefillParams p) {
    constexpr int EPI_WARP0 = epi_warp0(MAT);
    extern __shared__ uint8_t smem_raw[];
    // (first CTA) x_full: both CTAs' TMA bytes landed; w_full: both CTAs'
    // producer warps wrote W; acc_empty: both CTAs drained accumulator a.
    // (both CTAs) empty: the pair's MMAs of the stage finished; acc_full:
    // accumulator a computed (commits reach both CTAs).
    __shared__ __align__(8) uint64_t x_full[STAGES], w_full[STAGES], empty_bar[STAGES], acc_full[NACC],
        acc_empty[NACC], mma_done;
    __shared__ uint32_t tmem_holder;
    __shared__ volatile int abort_flag;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = sm100::cluster_ctarank();
    uint32_t cid, ncl;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(cid));
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(ncl));

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&x_full[s], 1);                   // the first CTA's TMA thread
            mbar_init(&w_full[s], MAT ? 1 : 2 * PRODUCER_WARPS);  // producer warps of both CTAs
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 2 * (EPI_WARPS / NACC));
        }
        mbar_init(&mma_done, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        sm100::prefetch_tensormap(&xmap);
        if (MAT) sm100::prefetch_tensormap(&wmap);
    }
    if (warp == 1) {
        sm100::tmem_alloc2(&tmem_holder, 512);
        sm100::tmem_relinquish2();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
    sm100::tc_fence_after();
    const uint32_t tmem_base = tmem_holder;
    pdl_launch_dependents();

    auto fail = [&]() {
        atomicOr(p.err, GLQ_DEVERR_TIMEOUT);
        abort_flag = 1;
    };
    auto live_acc = [&](int tok0) { return min(NACC, (p.B - tok0 + BN - 1) / BN); };
    // The first accumulator of an item: an item with one live accumulator (a
    // half tile, or a tile whose second 256 tokens are past the batch) takes
    // the two in turn, counted by the CTA's earlier such items, so its MMAs
    // run while the epilogue drains the previous one; a whole tile uses both.
    auto acc_first = [](int na, uint32_t singles) { return na == 1 ? (int)(singles & 1u) : 0; };
    // work item -> (weight-row tile, first token, live accumulators, K split)
    // and its 64-column steps [kb0, kb1) (splits on 128-column chunk
    // boundaries).  Items below tiles_whole are whole tiles; the rest are the
    // halves (256 tokens, one accumulator) of the tiles that follow, so that
    // a last partial wave of whole tiles takes half a tile's time.
    auto geom = [&](int item, int &rtile, int &tok0, int &na, int &ks, int &kb0, int &kb1) {
        int tile = item, half = -1;
        if (item >= p.tiles_whole) {
            const int u = item - p.tiles_whole;
            tile = p.tiles_whole + (u >> 1);
            half = u & 1;
        }
        ks = tile % p.ksplit;
        const int rest = tile / p.ksplit;
        rtile = rest / p.tiles_tok;
        const int ttile = rest - rtile * p.tiles_tok;
        tok0 = ttile * (BN * NACC) + (half > 0 ? BN : 0);
        na = half < 0 ? live_acc(tok0) : min(1, live_acc(tok0));
        kb0 = 2 * ((ks * p.KC) / p.ksplit);
        kb1 = 2 * (((ks + 1) * p.KC) / p.ksplit);
    };

    if (warp == 0) {
        // ---------------- TMA: this CTA's half of the activation tiles ----------------
        pdl_wait();  // the activations come from the input RHT
        if (lane == 0) {
            uint32_t it = 0;
            int32_t last_load = -1;
            for (int tile = (int)cid; tile < p.ntiles && !abort_flag; tile += (int)ncl) {
                int rtile, tok0, na, ks, kb0, kb1;
                geom(tile, rtile, tok0, na, ks, kb0, kb1);
                int halves = 0;  // live halves of both CTAs (a half past the last token is not loaded)
                for (int a = 0; a < na; ++a)
                    for (int r = 0; r < 2; ++r) halves += tok0 + a * BN + r * BNH < p.B;
                for (int kb = kb0; kb < kb1 && !abort_flag; ++kb, ++it) {
                    const uint32_t s = it % STAGES, use = it / STAGES;
                    if (!sm100::mbar_wait_cluster(&empty_bar[s], (use & 1) ^ 1, WAIT_CYCLES)) {
                        fail();
                        break;
                    }
                    const int wrow = rtile * (2 * BM);  // the pair's first weight row
                    const int wparts = MAT ? (wrow < p.m_pad) + (wrow + BM < p.m_pad) : 0;
                    if (rank == 0) mbar_expect_tx(&x_full[s], (uint32_t)(halves * X_BYTES + wparts * W_BYTES));
                    if (MAT && wrow + (int)rank * BM < p.m_pad)  // rows past m_pad are never stored
                        sm100::tma_load_2d_pair(smem + s * STAGE_BYTES, &wmap, &x_full[s], kb * BK,
                                                wrow + (int)rank * BM);
                    for (int a = 0; a < na; ++a) {
                        const int t0 = tok0 + a * BN + (int)rank * BNH;
                        if (t0 < p.B)
                            sm100::tma_load_2d_pair(smem + s * STAGE_BYTES + W_BYTES + a * X_BYTES, &xmap,
                                                    &x_full[s], kb * BK, t0);
                    }
                    last_load = (int32_t)it;
                }
            }
            if (abort_flag && rank == 0)  // let the copies in flight land before the CTA exits
                for (int32_t i = max(0, last_load - (STAGES - 1)); i <= last_load; ++i)
                    sm100::mbar_wait(&x_full[i % STAGES], (uint32_t)(i / STAGES) & 1, WAIT_CYCLES);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer of the pair ----------------
            const uint32_t idesc = sm100::idesc_f16_f32(2 * BM, BN);
            uint32_t it = 0, acc_use[NACC] = {0, 0}, singles = 0;
            for (int tile = (int)cid; tile < p.ntiles && !abort_flag; tile += (int)ncl) {
                int rtile, tok0, na, ks, kb0, kb1;
                geom(tile, rtile, tok0, na, ks, kb0, kb1);
                const int abase = acc_first(na, singles);
                for (int kb = kb0; kb < kb1 && !abort_flag; ++kb, ++it) {
                    const uint32_t s = it % STAGES, use = it / STAGES;
                    if (!sm100::mbar_wait_cluster(&x_full[s], use & 1, WAIT_CYCLES) ||
                        (!MAT && !sm100::mbar_wait_cluster(&w_full[s], use & 1, WAIT_CYCLES))) {
                        fail();
                        break;
                    }
                    sm100::tc_fence_after();
                    uint8_t *st = smem + s * STAGE_BYTES;
                    const uint64_t adesc = sm100::smem_desc_sw128(st);
                    for (int a = 0; a < na; ++a) {  // x slot a of the stage into accumulator abase + a
                        const int ac = abase + a;
                        if (kb == kb0) {  // both CTAs' epilogues must have drained this accumulator
                            if (!sm100::mbar_wait_cluster(&acc_empty[ac], (acc_use[ac] & 1) ^ 1, WAIT_CYCLES)) {
                                fail();
                                break;
                            }
                            sm100::tc_fence_after();
                        }
                        const uint64_t bdesc = sm100::smem_desc_sw128(st + W_BYTES + a * X_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            sm100::mma2_f16_ss(tmem_base + ac * BN, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                               (kb != kb0) || (kk != 0));
                        if (kb == kb1 - 1) sm100::mma2_commit_both(&acc_full[ac]);
                    }
                    sm100::mma2_commit_both(&empty_bar[s]);
                }
                for (int a = 0; a < na; ++a) ++acc_use[abase + a];
                singles += na == 1;
            }
            sm100::mma2_commit_both(&mma_done);  // every MMA of the pair has completed
            sm100::mbar_wait(&mma_done, 0, WAIT_CYCLES);
        } else if (lane == 0) {
            sm100::mbar_wait(&mma_done, 0, WAIT_CYCLES);  // the pair's last commit reaches both CTAs
        }
    } else if (!MAT && warp < EPI_WARP0) {
        // ---------------- dequantising producer of the W tiles ----------------
        // warp: 16-row tile rt_l of the CTA's 128 rows; lane (g, t) = slot lane
        // 4 g + t of the fragment-native stream: in 64-column step h of a
        // chunk, words s = 2h, 2h + 1 hold rows (g, g + 8) of groups 4 s + t,
        // i.e. groups t and 4 + t of the step.  Codeword i = 2 s2 + hi.
        const int rt_l = warp - 2;
        const int g = lane >> 2, t = lane & 3;
        uint32_t it = 0;
        for (int tile = (int)cid; tile < p.ntiles && !abort_flag; tile += (int)ncl) {
            int rtile, tok0, na, ks, kb0, kb1;
            geom(tile, rtile, tok0, na, ks, kb0, kb1);
            const int rt = (rtile * 2 + (int)rank) * (BM / GLQ_ROW_TILE) + rt_l;
            const bool live = rt < p.RT;
            const size_t slot0 = (size_t)rt * p.KC * 32 + lane;
            uint4 q1 = make_uint4(0, 0, 0, 0), q2 = q1, n1 = q1, n2 = q1;
            auto load_slot = [&](int kc, uint4 &a1, uint4 &a2) {
                if (!live || kc >= p.KC) return;
                a1 = ldg_nc_v4(p.idx1 + slot0 + (size_t)kc * 32);
                if (BPW == 4) a2 = ldg_nc_v4(p.idx16[0] + slot0 + (size_t)kc * 32);
                if (BPW == 3) {
                    const uint2 v = ldg_nc_v2(p.idx8 + slot0 + (size_t)kc * 32);
                    a2 = make_uint4(v.x, v.y, 0, 0);
                }
            };
            // gathers of step kb's 4 codewords (primary and residual)
            uint4 ca[4], cb[4];
            auto gather = [&](int kb) {
                const int h = kb & 1;
                const uint32_t wa = h ? q1.z : q1.x, wb = h ? q1.w : q1.y;
                const uint32_t e1[4] = {wa & 0xFFFFu, wa >> 16, wb & 0xFFFFu, wb >> 16};
#pragma unroll
                for (int i = 0; i < 4; ++i) ca[i] = live ? __ldg(p.cb_f16 + e1[i]) : make_uint4(0, 0, 0, 0);
                if (BPW == 4) {
                    const uint32_t va = h ? q2.z : q2.x, vb = h ? q2.w : q2.y;
                    const uint32_t e2[4] = {va & 0xFFFFu, va >> 16, vb & 0xFFFFu, vb >> 16};
#pragma unroll
                    for (int i = 0; i < 4; ++i) cb[i] = live ? __ldg(p.cb_f16 + e2[i]) : make_uint4(0, 0, 0, 0);
                } else if (BPW == 3) {  // bytes 2 s + hi of the 8-byte slot, s = 2h, 2h + 1
                    const uint32_t w = h ? q2.y : q2.x;
#pragma unroll
                    for (int i = 0; i < 4; ++i) cb[i] = live ? __ldg(p.tab8 + ((w >> (8 * i)) & 0xFFu)) : make_uint4(0, 0, 0, 0);
                }
            };
            load_slot(kb0 >> 1, q1, q2);
            load_slot((kb0 >> 1) + 1, n1, n2);
            gather(kb0);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                uint4 cw[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    cw[i] = BPW == 2 ? ca[i] : hfma8(BPW == 4 ? p.rs16_h2[0] : p.rs8_h2, cb[i], ca[i]);
                if (kb + 1 < kb1) {  // the next step's gathers are in flight while this one is stored
                    if (((kb + 1) & 1) == 0) {
                        q1 = n1;
                        q2 = n2;
                        load_slot(((kb + 1) >> 1) + 1, n1, n2);  // codes one chunk ahead
                    }
                    gather(kb + 1);
                }
                const uint32_t s = it % STAGES, use = it / STAGES;
                if (abort_flag || !sm100::mbar_wait_cluster(&empty_bar[s], (use & 1) ^ 1, WAIT_CYCLES)) {
                    if (!abort_flag) fail();
                    break;
                }
                uint8_t *wt = smem + s * STAGE_BYTES;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int hi = i & 1, s2 = i >> 1;
                    const int row = rt_l * GLQ_ROW_TILE + g + 8 * hi;
                    const int gl = 4 * s2 + t;
                    *reinterpret_cast<uint4 *>(wt + row * 128 + ((gl ^ (row & 7)) << 4)) = cw[i];
                }
                sm100::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0) sm100::mbar_arrive(&w_full[s]);
                    else sm100::mbar_arrive_remote(&w_full[s], 0);
                }
            }
        }
    } else {
        // ---------------- epilogue: TMEM -> z ----------------
        pdl_wait();  // the row info comes from the input RHT
        const int ew = warp - EPI_WARP0;   // 0..7
        const int q = warp & 3;            // TMEM lane quadrant this warp may access
        const int a = ew >> 2;             // the accumulator this warp drains
        uint32_t use = 0, singles = 0;
        for (int tile = (int)cid; tile < p.ntiles && !abort_flag; tile += (int)ncl) {
            int rtile, tok0, na, ks, kb0, kb1;
            geom(tile, rtile, tok0, na, ks, kb0, kb1);
            float *zk = p.z + (size_t)ks * p.zs;  // this split's partial sums
            const int abase = acc_first(na, singles);
            singles += na == 1;
            if (a < abase || a >= abase + na) continue;  // accumulator a is idle in this item
            const int tb = tok0 + (a - abase) * BN;
            const int row = (rtile * 2 + (int)rank) * BM + 32 * q + lane;
            if (abort_flag || !sm100::mbar_wait_cluster(&acc_full[a], use & 1, WAIT_CYCLES)) {
                if (!abort_flag) fail();
                break;
            }
            sm100::tc_fence_after();
            const int nlive = min(BN, p.B - tb);
            for (int c = 0; c < nlive; c += 32) {
                uint32_t r[32];
                sm100::tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + a * BN + c, r);
                // lane j holds ws 2^-e of token c + j; the warp shares it by shuffles
                const float sc = c + lane < nlive ? p.ws * p.info[tb + c + lane].inv_scale : 0.f;
                sm100::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float scj = __shfl_sync(0xffffffffu, sc, j);
                    if (row < p.m_pad && c + j < nlive)
                        zk[(size_t)(tb + c + j) * p.m_pad + row] = __uint_as_float(r[j]) * scj;
                }
            }
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) sm100::mbar_arrive(&acc_empty[a]);
                else sm100::mbar_arrive_remote(&acc_empty[a], 0);
            }
            ++use;
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::cluster_sync_all();  // no CTA leaves while its pair may still touch its memory
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc2(tmem_base, 512);
    }
}

}  // namespace

size_t prefill_smem_bytes() { return 1024 + (size_t)STAGES * STAGE_BYTES; }

int prefill_tile_tokens() { return BN * NACC; }

int prefill_tile_rows() { return 2 * BM; }

PrefillSplit plan_prefill(int64_t m_pad, int KC, int64_t B, int num_sms) {
    PrefillSplit ps{};
    const int tr = prefill_tile_rows(), tt = prefill_tile_tokens();
    const int pairs = num_sms / 2 > 1 ? num_sms / 2 : 1;
    const int tiles_m = (int)((m_pad + tr - 1) / tr);
    ps.tiles_tok = (int)((B + tt - 1) / tt);
    const int tiles = tiles_m * ps.tiles_tok;
    // K splits: fill the CTA pairs when the output has too few tiles, unless
    // the extra partial-sum traffic costs more than it saves.  Model (B200
    // measurements): a pair retires a tile's rows x tokens x K x 2 FLOP at
    // about 15 TFLOP/s; each extra split writes and reads B x m_pad fp32 at
    // about 6 TB/s.
    const double t_tile = (double)tr * (double)tt * (double)KC * GLQ_CHUNK_K * 2.0 / 15e12;
    const double t_traffic = (double)B * (double)m_pad * 8.0 / 6e12;
    ps.ksplit = 1;
    double best_t = 1e30;
    for (int S = 1; S <= 8 && S <= KC / 4 + (S == 1); ++S) {
        const double waves = std::ceil((double)tiles * S / pairs);
        const double t = waves * t_tile / S + (S - 1) * t_traffic;
        if (t < best_t * 0.97) {  // a split must pay for itself clearly
            best_t = t;
            ps.ksplit = S;
        }
    }
    ps.ntiles = tiles * ps.ksplit;
    ps.tiles_whole = ps.ntiles;
    // A last partial wave of whole tiles (one per CTA pair) runs as half
    // tiles of 256 tokens, twice as many items taking half the time: when it
    // has at most half a wave of tiles, and every tile has two live halves
    // (the last token tile holds more than 256 tokens).
    const int rest = ps.ntiles % pairs;
    if (ps.ksplit == 1 && ps.ntiles > pairs && rest > 0 && 2 * rest <= pairs && (B % tt == 0 || B % tt > tt / 2)) {
        ps.tiles_whole = ps.ntiles - rest;
        ps.ntiles = ps.tiles_whole + 2 * rest;
    }
    return ps;
}

cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &xmap, const CUtensorMap *wmap, int grid,
                           cudaStream_t s, bool pdl) {
    const size_t smem = prefill_smem_bytes();
    const bool mat = wmap != nullptr;
    const void *fn;
    // the kernel with W reconstructed does not depend on the bit width;
    // the dequantising producer exists for 2-4 bpw (two stages at most)
    switch ((mat ? 4 : p.bpw) * 2 + (mat ? 1 : 0)) {
        case 4: fn = (const void *)prefill_kernel<2, false>; break;
        case 6: fn = (const void *)prefill_kernel<3, false>; break;
        case 8: fn = (const void *)prefill_kernel<4, false>; break;
        case 9: fn = (const void *)prefill_kernel<4, true>; break;
        default: return cudaErrorInvalidValue;
    }
    static std::atomic<uint64_t> configured[10];  // per variant: devices set
    const int key = (mat ? 4 : p.bpw) * 2 + (mat ? 1 : 0);
    const cudaError_t e = once_per_device(configured[key], [fn] {
        return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMV_SMEM_LIMIT);
    });
    if (e != cudaSuccess) return e;
    if (smem > GEMV_SMEM_LIMIT || (grid & 1)) return cudaErrorInvalidValue;
    PrefillParams q = p;
    CUtensorMap m = xmap;
    CUtensorMap wm = mat ? *wmap : xmap;  // unused by the fused variant
    void *args[] = {&m, &wm, &q};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads_of(mat));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace glq
