// glq_wmat.cu -- the weights of a layer reconstructed once into an fp16
// matrix W16[m_pad][n_pad] = cb1 + rs_1 cb_1 + rs_2 cb_2 + ... (every
// residual stage in order, one fp16 fma each; the per-layer scale ws is
// applied in the GEMM epilogue), for the tensor-core path at large batches
// (glq 0.5.1 PyPI page, "How it works" 1 and 4, "Bit widths"; the pages'
// kernels never materialise W -- see the layer API for when this path runs).
//
// Design (B200): persistent CTAs, each holding the negation-folded nibble
// codebook (148 KB) in shared memory, so a codeword is one shared-memory load,
// a fold fix-up, and four byte permutes plus four fp16 FMAs: the nibble v
// becomes the fp16 1024 + v, and (1024 + v) / 2 - 515 = v/2 - 3 exactly.  A
// warp takes one (16-row tile, 128-column chunk) of the fragment-native index
// stream at a time: 512 coalesced bytes of codes per stream, 4 KB of W16
// out; the codes of its next item are already in flight meanwhile (16 warps
// per SM, so that enough loads are outstanding to cover the DRAM latency).
#include "glq_kernels.cuh"

namespace glq {

namespace {

constexpr int WARPS = 16;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t s, uint32_t b, uint32_t a) {  // s * b + a
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(s), "r"(b), "r"(a));
    return r;
}

constexpr uint32_t H2_HALF = 0x38003800u;  // (0.5, 0.5)
constexpr uint32_t H2_M515 = 0xE006E006u;  // (-515, -515)

// x = v/2 - 3 of the 8 nibbles of a table word (x0..x3 in the low nibbles of
// bytes 0..3, x4..x7 in the high nibbles), as 8 fp16 in coordinate order.
__device__ __forceinline__ uint4 expand_word(uint32_t w) {
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    const uint32_t K = 0x64646464u;
    return make_uint4(hfma2_bits(prmt(lo, K, 0x4140u), H2_HALF, H2_M515),
                      hfma2_bits(prmt(lo, K, 0x4342u), H2_HALF, H2_M515),
                      hfma2_bits(prmt(hi, K, 0x4140u), H2_HALF, H2_M515),
                      hfma2_bits(prmt(hi, K, 0x4342u), H2_HALF, H2_M515));
}

__device__ __forceinline__ uint4 hfma8(uint32_t rs2, uint4 b, uint4 a) {  // rs * b + a
    return make_uint4(hfma2_bits(rs2, b.x, a.x), hfma2_bits(rs2, b.y, a.y), hfma2_bits(rs2, b.z, a.z),
                      hfma2_bits(rs2, b.w, a.w));
}

__device__ __forceinline__ uint32_t fold_word(const uint32_t *T, uint32_t e, FoldParams f) {
    const bool neg = e >= (uint32_t)f.nb;
    const uint32_t w = T[neg ? e - (uint32_t)f.neg_base : e];
    return neg ? 0xCCCCCCCCu - w : w;
}

template <int BPW>
__global__ void __launch_bounds__(WARPS * 32, 1) wmat_kernel(PrefillParams p, __half *w16, int n_pad) {
    extern __shared__ __align__(16) uint32_t T[];
    __shared__ __align__(8) uint64_t bar;
    const uint4 *R8 = reinterpret_cast<const uint4 *>(T + p.table_words);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    if (tid == 0) mbar_init(&bar, 1);
    __syncthreads();
    if (tid == 0) {
        const uint32_t tbytes = (uint32_t)p.table_words * 4u, rbytes = Stages<BPW>::U8 ? 256u * 16u : 0u;
        mbar_expect_tx(&bar, tbytes + rbytes);
        for (uint32_t off = 0; off < tbytes; off += 32768u) {
            const uint32_t len = tbytes - off < 32768u ? tbytes - off : 32768u;
            bulk_g2s(reinterpret_cast<char *>(T) + off, reinterpret_cast<const char *>(p.table) + off, len, &bar);
        }
        if (Stages<BPW>::U8) bulk_g2s(const_cast<uint4 *>(R8), p.tab8, rbytes, &bar);
    }
    pdl_launch_dependents();
    const bool ok = __syncthreads_and(mbar_wait_bounded(&bar, 0, 1u << 24) ? 1 : 0) != 0;
    if (!ok) {
        if (tid == 0) atomicOr(p.err, GLQ_DEVERR_TIMEOUT);
        mbar_wait_bounded(&bar, 0, 1u << 24);  // let the copy land before exiting
        return;
    }
    pdl_wait();  // the previous user of w16 (the GEMM of an earlier call) has finished
    const long long items = (long long)p.RT * p.KC;
    const long long stride = (long long)gridDim.x * WARPS;
    constexpr int N16 = Stages<BPW>::N16, NA = Stages<BPW>::NA;
    auto load_codes = [&](long long it, uint4 &a1, uint4 (&ar)[NA], uint2 &a8) {
        const size_t slot = it * 32 + lane;  // [RT][KC][32]
        a1 = ldg_nc_v4(p.idx1 + slot);
#pragma unroll
        for (int k = 0; k < N16; ++k) ar[k] = ldg_nc_v4(p.idx16[k] + slot);
        if (Stages<BPW>::U8) a8 = ldg_nc_v2(p.idx8 + slot);
    };
    long long it = (long long)blockIdx.x * WARPS + warp;
    // the codes of the warp's next item
    uint4 n1 = make_uint4(0, 0, 0, 0), nr[NA];
    uint2 n8 = make_uint2(0, 0);
#pragma unroll
    for (int k = 0; k < NA; ++k) nr[k] = n1;
    if (it < items) load_codes(it, n1, nr, n8);
    for (; it < items; it += stride) {
        uint4 q1 = n1, qr[NA];
        const uint2 q8 = n8;
#pragma unroll
        for (int k = 0; k < NA; ++k) qr[k] = nr[k];
        if (it + stride < items) load_codes(it + stride, n1, nr, n8);
        const int rt = (int)(it / p.KC), kc = (int)(it - (long long)rt * p.KC);
        const uint32_t c1[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                uint4 cw = expand_word(fold_word(T, hi ? (c1[s] >> 16) : (c1[s] & 0xFFFFu), p.fold));
#pragma unroll
                for (int k = 0; k < N16; ++k) {  // the 16-bit stages in order
                    const uint32_t ck[4] = {qr[k].x, qr[k].y, qr[k].z, qr[k].w};
                    cw = hfma8(p.rs16_h2[k], expand_word(fold_word(T, hi ? (ck[s] >> 16) : (ck[s] & 0xFFFFu), p.fold)),
                               cw);
                }
                if (Stages<BPW>::U8) {  // the 8-bit stage last: byte 2 s + hi of the 8-byte slot
                    const uint32_t i2 = ((s < 2 ? q8.x : q8.y) >> (8 * (2 * (s & 1) + hi))) & 0xFFu;
                    cw = hfma8(p.rs8_h2, R8[i2], cw);
                }
                const int row = rt * GLQ_ROW_TILE + g + 8 * hi;
                const int col = kc * GLQ_CHUNK_K + 8 * (4 * s + t);
                *reinterpret_cast<uint4 *>(w16 + (size_t)row * n_pad + col) = cw;
            }
    }
}

}  // namespace

size_t wmat_smem_bytes(int table_words, int bpw) { return (size_t)table_words * 4 + (stage8(bpw) ? 256 * 16 : 0); }

cudaError_t launch_wmat(const PrefillParams &p, __half *w16, int n_pad, int num_sms, cudaStream_t s, bool pdl) {
    const void *fn = nullptr;
    switch (p.bpw) {
        case 2: fn = (const void *)wmat_kernel<2>; break;
        case 3: fn = (const void *)wmat_kernel<3>; break;
        case 4: fn = (const void *)wmat_kernel<4>; break;
        case 5: fn = (const void *)wmat_kernel<5>; break;
        case 6: fn = (const void *)wmat_kernel<6>; break;
        case 7: fn = (const void *)wmat_kernel<7>; break;
        case 8: fn = (const void *)wmat_kernel<8>; break;
        default: return cudaErrorInvalidValue;
    }
    static std::atomic<uint64_t> configured[9];  // per bit width: devices set
    const cudaError_t e = once_per_device(configured[p.bpw], [fn] {
        return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)wmat_smem_bytes(GLQ_TABLE_MAX_WORDS, 3));
    });
    if (e != cudaSuccess) return e;
    const long long items = (long long)p.RT * p.KC;
    const int grid = (int)std::min<long long>(num_sms, (items + WARPS - 1) / WARPS);
    PrefillParams q = p;
    __half *w = w16;
    int np = n_pad;
    void *args[] = {&q, &w, &np};
    return launch_ex(fn, dim3(grid), dim3(WARPS * 32), wmat_smem_bytes(p.table_words, p.bpw), s, pdl, args);
}

}  // namespace glq
