// glq_dequant.cu -- explicit reconstruction of W^ (glq 0.5.1 PyPI page,
// "How it works" 1 and "Bit widths": a 16-bit E8 index per 8-weight group,
// then the residual stages of the bit width (16-bit E8 stages, an 8-bit
// stage last for an odd bpw), one global scale per layer).  It reads the
// same device index streams and folded codebook as the GEMV and decodes
// with the same routines, then forms, stage by stage in that order,
//     c = cb1;  c = fma_f32(rs_k, cb_k, c);  w = fp32(ws * c)
// with explicit round-to-nearest intrinsics (no contraction changes it).
#include "glq_kernels.cuh"

namespace glq {

namespace {

__global__ void dequant_kernel(DequantParams p) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= p.m * p.G) return;
    const int64_t r = gid / p.G;
    const int grp = (int)(gid - r * p.G);
    // fragment-native address of (row r, group grp)
    const int64_t rt = r / GLQ_ROW_TILE;
    const int rr = (int)(r % GLQ_ROW_TILE);
    const int kc = grp / GLQ_GROUPS_PER_CHUNK;
    const int s = (grp % GLQ_GROUPS_PER_CHUNK) / 4;
    const int t = grp % 4;
    const int lane = 4 * (rr & 7) + t;
    const int hi = rr >> 3;
    const size_t slot = ((size_t)rt * p.KC + kc) * 32 + lane;

    const uint32_t *w1 = reinterpret_cast<const uint32_t *>(p.idx1 + slot);
    uint32_t code1 = (w1[s] >> (16 * hi)) & 0xFFFFu;
    float c[8], cs[8];
    unpack_exact(table_word_global(p.table, code1, p.fold), c);
    // the residual stages in order: 16-bit E8 stages, then the 8-bit one
    const int n16 = stages16(p.bpw);
    for (int k = 0; k < n16; ++k) {
        const uint32_t *wk = reinterpret_cast<const uint32_t *>(p.idx16[k] + slot);
        unpack_exact(table_word_global(p.table, (wk[s] >> (16 * hi)) & 0xFFFFu, p.fold), cs);
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = __fmaf_rn(p.rs16[k], cs[j], c[j]);
    }
    if (stage8(p.bpw)) {
        const uint8_t *b8 = reinterpret_cast<const uint8_t *>(p.idx8 + slot);
        const __half *e = reinterpret_cast<const __half *>(p.tab8 + b8[2 * s + hi]);
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = __fmaf_rn(p.rs8, __half2float(e[j]), c[j]);
    }
    float *out = p.w + r * (int64_t)p.n + (int64_t)grp * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) out[j] = __fmul_rn(p.ws, c[j]);
}

}  // namespace

cudaError_t launch_dequant(const DequantParams &p, cudaStream_t s) {
    const int64_t total = p.m * p.G;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    dequant_kernel<<<(unsigned)blocks, threads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace glq
