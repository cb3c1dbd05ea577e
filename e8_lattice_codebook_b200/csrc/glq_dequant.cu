// glq_dequant.cu -- explicit reconstruction of W^ (glq 0.5.1 PyPI page,
// "How it works" 1 and "Bit widths": a 16-bit E8 index per 8-weight group,
// an optional 8-bit / 16-bit residual stage, one global scale per layer).
// It reads the same device index streams and folded codebook as the GEMV
// and decodes with the same routines, then forms
//     w = fp32(ws * fma_f32(rs, cb2, cb1))
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
    float c1[8], c2[8];
    unpack_exact(table_word_global(p.table, code1, p.fold), c1);
    if (p.bpw == 4) {
        const uint32_t *w2 = reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint4 *>(p.idx2) + slot);
        uint32_t code2 = (w2[s] >> (16 * hi)) & 0xFFFFu;
        unpack_exact(table_word_global(p.table, code2, p.fold), c2);
    } else if (p.bpw == 3) {
        const uint8_t *b2 = reinterpret_cast<const uint8_t *>(reinterpret_cast<const uint2 *>(p.idx2) + slot);
        uint32_t i2 = b2[2 * s + hi];
        const __half *e = reinterpret_cast<const __half *>(p.res8 + i2);
#pragma unroll
        for (int j = 0; j < 8; ++j) c2[j] = __half2float(e[j]);
    }
    float *out = p.w + r * (int64_t)p.n + (int64_t)grp * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float c = c1[j];
        if (p.bpw > 2) c = __fmaf_rn(p.rs, c2[j], c);
        out[j] = __fmul_rn(p.ws, c);
    }
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
