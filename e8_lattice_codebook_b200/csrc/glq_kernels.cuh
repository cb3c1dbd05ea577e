// glq_kernels.cuh -- kernel parameter blocks and launchers of glq-b200.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "glq_device.cuh"
#include "glq_internal.h"

namespace glq {

struct RhtInParams {
    const void *x;  // [B][n] fp16 / bf16
    int x_bf16;
    int n, n_pad;
    int B;
    const uint32_t *sign_bits;  // bit k set: S_in[k] = -1
    glq_blocks blocks;
    __half *xr_h;          // [B][n_pad] scaled fp16 (product path) or null
    glq_rowinfo *info;     // [B] (product path) or null
    float *xr_f32;         // [B][n] unscaled fp32 (test entry point) or null
};

struct RhtOutParams {
    int m, m_pad, B;
    const float *partials;  // [splits][B][m_pad] (decode path) or null
    int splits;
    const float *z;         // [B][z_ld] fp32 (tensor path / test entry point) or null
    int z_ld;
    const glq_rowinfo *info;  // used with partials
    float ws;
    float corr_mult;
    const uint32_t *sign_bits;  // bit r set: S_out[r] = -1
    glq_blocks blocks;
    void *y;  // [B][m]
    int y_dtype;  // 0 f16, 1 bf16, 2 f32
};

struct GemvParams {
    const uint4 *idx1;     // [RT][KC][32] 16 B
    const void *idx2;      // [RT][KC][32] 16 B (4 bpw) / 8 B (3 bpw)
    const uint32_t *table; // folded nibble table (global), table_words (multiple of 4)
    int table_words;
    FoldParams fold;
    const uint4 *res8;     // 3 bpw: [256] x 8 fp16, columns 2,3,6,7 scaled by 16
    const __half *xr;      // [B][n_pad]
    int B, n_pad, KC, RT;
    int bands, splits, cps;
    float rs_acc;          // residual weight of acc2 in the partial sum: rs (4 bpw),
                           // rs * 2^-23 (3 bpw: acc2 holds unscaled fp16 products)
    float *partials;       // [splits][B][m_pad]
    int m_pad;
    unsigned *err;
};

struct DequantParams {
    const uint4 *idx1;
    const void *idx2;
    const uint32_t *table;
    FoldParams fold;
    const uint4 *res8;
    int bpw;
    int64_t m;
    int n, G, KC;
    float ws, rs;
    float *w;  // [m][n]
};

// cudaLaunchKernelExC with optional programmatic stream serialisation.
inline cudaError_t launch_ex(const void *fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             bool pdl, void **args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// Launchers (return cudaError_t of the launch).  `pdl` enables
// programmatic dependent launch on the stream.
cudaError_t launch_rht_in(const RhtInParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_rht_out(const RhtOutParams &p, cudaStream_t s, bool pdl);
cudaError_t launch_gemv(const GemvParams &p, int bpw, int grid, cudaStream_t s, bool pdl);
cudaError_t launch_dequant(const DequantParams &p, cudaStream_t s);

constexpr int GEMV_WARPS = 16;
constexpr int GEMV_PREFETCH = 4;
size_t gemv_smem_bytes(int table_words, int bpw);

}  // namespace glq
