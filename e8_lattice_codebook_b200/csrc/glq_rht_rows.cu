// glq_rht_rows.cu -- the input and output randomized Hadamard transforms of
// the tensor-core (many-token) path: xr = H_n (S_in x) and y = S_out (H_m z),
// H block-diagonal over the binary decomposition of the size, each block a
// Sylvester-ordered FWHT normalised by 1/sqrt(block) (glq 0.5.1 PyPI page,
// "How it works" 2 and "Bit widths": block-diagonal FHT for sizes that are
// not powers of two; GLQ v0.3.2 release notes, input_rht / output_rht).
//
// Design (B200): throughput over many rows, sizes up to 16384.  One CTA per
// row with one thread per 16 consecutive values:
//   * spans 1..8 run in registers, spans 16..256 as warp shuffles (lane bits
//     of the thread index), and the remaining spans of blocks above 512 values
//     as shared-memory rounds over the row (value-major, conflict-free), two
//     spans per round (radix 4), one barrier each;
//   * a block smaller than 16 values (only the last block, of 8) keeps its
//     thread's upper half as padding;
//   * the input direction also finds the row's max |xr| (one reduction) and
//     writes either the fp16 operand of the tensor-core GEMM, xr 2^e with
//     max |xr| 2^e < 2^14, or the decode GEMV's operand X = round(xr 2^e) as
//     high / low bytes with its exact row sum (a second reduction), plus 2^-e.
#include "glq_kernels.cuh"

namespace glq {

namespace {

constexpr int VPT = 16;  // values per thread

// block (offset, size) of the Hadamard decomposition containing column c
__device__ __forceinline__ int block_size_at(const RowsParams &p, int c, float *norm) {
    for (int i = 0; i < p.nblk; ++i)
        if (c >= p.blk_off[i] && c < p.blk_off[i] + p.blk_len[i]) {
            *norm = p.blk_norm[i];
            return p.blk_len[i];
        }
    *norm = 0.f;
    return 0;
}

__device__ __forceinline__ void load16_act(const void *x, size_t i, int bf16, int valid, float v[16]) {
    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + i);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint4 r = make_uint4(0, 0, 0, 0);
        if (8 * q < valid) r = ldg_nc_v4(src + q);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (bf16) {
                v[8 * q + 2 * j] = __uint_as_float(w[j] << 16);
                v[8 * q + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            } else {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[j]));
                v[8 * q + 2 * j] = f.x;
                v[8 * q + 2 * j + 1] = f.y;
            }
        }
    }
}

template <bool IN>
__global__ void __launch_bounds__(1024) rht_rows_kernel(RowsParams p) {
    extern __shared__ float srow[];  // the row, for spans above 256
    __shared__ float s_red[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;
    const int c0 = VPT * tid;  // first column of this thread
    pdl_launch_dependents();
    if (c0 < p.len) {  // warm L2 and the TLB before waiting on the producer
        if (IN) prefetch_l2(static_cast<const uint16_t *>(p.x) + (size_t)b * p.len + c0);
        else prefetch_l2(p.z + (size_t)b * p.z_ld + c0);  // the first split
    }
    pdl_wait();  // the input comes from the previous kernel

    float norm;
    const int bsz = c0 < p.len ? block_size_at(p, c0, &norm) : 0;
    const int valid = max(0, min(VPT, p.len - c0));  // 16, 8 (last block of 8) or 0
    float v[VPT];
    if (IN) {
        load16_act(p.x, (size_t)b * p.len + c0, p.x_bf16, valid, v);
        const uint32_t sb = valid ? (p.sign_bits[c0 >> 5] >> (c0 & 31)) & 0xFFFFu : 0u;
#pragma unroll
        for (int j = 0; j < VPT; ++j)
            if ((sb >> j) & 1u) v[j] = -v[j];
    } else {
#pragma unroll
        for (int j = 0; j < VPT; ++j) v[j] = 0.f;
        for (int sp = 0; sp < p.zsplits; ++sp) {  // K-split partial sums, in split order
            const float4 *src = reinterpret_cast<const float4 *>(p.z + sp * p.zs + (size_t)b * p.z_ld + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
                if (4 * q < valid) r = __ldcs(src + q);
                v[4 * q] += r.x;
                v[4 * q + 1] += r.y;
                v[4 * q + 2] += r.z;
                v[4 * q + 3] += r.w;
            }
        }
    }
    if (valid < VPT)
#pragma unroll
        for (int j = 8; j < VPT; ++j) v[j] = 0.f;  // padding past the row
    // spans 1, 2, 4, 8 in registers
#pragma unroll
    for (int h = 1; h < VPT; h <<= 1)
        if (h < bsz)
#pragma unroll
            for (int j = 0; j < VPT; ++j)
                if ((j & h) == 0) {
                    const float a = v[j], c = v[j + h];
                    v[j] = a + c;
                    v[j + h] = a - c;
                }
    // spans 16 .. 256: lane bits
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int off = 1 << k;
        const bool act = (VPT << k) < bsz;
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, v[j], off);
            if (act) v[j] = upper ? o - v[j] : v[j] + o;
        }
    }
    // spans 512 and up: shared memory rounds over the row, stored value-major
    // (value j of thread t at j * T + t) so that a warp's accesses are
    // consecutive words; column c = 16 t + j pairs with thread t + h / 16
    if (p.max_blk > 32 * VPT) {
        const int T = blockDim.x;
#pragma unroll
        for (int j = 0; j < VPT; ++j) srow[j * T + tid] = v[j];
        __syncthreads();
        int h = 32 * VPT;
        for (; 2 * h < p.max_blk; h <<= 2) {  // spans h and 2h in one round (radix 4)
            const int dt = h / VPT;
            if (2 * h < bsz && (tid & (3 * dt)) == 0) {  // this thread's columns are the first quarter
#pragma unroll 4
                for (int j = 0; j < VPT; ++j) {
                    float *r = srow + j * T + tid;
                    const float a = r[0], b = r[dt], c = r[2 * dt], d = r[3 * dt];
                    const float ab = a + b, amb = a - b, cd = c + d, cmd = c - d;
                    r[0] = ab + cd;
                    r[dt] = amb + cmd;
                    r[2 * dt] = ab - cd;
                    r[3 * dt] = amb - cmd;
                }
            } else if (h < bsz && 2 * h >= bsz && (tid & dt) == 0) {  // a block ending at span h
#pragma unroll 4
                for (int j = 0; j < VPT; ++j) {
                    float *r = srow + j * T + tid;
                    const float a = r[0], c = r[dt];
                    r[0] = a + c;
                    r[dt] = a - c;
                }
            }
            __syncthreads();
        }
        if (h < p.max_blk) {  // one span left
            const int dt = h / VPT;
            if (h < bsz && (tid & dt) == 0) {
#pragma unroll 4
                for (int j = 0; j < VPT; ++j) {
                    float *r = srow + j * T + tid;
                    const float a = r[0], c = r[dt];
                    r[0] = a + c;
                    r[dt] = a - c;
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int j = 0; j < VPT; ++j) v[j] = srow[j * T + tid];
    }
#pragma unroll
    for (int j = 0; j < VPT; ++j) v[j] *= norm;  // norm 0 past the row: padding stays 0

    if (IN) {
        float mx = 0.f;
#pragma unroll
        for (int j = 0; j < VPT; ++j) mx = fmaxf(mx, fabsf(v[j]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) s_red[warp] = mx;
        __syncthreads();
        float rowmax = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) rowmax = fmaxf(rowmax, s_red[w]);
        float scale = 1.f;
        if (rowmax > 0.f && isfinite(rowmax)) {
            int e;
            frexpf(rowmax, &e);  // rowmax < 2^e
            scale = ldexpf(1.f, 14 - e);
        }
        if (p.xq) {  // decode GEMV operand: X = round(xr 2^e), bytes per 8-column group
            int sum = 0;
            if (c0 < p.len_pad) {
                uint32_t hb[4] = {0u, 0u, 0u, 0u}, lb[4] = {0u, 0u, 0u, 0u};
                uint32_t hx[8];
#pragma unroll
                for (int j = 0; j < VPT; ++j) {
                    const int X = __float2int_rn(v[j] * scale);
                    sum += X;
                    hb[j >> 2] |= (uint32_t)((X >> 8) & 0xFF) << (8 * (j & 3));
                    lb[j >> 2] |= (uint32_t)(X & 0xFF) << (8 * (j & 3));
                    const __half hX = __int2half_rn(X);
                    if (j & 1) hx[j >> 1] |= (uint32_t)__half_as_ushort(hX) << 16;
                    else hx[j >> 1] = __half_as_ushort(hX);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(p.xq + ((size_t)b * p.len_pad + c0) * 2);
                dst[0] = make_uint4(hb[0], hb[1], lb[0], lb[1]);  // group c0 / 8
                dst[1] = make_uint4(hb[2], hb[3], lb[2], lb[3]);  // group c0 / 8 + 1
                if (p.xh) {
                    uint4 *dh = reinterpret_cast<uint4 *>(p.xh + (size_t)b * p.len_pad + c0);
                    dh[0] = make_uint4(hx[0], hx[1], hx[2], hx[3]);
                    dh[1] = make_uint4(hx[4], hx[5], hx[6], hx[7]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            __syncthreads();  // s_red is reused
            if (lane == 0) reinterpret_cast<int *>(s_red)[warp] = sum;
            __syncthreads();
            if (tid == 0) {
                long long total = 0;
                for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += reinterpret_cast<int *>(s_red)[w];
                p.info[b] = glq_rowinfo{total, 1.f / scale, 0.f};
            }
        } else {
            if (c0 < p.len_pad) {  // padding columns [len, len_pad) hold zeros
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const __half2 h2 = __floats2half2_rn(v[2 * j] * scale, v[2 * j + 1] * scale);
                    w[j] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(p.xh + (size_t)b * p.len_pad + c0);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
            if (tid == 0) p.info[b] = glq_rowinfo{0, 1.f / scale, 0.f};
        }
    } else if (valid) {
        const uint32_t sb = (p.sign_bits[c0 >> 5] >> (c0 & 31)) & 0xFFFFu;
#pragma unroll
        for (int j = 0; j < VPT; ++j)
            if ((sb >> j) & 1u) v[j] = -v[j];
        const size_t off = (size_t)b * p.len + c0;
        for (int q = 0; q < valid / 8; ++q) {
            const float *r = v + 8 * q;
            if (p.y_dtype == 2) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.y) + off + 8 * q);
                dst[0] = make_float4(r[0], r[1], r[2], r[3]);
                dst[1] = make_float4(r[4], r[5], r[6], r[7]);
            } else {
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (p.y_dtype == 1) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(r[2 * j], r[2 * j + 1]);
                        w[j] = *reinterpret_cast<const uint32_t *>(&h2);
                    } else {
                        const __half2 h2 = __floats2half2_rn(r[2 * j], r[2 * j + 1]);
                        w[j] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                }
                *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.y) + off + 8 * q) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
}

}  // namespace

bool rht_rows_supported(int len) { return len <= 32 * 32 * VPT && len >= 8; }

cudaError_t launch_rht_rows(const RowsParams &p, bool input, int B, cudaStream_t s, bool pdl) {
    const int cover = input ? p.len_pad : p.len;
    const int threads = ((cover + VPT - 1) / VPT + 31) / 32 * 32;
    if (threads > 1024 || B <= 0) return cudaErrorInvalidValue;
    // the row, one slot per thread's 16 columns (threads past the row included)
    const size_t smem = p.max_blk > 32 * VPT ? (size_t)threads * VPT * sizeof(float) : 0;
    const void *fn = input ? (const void *)rht_rows_kernel<true> : (const void *)rht_rows_kernel<false>;
    static bool configured[2] = {false, false};
    if (!configured[input ? 1 : 0]) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 1024 * VPT * 4);
        if (e != cudaSuccess) return e;
        configured[input ? 1 : 0] = true;
    }
    RowsParams q = p;
    void *args[] = {&q};
    return launch_ex(fn, dim3(B), dim3(threads), smem, s, pdl, args);
}

}  // namespace glq
