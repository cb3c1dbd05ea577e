// glq_shard.cu -- the two small kernels of a row-parallel shard of the GLQ
// linear layer (a layer split over its input columns, each part's fp32
// partial output summed across GPUs by one all-reduce).
//
// The decode GEMV's exact finish turns sum v X into sum x X with the row sum
// of X (x = v/2 - 3 per codeword nibble): a shard needs that sum over its own
// columns, which shard_rowsum_kernel forms from the quantised activations the
// input transform wrote for the whole row.  cast_kernel rounds the summed
// fp32 output to the caller's dtype.
#include "glq_kernels.cuh"

namespace glq {

namespace {

constexpr int SUM_THREADS = 256;

__global__ void __launch_bounds__(SUM_THREADS) shard_rowsum_kernel(const uint8_t *xq, size_t row_bytes, int c0,
                                                                   int c1, const glq_rowinfo *in,
                                                                   glq_rowinfo *out) {
    __shared__ long long s_part[SUM_THREADS / 32];
    pdl_launch_dependents();
    pdl_wait();  // xq and the row info come from the input transform
    const int b = blockIdx.x;
    const uint8_t *row = xq + (size_t)b * row_bytes;
    long long sum = 0;
    for (int k = c0 + (int)threadIdx.x; k < c1; k += SUM_THREADS) {
        const int grp = k >> 3, j = k & 7;  // per group of 8 columns: 8 high bytes, then 8 low bytes
        sum += (long long)((int)(int8_t)row[grp * 16 + j] * 256 + (int)row[grp * 16 + 8 + j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long t = 0;
        for (int w = 0; w < SUM_THREADS / 32; ++w) t += s_part[w];  // fixed order
        out[b] = glq_rowinfo{t, in[b].inv_scale, 0.f};
    }
}

__global__ void cast_kernel(const float *src, void *dst, int dtype, int64_t count) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = src[i];
        if (dtype == 1) static_cast<__nv_bfloat16 *>(dst)[i] = __float2bfloat16_rn(v);
        else if (dtype == 0) static_cast<__half *>(dst)[i] = __float2half_rn(v);
        else static_cast<float *>(dst)[i] = v;
    }
}

}  // namespace

cudaError_t launch_shard_rowsum(const uint8_t *xq, size_t row_bytes, int c0, int c1, const glq_rowinfo *in,
                                glq_rowinfo *out, int B, cudaStream_t s, bool pdl) {
    if (B <= 0) return cudaSuccess;
    const void *fn = (const void *)shard_rowsum_kernel;
    void *args[] = {&xq, &row_bytes, &c0, &c1, &in, &out};
    return launch_ex(fn, dim3(B), dim3(SUM_THREADS), 0, s, pdl, args);
}

cudaError_t launch_cast(const float *src, void *dst, int dtype, int64_t count, cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((count + threads - 1) / threads, 148 * 8);
    cast_kernel<<<(unsigned)blocks, threads, 0, s>>>(src, dst, dtype, count);
    return cudaGetLastError();
}

}  // namespace glq
