// glq_rht.cu -- the two Randomized Hadamard Transform stages of the GLQ
// linear layer (glq 0.5.1 PyPI page, "How it works" 2: random sign flips
// followed by a fast Walsh-Hadamard transform; "Bit widths": block-diagonal
// transform over the binary decomposition of a size that is not a power of
// two; GLQ v0.3.2 release notes: input_rht / output_rht ops).
//
// One CTA per token row; the row lives in shared memory as fp32 (up to
// 32,768 values = 128 KB) and every block of the decomposition is
// transformed in place with radix-2 butterflies.
#include "glq_kernels.cuh"

namespace glq {

namespace {

constexpr int RHT_THREADS = 1024;

__device__ __forceinline__ float load_act(const void *x, size_t i, int bf16) {
    uint16_t bits = reinterpret_cast<const uint16_t *>(x)[i];
    if (bf16) return __uint_as_float((uint32_t)bits << 16);
    return __half2float(__ushort_as_half(bits));
}

__device__ __forceinline__ bool sign_neg(const uint32_t *bits, int k) {
    return (bits[k >> 5] >> (k & 31)) & 1u;
}

// In-place unnormalised Walsh-Hadamard transform of a[0..K) (K a power of
// two, Sylvester order), then multiplication by norm.  Ends synchronised.
__device__ void fwht_smem(float *a, int K, float norm) {
    const int T = blockDim.x, tid = threadIdx.x;
    for (int h = 1; h < K; h <<= 1) {
        for (int i = tid; i < (K >> 1); i += T) {
            int lo = ((i & ~(h - 1)) << 1) | (i & (h - 1));
            float u = a[lo], v = a[lo + h];
            a[lo] = u + v;
            a[lo + h] = u - v;
        }
        __syncthreads();
    }
    for (int i = tid; i < K; i += T) a[i] *= norm;
    __syncthreads();
}

__global__ void __launch_bounds__(RHT_THREADS) rht_in_kernel(RhtInParams p) {
    extern __shared__ float buf[];
    __shared__ float red[32];
    __shared__ double red_d[32];
    const int b = blockIdx.x, tid = threadIdx.x, T = blockDim.x;
    pdl_launch_dependents();
    pdl_wait();  // x may come from the previous kernel on the stream

    const size_t row = (size_t)b * p.n;
    float ss = 0.f;
    for (int k = tid; k < p.n; k += T) {
        float v = load_act(p.x, row + k, p.x_bf16);
        if (sign_neg(p.sign_bits, k)) v = -v;
        buf[k] = v;
        ss += v * v;
    }
    ss = block_sum(ss, red);  // synchronises: buf complete
    for (int i = 0; i < p.blocks.count; ++i)
        fwht_smem(buf + p.blocks.offset[i], p.blocks.size[i], p.blocks.inv_sqrt[i]);

    if (p.xr_f32) {
        for (int k = tid; k < p.n; k += T) p.xr_f32[row + k] = buf[k];
        return;
    }
    // |xr_k| <= ||x||_2 (orthonormal rows), so scaling by 2^(13 - e) with
    // ||x|| < 2^e keeps every fp16 activation below 2^13.
    float nrm = sqrtf(ss);
    float scale = 1.f;
    if (nrm > 0.f && isfinite(nrm)) {
        int e;
        frexpf(nrm, &e);
        scale = ldexpf(1.f, 13 - e);
    }
    // X_k = xr_k * scale, stored /16 on columns k mod 8 in {2,3,6,7}, whose
    // decoded codeword operands carry the factor 16 (glq_internal.h)
    double corr = 0.0;
    __half *out = p.xr_h + (size_t)b * p.n_pad;
    for (int k = tid; k < p.n_pad; k += T) {
        const bool slot16 = (k >> 1) & 1;
        float v = k < p.n ? buf[k] * scale : 0.f;
        __half h = __float2half_rn(slot16 ? v * 0.0625f : v);
        out[k] = h;
        corr += (double)__half2float(h) * (slot16 ? 16.0 : 1.0);
    }
    corr = GLQ_NIB_OFFSET * block_sum_d(corr, red_d);
    if (tid == 0) p.info[b] = glq_rowinfo{corr, 1.f / scale, 0.f};
}

__global__ void __launch_bounds__(RHT_THREADS) rht_out_kernel(RhtOutParams p) {
    extern __shared__ float buf[];
    const int b = blockIdx.x, tid = threadIdx.x, T = blockDim.x;
    pdl_launch_dependents();
    pdl_wait();  // partials / z come from the previous kernel

    if (p.partials) {
        // z = ws 2^-e (2^23 sum_splits P - corr_mult * 3 sum_k X_k)
        const glq_rowinfo info = p.info[b];
        const double mul = (double)p.ws * (double)info.inv_scale;
        const double sub = (double)p.corr_mult * info.corr;
        for (int r = tid; r < p.m; r += T) {
            float z = 0.f;
            for (int s = 0; s < p.splits; ++s)  // fixed order: deterministic
                z += p.partials[((size_t)s * p.B + b) * p.m_pad + r];
            buf[r] = (float)(((double)z * (double)GLQ_ACC_SCALE - sub) * mul);
        }
    } else {
        for (int r = tid; r < p.m; r += T) buf[r] = p.z[(size_t)b * p.z_ld + r];
    }
    __syncthreads();
    for (int i = 0; i < p.blocks.count; ++i)
        fwht_smem(buf + p.blocks.offset[i], p.blocks.size[i], p.blocks.inv_sqrt[i]);

    const size_t row = (size_t)b * p.m;
    for (int r = tid; r < p.m; r += T) {
        float v = buf[r];
        if (sign_neg(p.sign_bits, r)) v = -v;
        if (p.y_dtype == 2) {
            reinterpret_cast<float *>(p.y)[row + r] = v;
        } else if (p.y_dtype == 1) {
            reinterpret_cast<__nv_bfloat16 *>(p.y)[row + r] = __float2bfloat16_rn(v);
        } else {
            reinterpret_cast<__half *>(p.y)[row + r] = __float2half_rn(v);
        }
    }
}

}  // namespace

// The dynamic shared memory limit of each kernel is raised once, to the
// largest row any layer can have: a graph captured over several layers
// replays every node against the attribute value current at replay time.
cudaError_t ensure_rht_smem() {
    static bool done = false;
    if (done) return cudaSuccess;
    const int bytes = GLQ_RHT_MAX_N * (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(rht_in_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(rht_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done = true;
    return e;
}

cudaError_t launch_rht_in(const RhtInParams &p, cudaStream_t s, bool pdl) {
    size_t smem = (size_t)p.n * sizeof(float);
    cudaError_t e = ensure_rht_smem();
    if (e != cudaSuccess) return e;
    RhtInParams q = p;
    void *args[] = {&q};
    return launch_ex((const void *)rht_in_kernel, dim3(p.B), dim3(RHT_THREADS), smem, s, pdl, args);
}

cudaError_t launch_rht_out(const RhtOutParams &p, cudaStream_t s, bool pdl) {
    size_t smem = (size_t)p.m * sizeof(float);
    cudaError_t e = ensure_rht_smem();
    if (e != cudaSuccess) return e;
    RhtOutParams q = p;
    void *args[] = {&q};
    return launch_ex((const void *)rht_out_kernel, dim3(p.B), dim3(RHT_THREADS), smem, s, pdl, args);
}

}  // namespace glq
