// glq_device.cuh -- device helpers shared by the glq-b200 kernels: the
// codeword decode (fold + nibble unpack), the warp MMA, fixed-order
// reductions, bounded waits and PDL controls.  Layouts: glq_internal.h.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "glq_internal.h"

namespace glq {

// ---------------------------------------------------------------------------
// Codeword decode
// ---------------------------------------------------------------------------

struct FoldParams {
    int nb;        // table words
    int neg_base;  // code e >= nb reads T[e - neg_base], negated
};

// Table word of code e (a 16-bit value), negation applied.
// T is a shared-memory (or global) array of nibble words.
__device__ __forceinline__ uint32_t table_word(const uint32_t *T, uint32_t e, FoldParams f) {
    bool neg = e >= (uint32_t)f.nb;
    uint32_t pos = neg ? e - (uint32_t)f.neg_base : e;
    uint32_t w = T[pos];
    return neg ? 0xCCCCCCCCu - w : w;
}

// Unpacks a nibble word into four fp16x2 registers of exact subnormals:
//   h[0] = (v0, v1) 2^-24,     h[1] = (v2, v3) 16 * 2^-24,
//   h[2] = (v4, v5) 2^-24,     h[3] = (v6, v7) 16 * 2^-24,
// with v_j = 2 x_j + 6 (layout: glq_internal.h).
__device__ __forceinline__ void unpack_sub(uint32_t w, uint32_t h[4]) {
    uint32_t w8 = w >> 8;
    h[0] = w & 0x000F000Fu;
    h[1] = w & 0x00F000F0u;
    h[2] = w8 & 0x000F000Fu;
    h[3] = w8 & 0x00F000F0u;
}

// Exact float coordinates x0..x7 of a nibble word: the same unpack, then
// x = h * 2^23 - 3 (x 2^19 for the h[1], h[3] pairs), exact in fp32.
__device__ __forceinline__ void unpack_exact(uint32_t w, float x[8]) {
    uint32_t h[4];
    unpack_sub(w, h);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        __half2 v = *reinterpret_cast<__half2 *>(&h[p]);
        float mul = (p & 1) ? 524288.0f : 8388608.0f;  // 2^19 : 2^23
        x[2 * p] = __low2float(v) * mul - 3.0f;
        x[2 * p + 1] = __high2float(v) * mul - 3.0f;
    }
}

// ---------------------------------------------------------------------------
// Warp MMA  D = A(16x16, f16, row) . B(16x8, f16, col) + D (f32)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Loads
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

// cached in L1: activations reused by every warp of a CTA
__device__ __forceinline__ uint4 ldg_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch
// ---------------------------------------------------------------------------

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Bulk copy global -> shared with an mbarrier, bounded wait
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// 1-D bulk copy; dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Waits for phase `parity` of the barrier; gives up after max_polls polls.
// Returns true on completion.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint32_t max_polls) {
    uint32_t done = 0;
    for (uint32_t i = 0; i < max_polls; ++i) {
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(smem_addr(bar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// ---------------------------------------------------------------------------
// Fixed-order block reduction (deterministic): warp tree, then warps in order
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// scratch: >= 32 floats of shared memory.  All threads get the result.
__device__ __forceinline__ float block_sum(float v, float *scratch) {
    int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float s = 0.f;
    for (int w = 0; w < nw; ++w) s += scratch[w];
    return s;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ double block_sum_d(double v, double *scratch) {
    int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    v = warp_sum_d(v);
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    double s = 0.0;
    for (int w = 0; w < nw; ++w) s += scratch[w];
    return s;
}

}  // namespace glq
