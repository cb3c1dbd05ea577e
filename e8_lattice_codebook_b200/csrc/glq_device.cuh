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
// T is a shared-memory array of nibble words (address space shared).
__device__ __forceinline__ uint32_t table_word(const uint32_t *T, uint32_t e, FoldParams f) {
    uint32_t w;
    asm("{\n"
        " .reg .pred p;\n"
        " .reg .u32 c, a;\n"
        " setp.ge.u32 p, %1, %2;\n"
        " mov.u32 c, %1;\n"
        " @p sub.u32 c, %1, %3;\n"
        " shl.b32 a, c, 2;\n"
        " add.u32 a, a, %4;\n"
        " ld.shared.u32 %0, [a];\n"
        " @p sub.u32 %0, 0xCCCCCCCC, %0;\n"
        "}\n"
        : "=r"(w)
        : "r"(e), "r"((uint32_t)f.nb), "r"((uint32_t)f.neg_base),
          "r"((uint32_t)__cvta_generic_to_shared(T)));
    return w;
}

// Multipliers the GEMV's lookups take at run time (4, 16 and -1): given as
// kernel parameters, the compiler cannot turn the multiply-adds that use them
// into shifts or logic, so address, negation and scaling run on the integer
// multiply-add (FMA) pipe beside the logic ops on the ALU pipe.
struct LookupConsts {
    uint32_t four, sixteen, neg_one;
};

// The two A-fragment registers of code e scaled by 16: lo16 = 16 (v0..v3),
// hi16 = 16 (v4..v7) as u8 (16 v <= 192).  tbase / tneg are the shared
// addresses of T[0] and T[-neg_base].
__device__ __forceinline__ void table_a16(uint32_t tbase, uint32_t tneg, uint32_t e, uint32_t nb,
                                          LookupConsts k, uint32_t &lo16, uint32_t &hi16) {
    asm("{\n"
        " .reg .pred p;\n"
        " .reg .u32 a, w, t;\n"
        " setp.ge.u32 p, %2, %3;\n"
        " mad.lo.u32 a, %2, %4, %5;\n"
        " @p mad.lo.u32 a, %2, %4, %6;\n"
        " ld.shared.u32 w, [a];\n"
        " @p mad.lo.u32 w, w, %7, %8;\n"
        " and.b32 %1, w, 0xF0F0F0F0;\n"
        " mul.lo.u32 t, w, %9;\n"
        " and.b32 %0, t, 0xF0F0F0F0;\n"
        "}\n"
        : "=r"(lo16), "=r"(hi16)
        : "r"(e), "r"(nb), "r"(k.four), "r"(tbase), "r"(tneg), "r"(k.neg_one), "r"(0xCCCCCCCCu),
          "r"(k.sixteen));
}

// The same lookup from a global-memory table (reference decode).
__device__ __forceinline__ uint32_t table_word_global(const uint32_t *T, uint32_t e, FoldParams f) {
    const bool neg = e >= (uint32_t)f.nb;
    const uint32_t w = T[neg ? e - (uint32_t)f.neg_base : e];
    return neg ? 0xCCCCCCCCu - w : w;
}

// The two A-fragment registers of one codeword for the integer MMA:
// lo = (v0, v1, v2, v3), hi = (v4, v5, v6, v7) as u8, v = 2x + 6.
__device__ __forceinline__ uint32_t nib_lo(uint32_t w) { return w & 0x0F0F0F0Fu; }
__device__ __forceinline__ uint32_t nib_hi(uint32_t w) { return (w >> 4) & 0x0F0F0F0Fu; }

// Exact float coordinates x0..x7 of a table word (reference decode): the
// same byte unpack, then x = v/2 - 3.
__device__ __forceinline__ void unpack_exact(uint32_t w, float x[8]) {
    const uint32_t lo = nib_lo(w), hi = nib_hi(w);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[j] = 0.5f * (float)((lo >> (8 * j)) & 0xFFu) - 3.0f;
        x[4 + j] = 0.5f * (float)((hi >> (8 * j)) & 0xFFu) - 3.0f;
    }
}

// ---------------------------------------------------------------------------
// Warp MMAs
// ---------------------------------------------------------------------------

// D(16x8, s32) += A(16x32, u8, row) . B(32x8, s8, col)
__device__ __forceinline__ void mma_u8s8(int d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D(16x8, s32) += A(16x32, u8, row) . B(32x8, u8, col)
__device__ __forceinline__ void mma_u8u8(int d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D(16x8, f32) += A(16x16, f16, row) . B(16x8, f16, col)
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

// Bring a line into L2 (no register result).  Safe before the wait on a
// producing kernel: L2 is the point of coherence, so the producer's later
// writes replace whatever the prefetch brought in; it warms the TLB and L2
// for data that is already final.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned *p, unsigned v) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
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
