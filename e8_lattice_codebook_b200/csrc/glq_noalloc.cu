// glq_noalloc.cu -- glq_linear_noalloc: the decode path of glq_linear for
// callers that cannot allocate device memory at call time.
//
// Who needs it: code that runs where cudaMalloc is unavailable or unsafe --
// while a CUDA graph is being captured (an allocation would break the
// capture), inside a host callback or a custom memory-pool regime that
// forbids driver allocations, or in a process whose allocator is owned by
// another framework.  glq_linear allocates its per-layer workspace on first
// use; this entry point instead keeps every transient buffer in one
// file-scope device array that exists for as long as the library is loaded
// on a device.
//
// The kernels are the ones glq_linear launches (input RHT, codebook GEMV,
// output RHT); only the workspace pointers differ, and the split-K plan is
// narrowed, when its partial sums would not fit the array, to a split
// count whose partial sums do.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "../../include/glq.h"
#include "glq_handles.h"
#include "glq_internal.h"
#include "glq_kernels.cuh"

// The scratch array: activations, per-token row info, the output of the
// GEMV, the per-band counters and the split-K partial sums of one call.
// Every GPU that loads the library holds it until the process exits.  Calls
// share it: two calls whose kernels overlap on the GPU (different streams,
// or different layers without ordering) race on it.  A call also uses the
// layer's own device words (its error flag and the output-block counters of
// the fused output transform), so calls on one layer must not overlap on
// the GPU whichever entry point they use.
static __device__ __align__(256) unsigned char g_glq_noalloc_scratch[GLQ_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int MAX_DEVICES = 128;
std::mutex g_scratch_mu;
void *g_scratch_ptr[MAX_DEVICES] = {};

// Device address of the scratch array on `dev` (which must be current).
// In host code the array's name is only a host-side stand-in, so the
// address comes from cudaGetSymbolAddress, once per device.
glq_status scratch_address(int dev, void **out) {
    if (dev < 0 || dev >= MAX_DEVICES) return GLQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_glq_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return GLQ_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GLQ_OK;
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace

extern "C" glq_status glq_linear_noalloc(glq_layer L, const void *x_dev, glq_dtype x_dtype, void *y_dev,
                                         glq_dtype y_dtype, int64_t B, void *stream) {
    if (!L || L->shard) return GLQ_ERR_INVALID_ARG;  // a shard's row sums need the shared workspace
    if (B < 0 || B > GLQ_DECODE_MAX_B) return GLQ_ERR_SHAPE;
    if (x_dtype != GLQ_F16 && x_dtype != GLQ_BF16) return GLQ_ERR_DTYPE;
    if (y_dtype != x_dtype && y_dtype != GLQ_F32) return GLQ_ERR_DTYPE;
    if (B == 0) return GLQ_OK;
    if (!x_dev || !y_dev) return GLQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x_dev) & 15) || (reinterpret_cast<uintptr_t>(y_dev) & 15))
        return GLQ_ERR_INVALID_ARG;

    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) {
        cudaGetLastError();
        return GLQ_ERR_CUDA;
    }
    const bool switched = prev != L->device;
    if (switched && cudaSetDevice(L->device) != cudaSuccess) {
        cudaGetLastError();
        return GLQ_ERR_CUDA;
    }
    void *base = nullptr;
    glq_status st = scratch_address(L->device, &base);

    // carve the array: xq | xh | info | z | counters | partials
    const size_t xq_b = align256((size_t)B * L->n_pad * 2);
    const size_t xh_b = L->has8 ? align256((size_t)B * L->n_pad * sizeof(__half)) : 0;
    const size_t info_b = align256((size_t)B * sizeof(glq_rowinfo));
    const size_t z_b = align256((size_t)B * L->m_pad * sizeof(float));
    const int max_bands = std::max(L->plan[0].bands, L->plan[1].bands);
    const size_t cnt_b = align256((size_t)max_bands * sizeof(unsigned));
    const size_t fixed = xq_b + xh_b + info_b + z_b + cnt_b;
    const size_t per_split = (size_t)B * L->m_pad * sizeof(double);
    glq::DecodeCfg cfg;
    if (st == GLQ_OK) {
        if (fixed > GLQ_NOALLOC_SCRATCH_BYTES) {
            st = GLQ_ERR_SHAPE;  // the activations and outputs alone do not fit
        } else {
            // glq_linear's plan, unless its partial sums would not fit: only
            // a split plan without the cluster reduction keeps them in global
            // memory (one split writes z directly; the cluster reduction adds
            // them in distributed shared memory).  Then the split count is
            // bounded by the room left.
            const size_t room = GLQ_NOALLOC_SCRATCH_BYTES - fixed;
            auto global_partials = [&](const glq::DecodeCfg &c) {
                return c.plan.splits > 1 && c.clu == 0 ? (size_t)c.plan.splits * per_split : (size_t)0;
            };
            cfg = glq::decode_config(L, (int)B, x_dev, y_dev, (int)y_dtype);
            if (global_partials(cfg) > room) {
                const int max_splits = (int)std::max<size_t>(1, std::min<size_t>(room / per_split, 1u << 30));
                cfg = glq::decode_config(L, (int)B, x_dev, y_dev, (int)y_dtype, max_splits);
                if (global_partials(cfg) > room) st = GLQ_ERR_SHAPE;
            }
        }
    }
    if (st == GLQ_OK) {
        char *p = static_cast<char *>(base);
        glq_workspace w;
        w.xq = reinterpret_cast<uint8_t *>(p);
        w.xh = L->has8 ? reinterpret_cast<__half *>(p + xq_b) : nullptr;
        w.info = reinterpret_cast<glq_rowinfo *>(p + xq_b + xh_b);
        w.z = reinterpret_cast<float *>(p + xq_b + xh_b + info_b);
        w.cnt = reinterpret_cast<unsigned *>(p + xq_b + xh_b + info_b + z_b);
        w.part = cfg.plan.splits > 1 ? reinterpret_cast<double *>(p + fixed) : nullptr;
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        // the band counters must start at zero (the array keeps whatever the
        // previous call, of any layer, left there)
        if (cudaMemsetAsync(w.cnt, 0, (size_t)cfg.plan.bands * sizeof(unsigned), s) != cudaSuccess ||
            glq::run_decode(L, w, cfg, x_dev, x_dtype == GLQ_BF16, y_dev, (int)y_dtype, (int)B, s) !=
                cudaSuccess) {
            cudaGetLastError();
            st = GLQ_ERR_CUDA;
        }
    }
    if (switched) cudaSetDevice(prev);
    return st;
}
