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
// narrowed, if needed, so that the partial sums fit the array.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "../../include/glq.h"
#include "glq_handles.h"
#include "glq_internal.h"
#include "glq_kernels.cuh"

// The scratch array: activations (fp16), per-token row info and split-K
// partial sums of one call.  Every GPU that loads the library holds it
// until the process exits.  Calls share it: two calls whose kernels overlap
// on the GPU (different streams, or different layers without ordering)
// race on it.
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
    if (!L) return GLQ_ERR_INVALID_ARG;
    if (B < 0 || B > GLQ_DECODE_MAX_B) return GLQ_ERR_SHAPE;
    if (x_dtype != GLQ_F16 && x_dtype != GLQ_BF16) return GLQ_ERR_DTYPE;
    if (y_dtype != x_dtype && y_dtype != GLQ_F32) return GLQ_ERR_DTYPE;
    if (B == 0) return GLQ_OK;
    if (!x_dev || !y_dev) return GLQ_ERR_INVALID_ARG;

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
    glq_status st = GLQ_OK;
    void *base = nullptr;
    st = scratch_address(L->device, &base);

    // carve the array: xr [B][n_pad] fp16 | info [B] | partials [splits][B][m_pad]
    const size_t xr_bytes = align256((size_t)B * L->n_pad * sizeof(__half));
    const size_t info_bytes = align256((size_t)B * sizeof(glq_rowinfo));
    const size_t per_split = (size_t)B * L->m_pad * sizeof(float);
    int splits = L->splits, cps = L->cps;
    if (st == GLQ_OK) {
        if (xr_bytes + info_bytes + per_split > GLQ_NOALLOC_SCRATCH_BYTES) {
            st = GLQ_ERR_SHAPE;  // even one split does not fit the array
        } else {
            // narrow the split-K plan until its partial sums fit
            const size_t room = GLQ_NOALLOC_SCRATCH_BYTES - xr_bytes - info_bytes;
            while ((size_t)splits * per_split > room) {
                cps = cps + 1;
                splits = (L->KC + cps - 1) / cps;
            }
        }
    }
    if (st == GLQ_OK) {
        char *p = static_cast<char *>(base);
        __half *xr = reinterpret_cast<__half *>(p);
        glq_rowinfo *info = reinterpret_cast<glq_rowinfo *>(p + xr_bytes);
        float *part = reinterpret_cast<float *>(p + xr_bytes + info_bytes);
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        const int nb = (int)B;

        glq::RhtInParams pin{};
        pin.x = x_dev;
        pin.x_bf16 = x_dtype == GLQ_BF16;
        pin.n = (int)L->n;
        pin.n_pad = (int)L->n_pad;
        pin.B = nb;
        pin.sign_bits = L->d_sin;
        pin.blocks = L->bn;
        pin.xr_h = xr;
        pin.info = info;

        glq::GemvParams pg{};
        pg.idx1 = L->d_idx1;
        pg.idx2 = L->d_idx2;
        pg.table = L->primary->d_table;
        pg.table_words = L->primary->table_words;
        pg.fold = glq::FoldParams{L->primary->fold.nb, L->primary->fold.neg_base};
        pg.res8 = (L->bpw == 3) ? reinterpret_cast<const uint4 *>(L->d_r8) : nullptr;
        pg.xr = xr;
        pg.B = nb;
        pg.n_pad = (int)L->n_pad;
        pg.KC = L->KC;
        pg.RT = L->RT;
        pg.bands = L->bands;
        pg.splits = splits;
        pg.cps = cps;
        pg.rs_acc = L->bpw == 3 ? L->rs / GLQ_ACC_SCALE : L->rs;
        pg.partials = part;
        pg.m_pad = (int)L->m_pad;
        pg.err = L->d_err;
        const int grid = (int)std::min<int64_t>((int64_t)L->bands * splits, L->num_sms);

        glq::RhtOutParams pout{};
        pout.m = (int)L->m;
        pout.m_pad = (int)L->m_pad;
        pout.B = nb;
        pout.partials = part;
        pout.splits = splits;
        pout.info = info;
        pout.ws = L->ws;
        pout.corr_mult = L->bpw == 4 ? 1.f + L->rs : 1.f;
        pout.sign_bits = L->d_sout;
        pout.blocks = L->bm;
        pout.y = y_dev;
        pout.y_dtype = (int)y_dtype;

        if (glq::launch_rht_in(pin, s, true) != cudaSuccess ||
            glq::launch_gemv(pg, L->bpw, grid, s, true) != cudaSuccess ||
            glq::launch_rht_out(pout, s, true) != cudaSuccess) {
            cudaGetLastError();
            st = GLQ_ERR_CUDA;
        }
    }
    if (switched) cudaSetDevice(prev);
    return st;
}
