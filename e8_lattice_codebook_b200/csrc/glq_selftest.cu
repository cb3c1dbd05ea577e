// glq_selftest.cu -- a check of the library's bounded device waits, for
// testing failure detection without faulting or hanging the GPU.
//
// Every wait in the layer's kernels (the tensor-core pipeline's mbarriers,
// its cluster-scope ones, the codebook-table loads of the GEMV and the W
// reconstruction) gives up after a limit and reports GLQ_DEVERR_TIMEOUT
// through the layer's device error word.  This kernel runs the same wait
// helpers on an mbarrier that only some of its expected arrivals reach, so
// that the wait runs out for certain (a flag that nothing sets), with a
// short limit chosen by the caller; no copy or other memory operation is
// pending on the barrier.
#include "glq_kernels.cuh"
#include "glq_sm100.cuh"

namespace glq {

namespace {

__global__ void wait_selftest_kernel(unsigned *err, int kind, int arrivals, unsigned long long limit) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) mbar_init(&bar, 2);  // phase 0 completes after two arrivals
    __syncthreads();
    if (threadIdx.x != 0) return;
    for (int i = 0; i < arrivals; ++i) sm100::mbar_arrive(&bar);
    bool ok;
    if (kind == 0) ok = sm100::mbar_wait(&bar, 0, limit);
    else if (kind == 1) ok = sm100::mbar_wait_cluster(&bar, 0, limit);
    else ok = mbar_wait_bounded(&bar, 0, (uint32_t)limit);
    if (!ok) atomicOr(err, GLQ_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned *err, int kind, int arrivals, unsigned long long limit, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(err, kind, arrivals, limit);
    return cudaGetLastError();
}

}  // namespace glq
