// Self-test of the bounded mbarrier wait used by every pipelined kernel: one
// thread waits on a barrier that nothing ever arrives at; the wait gives up
// after the requested number of polls and reports PA_DEVERR_TIMEOUT, and the
// kernel returns normally so the CUDA context stays usable.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

__global__ void selftest_wait_kernel(int32_t *dev_error, int64_t max_polls) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, dev_error, (uint32_t)max_polls);
}

}  // namespace

cudaError_t launch_selftest_wait(int32_t *dev_error, int64_t max_polls, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(dev_error, max_polls);
    return cudaGetLastError();
}

}  // namespace pa
