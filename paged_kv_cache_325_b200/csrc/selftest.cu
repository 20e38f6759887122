// Self-tests of device building blocks:
//  * the bounded mbarrier wait used by every pipelined kernel: one thread
//    waits on a barrier that nothing ever arrives at; the wait gives up after
//    the requested number of polls and reports PA_DEVERR_TIMEOUT, and the
//    kernel returns normally so the CUDA context stays usable;
//  * the prefill softmax's two exponentials: the FMA-pipe polynomial
//    (exp2_poly2) and the special-function unit's ex2, evaluated on the
//    caller's inputs so that a test can hold both to an error bound.
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

__global__ void selftest_exp2_kernel(const float *x, float *y_poly, float *y_sfu, int32_t n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
    float p0, p1;
    f2_unpack(exp2_poly2(f2_pack(x0, x1)), p0, p1);
    y_poly[i] = p0;
    y_sfu[i] = fast_exp2(x0);
    if (i + 1 < n) {
        y_poly[i + 1] = p1;
        y_sfu[i + 1] = fast_exp2(x1);
    }
}

}  // namespace

cudaError_t launch_selftest_exp2(const float *x, float *y_poly, float *y_sfu, int32_t n, cudaStream_t stream) {
    const int pairs = (n + 1) / 2;
    selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y_poly, y_sfu, n);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(int32_t *dev_error, int64_t max_polls, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(dev_error, max_polls);
    return cudaGetLastError();
}

}  // namespace pa
