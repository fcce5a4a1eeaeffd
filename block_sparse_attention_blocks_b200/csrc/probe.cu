// Failure-detection check for the bounded device waits: one CTA waits on an mbarrier that
// nothing ever arrives at.  The wait gives up after the configured limit, records the timeout in
// the device error word and the kernel returns normally.
#include "bsa_internal.h"

namespace bsa {

__global__ void bounded_wait_probe_kernel(unsigned long long wait_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, wait_ns, (volatile int *)&abort_flag);
}

// Evaluates the softmax's FMA-pipe 2^x (exp2_poly2) element-wise, for tests against exp2f.
__global__ void exp2_poly_kernel(const float *x, float *y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
        y[i] = r.x;
        y[i + 1] = r.y;
    } else if (i < n) {
        y[i] = exp2_poly2(make_float2(x[i], x[i])).x;
    }
}

cudaError_t exp2_poly_eval(const float *x, float *y, int n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int pairs = (n + 1) / 2;
    exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y, n);
    return cudaGetLastError();
}

cudaError_t bounded_wait_probe(unsigned long long wait_ns, cudaStream_t st) {
    bounded_wait_probe_kernel<<<1, 32, 0, st>>>(wait_ns);
    return cudaGetLastError();
}

}  // namespace bsa
