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

cudaError_t bounded_wait_probe(unsigned long long wait_ns, cudaStream_t st) {
    bounded_wait_probe_kernel<<<1, 32, 0, st>>>(wait_ns);
    return cudaGetLastError();
}

}  // namespace bsa
