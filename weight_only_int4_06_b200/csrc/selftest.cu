// Self-test of the bounded waits: every mbarrier wait in the library gives up after a time limit,
// records W4_ERR_DEVICE_TIMEOUT and lets the kernel return, so that a lost arrival cannot hang the
// GPU and the context stays usable.  This kernel waits on a barrier that nothing arrives at.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace w4 {

__global__ void __launch_bounds__(32) selftest_wait_kernel(uint64_t limit_ns, int* status) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (!mbar_wait_bounded(b, 0, nullptr, limit_ns) && threadIdx.x == 0) record_status(status, W4_ERR_DEVICE_TIMEOUT);
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, int* status, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns, status);
    return cudaGetLastError();
}

}  // namespace w4
