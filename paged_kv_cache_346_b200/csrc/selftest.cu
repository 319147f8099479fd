// Failure-detection self-test: the bounded mbarrier wait every decode kernel
// uses, on a barrier that nothing completes.
#include "device_common.cuh"

namespace pkv {

__global__ void wait_timeout_kernel(long long limit, unsigned int* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    // phase 0 never completes: nobody arrives and no copy is expected
    mbar_wait_limit(&bar, 0, status, limit);
}

cudaError_t launch_wait_timeout(long long limit, unsigned int* status, cudaStream_t stream) {
    wait_timeout_kernel<<<1, 32, 0, stream>>>(limit, status);
    return cudaGetLastError();
}

}  // namespace pkv
