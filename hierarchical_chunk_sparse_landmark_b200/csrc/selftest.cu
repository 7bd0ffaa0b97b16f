// selftest.cu -- exercises the failure path shared by every bounded wait of
// the library's kernels, without a fault or a hang: one block waits on an
// mbarrier that nothing ever arrives on, gives up after its cycle budget, sets
// the timeout flag in the caller's status word and exits.  The host then reads
// the flag through hsa_check like after any other call.
#include "common.cuh"
#include "tc.cuh"

namespace hsa {

__global__ void __launch_bounds__(32, 1) selftest_wait_kernel(unsigned *status, long long budget) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_barrier_init();
    }
    __syncwarp();
    // phase 0 never completes: the arrival it waits for is never made
    if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0u, budget)) atomicOr(status, kFlagTimeout);
}

cudaError_t launch_selftest_wait(unsigned *status, long long budget, cudaStream_t st) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(status, budget);
    return cudaGetLastError();
}

}  // namespace hsa
