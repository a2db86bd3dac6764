// Diagnostic for the library's failure detection: one CTA waits, through the
// same bounded mbarrier wait the pipelined kernels use, on a barrier that
// nothing will ever arrive on.  The wait gives up after `limit_ns`, records
// MOE_ERR_TIMEOUT in the device status word and the kernel returns, so the
// context stays usable.  No trap, no fault, no unbounded spin.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival that never comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, &abort_flag, status, limit_ns);
    __syncthreads();
}

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int* status, cudaStream_t st) {
    bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, status);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
