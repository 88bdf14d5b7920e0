// selftest.cu -- a device check of the pipeline waits' time limit: one warp
// waits, with the bounded mbarrier wait every GEMM pipeline uses, on a barrier
// that nothing arrives on, and reports the timeout in the caller's status word
// instead of hanging or trapping.
#include "internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(32, 1) wait_limit_kernel(int32_t* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        // phase 0 of a fresh barrier completes only on an arrival, and none comes
        if (!mbar_wait(&bar, 0, &abort_flag)) status_or(status, MOE_DEV_TIMEOUT);
    }
}

}  // namespace

cudaError_t launch_wait_limit_selftest(int32_t* status, cudaStream_t st) {
    wait_limit_kernel<<<1, 32, 0, st>>>(status);
    return cudaGetLastError();
}

}  // namespace moe
