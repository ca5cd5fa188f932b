// Self-test of the bounded waits: one thread waits on an mbarrier phase that nothing completes,
// with the same bounded wait the pipelines use; when it gives up, the kernel records the
// timeout status and returns (no trap, no fault, the context stays usable).
#include "device_common.cuh"
#include "launchers.h"
#include "sm100_ptx.cuh"

namespace rkv {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(int32_t* err)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);   // one arrival completes phase 0; nothing arrives
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, &abort_flag))
        report(err, RKV_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int32_t* err, cudaStream_t st)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(err);
    return cudaGetLastError();
}

}  // namespace rkv
