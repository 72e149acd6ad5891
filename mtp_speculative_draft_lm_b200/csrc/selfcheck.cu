// Self-check of the pipelines' bounded waits: a wait that can never complete must give
// up, report MTP_DEVFLAG_TIMEOUT through the device error word and let the kernel end,
// leaving the context usable. The kernel runs the same wait helpers every sweep and the
// prefill use, on an mbarrier phase that no thread completes or on a global counter that
// nothing increments, with a short limit instead of the pipelines' one second.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int which, long long limit,
                                                          const uint32_t* counter,
                                                          int32_t* dev_err) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected: none ever comes
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncwarp();
    bool ok = true;
    if (threadIdx.x == 0) {
        if (which == 0)
            ok = mbar_wait_bounded(&bar, 0u, &abort_flag, limit);
        else
            ok = counter_wait_bounded(counter, 1u, &abort_flag, limit);
        if (!ok && abort_flag) raise_flag(dev_err, DEVFLAG_TIMEOUT);
    }
    __syncwarp();
}

}  // namespace

cudaError_t wait_timeout_launch(int which, long long limit_cycles, const uint32_t* counter,
                                int32_t* dev_err, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(which, limit_cycles, counter, dev_err);
    return cudaGetLastError();
}

}  // namespace mtp
