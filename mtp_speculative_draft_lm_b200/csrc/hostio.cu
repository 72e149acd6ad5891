// Host-resident inputs and results for the lm_head sweep (mtp_lm_head_argmax_host).
//
// x arrives in pinned host memory, which the device reaches through its mapped address.
// One small kernel copies it into the workspace: it loads its share first, then waits for
// the previous grid in the stream (programmatic dependent launch) before storing, so the
// host-link latency overlaps the previous sweep's tail while that sweep's own reads of
// the same workspace bytes are finished before they are overwritten. The sweep that
// follows writes its indices and values straight into the caller's pinned result buffer.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

constexpr int kFetchThreads = 256;
constexpr int kFetchPer = 4;  // 16-byte vectors per thread

__global__ void __launch_bounds__(kFetchThreads) fetch_x_kernel(const uint4* __restrict__ src,
                                                                 uint4* __restrict__ dst,
                                                                 int64_t n16) {
    pdl_launch_dependents();
    const int64_t base = (int64_t)blockIdx.x * kFetchThreads * kFetchPer + threadIdx.x;
    uint4 v[kFetchPer];
#pragma unroll
    for (int j = 0; j < kFetchPer; ++j) {
        const int64_t i = base + (int64_t)j * kFetchThreads;
        if (i < n16) v[j] = __ldcv(src + i);  // host memory: fetched anew on every call
    }
    pdl_wait();
#pragma unroll
    for (int j = 0; j < kFetchPer; ++j) {
        const int64_t i = base + (int64_t)j * kFetchThreads;
        if (i < n16) dst[i] = v[j];
    }
}

}  // namespace

cudaError_t fetch_x_launch(const void* src, void* dst, size_t bytes, cudaStream_t s) {
    const int64_t n16 = (int64_t)(bytes / 16);
    if (n16 < 1 || bytes % 16) return cudaErrorInvalidValue;
    const int64_t per_cta = (int64_t)kFetchThreads * kFetchPer;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((n16 + per_cta - 1) / per_cta));
    cfg.blockDim = dim3(kFetchThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fetch_x_kernel, static_cast<const uint4*>(src),
                                       static_cast<uint4*>(dst), n16);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace mtp
