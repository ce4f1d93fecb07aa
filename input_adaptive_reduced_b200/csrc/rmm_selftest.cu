// rmm_selftest.cu -- a kernel that makes the library's bounded wait run out,
// so that the failure path (error word, RMM_ERR_TIMEOUT, a usable context)
// can be tested without faulting, trapping or hanging the GPU.
#include <cstdint>

#include <cuda_runtime.h>

#include "rmm.h"
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

// One thread waits on an mbarrier that expects one arrival and never gets it.
__global__ void wait_timeout_kernel(int* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, kErrTimeoutMma);
}

}  // namespace
}  // namespace rmm

extern "C" rmm_status rmm_selftest_wait_timeout(const rmm_plan* plan, void* ws, size_t ws_bytes, void* stream) {
    if (!plan || !ws) return RMM_ERR_INVALID_ARG;
    if (ws_bytes < plan->ws_bytes || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return RMM_ERR_WORKSPACE;
    int* err = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + plan->off_err);
    rmm::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err);
    return cudaGetLastError() == cudaSuccess ? RMM_OK : RMM_ERR_CUDA;
}
