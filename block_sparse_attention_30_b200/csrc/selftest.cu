// selftest.cu -- exercises the failure path every kernel relies on: a bounded
// mbarrier wait that gives up, records VSA_ERR_TIMEOUT in the workspace status
// word and returns, leaving the CUDA context usable.  Nothing faults: the
// kernel waits on a barrier that no thread ever arrives at.
#include <cuda_runtime.h>

#include "../../include/vsa.h"
#include "common.cuh"
#include "sm100.cuh"

namespace vsa {
using namespace sm100;

__global__ void __launch_bounds__(32) wait_timeout_kernel(int* status, unsigned long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    // no thread arrives on `bar`: phase 0 never completes
    const bool ok = mbar_wait_for(&bar, 0, &abort_flag, limit);
    if (!ok && threadIdx.x == 0) report(status, kStatusTimeout);
}

}  // namespace vsa

extern "C" {
#pragma GCC visibility push(default)

vsa_status vsa_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                     unsigned int limit_cycles, vsa_stream_t stream) {
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 15u)) return VSA_ERR_WORKSPACE;
    if (workspace_bytes < 256) return VSA_ERR_WORKSPACE;
    if (limit_cycles == 0) return VSA_ERR_INVALID_ARGUMENT;
    vsa::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<int*>(workspace),
                                                                  (unsigned long long)limit_cycles);
    return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

#pragma GCC visibility pop
}  // extern "C"
