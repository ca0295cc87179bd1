// linear.h -- internal launch interface of the linear-branch state kernel.
#pragma once
#include <cuda_runtime.h>

#include "common.cuh"

namespace vsa {
cudaError_t launch_linear_state(const Grid& g, const void* k, const void* v, float* S, float* z,
                                cudaStream_t stream);
}  // namespace vsa
