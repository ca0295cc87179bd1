// linear.h -- internal launch interface of the linear-branch state kernel.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace vsa {
// S, z are zeroed on `stream` and then accumulated; status may be null.
cudaError_t launch_linear_state(const Grid& g, const void* k, const void* v, float* S, float* z,
                                int* status, cudaStream_t stream,
                                PFN_cuTensorMapEncodeTiled_v12000 enc);
}  // namespace vsa
