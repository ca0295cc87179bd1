// tiles.h -- internal launch interface of the cube gather / scatter kernels.
#pragma once
#include <cuda_runtime.h>

#include "common.cuh"

namespace vsa {
cudaError_t launch_gather(const Grid& g, const void* x, void* x_tiles, cudaStream_t stream);
cudaError_t launch_scatter(const Grid& g, const void* x_tiles, void* x, cudaStream_t stream);
}  // namespace vsa
