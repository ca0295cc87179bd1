// quant.h -- internal launch interface of the E4M3 quantisation kernel.
#pragma once
#include <cuda_runtime.h>

#include "common.cuh"

namespace vsa {
// q8, k8: [B][N][heads][d] E4M3 codes (valid tokens written); q_scale,
// k_scale: [B][heads][nt] fp32.
cudaError_t launch_quant_e4m3(const Grid& g, const void* q, const void* k, void* q8, void* k8,
                              float* q_scale, float* k_scale, cudaStream_t stream);
}  // namespace vsa
