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
// Bytes of the per-(b, head) operand image of (S, z) the fine kernel copies
// into shared memory: S hi, S lo (bf16, d x d each) and z (fp32, d).
__host__ __device__ constexpr long long linear_image_bytes(int d) { return 4ll * d * d + 4ll * d; }

// Writes the operand images of all (b, head) into `image`
// (B * heads * linear_image_bytes(d) bytes, 16-byte aligned).
cudaError_t launch_linear_pack(const Grid& g, const float* S, const float* z, void* image,
                               cudaStream_t stream);
}  // namespace vsa
