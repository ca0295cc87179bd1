// linear.h -- internal launch interface of the linear-branch kernels.
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

// 3-D TMA view (heads*d, N, B) of a [B][N][heads][d] bf16 tensor, box = 64
// features x 64 tokens of one batch, 128-byte swizzle, zero fill past N.
bool encode_token_map(CUtensorMap* m, const void* base, const Grid& g,
                      PFN_cuTensorMapEncodeTiled_v12000 fn);

// Backward of the linear branch (linear_bwd.cu).  Scratch (device, 256-byte
// aligned, linear_bwd_scratch_bytes(g) bytes) holds the operand image of
// (S, z), the fp32 (dS, dz) sums and their operand image.  dq, dk, dv are
// overwritten, or added to when `accumulate` is nonzero.
long long linear_bwd_scratch_bytes(const Grid& g);
cudaError_t launch_linear_bwd(const Grid& g, const void* q, const void* k, const void* v,
                              const void* dout, const float* S, const float* z, void* dq, void* dk,
                              void* dv, int accumulate, uint8_t* scratch, int* status,
                              cudaStream_t stream, PFN_cuTensorMapEncodeTiled_v12000 enc);
}  // namespace vsa
