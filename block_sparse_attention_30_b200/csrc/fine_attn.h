// fine_attn.h -- internal launch interface of the fine-pass kernel.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace vsa {

struct FineArgs {
    Grid g;
    const void* q;               // bf16 q [B][N][heads][d] (the persistent kernel reads rows)
    const CUtensorMap* mq;       // 5-D maps over q, k, v (see api.cu)
    const CUtensorMap* mk;
    const CUtensorMap* mv;
    const int32_t* block_idx;    // [B][heads][nt][topk]
    int topk;
    const void* lin_image;       // optional linear-branch operand images, one per
                                 // (b, head) (linear_image_bytes(d) each, see linear.h)
    void* out;                   // bf16 [B][N][heads][d]
    float* out32;                // optional fp32 copy of out (for the backward pass)
    float* lse;                  // optional [B][heads][nt][64]: log2 softmax normaliser
                                 // of the scaled scores per cube slot (+inf if padded)
    const float* q_scale;        // low-precision variant: E4M3 q, k with one scale
    const float* k_scale;        // per (b, head, cube) [B][heads][nt]; null for bf16
    int* status;                 // device status word
};

cudaError_t launch_fine(const FineArgs& a, cudaStream_t stream);
cudaError_t launch_fine_single(const FineArgs& a, cudaStream_t stream);
cudaError_t launch_fine_pair(const FineArgs& a, cudaStream_t stream);
int fine_smem_bytes(int d);

}  // namespace vsa
