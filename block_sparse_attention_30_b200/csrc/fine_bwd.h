// fine_bwd.h -- internal launch interface of the backward pass of the fine
// block-sparse attention.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace vsa {

struct BwdArgs {
    Grid g;
    const CUtensorMap* mq;       // 5-D maps over q, k, v, dout (same view as the forward)
    const CUtensorMap* mk;
    const CUtensorMap* mv;
    const CUtensorMap* mg;
    const int32_t* block_idx;    // [B][heads][nt][topk], rows ascending
    int topk;
    const float* out32;          // forward output in fp32, [B][N][heads][d]
    const void* dout;            // its gradient, bf16 [B][N][heads][d]
    const float* lse;            // [B][heads][nt][64] from the forward (log2 units, +inf padded)
    void* dq;                    // bf16 [B][N][heads][d], fully written
    void* dk;
    void* dv;
    void* scratch;               // bwd_scratch_bytes(g, topk) bytes, 256-byte aligned
    int* status;                 // device status word
};

size_t bwd_scratch_bytes(const Grid& g, int topk);
bool bwd_supported(const Grid& g);   // one row of the transpose's bitmap fits its shared memory
cudaError_t launch_fine_bwd(const BwdArgs& a, cudaStream_t stream);

}  // namespace vsa
