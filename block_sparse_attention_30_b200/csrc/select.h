// select.h -- internal launch interface of the block-selection kernels.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "common.cuh"

namespace vsa {

struct SelectArgs {
    Grid g;
    const uint16_t* q;      // bf16 [B][N][heads][d]
    const uint16_t* k;
    int topk;
    int32_t* block_idx;     // [B][heads][nt][topk]
    void* scratch;          // select_scratch_bytes(g) bytes, 16-byte aligned
    int* status;            // device status word (timeouts), or null
};

bool select_supported(const Grid& g);   // nt small enough for the score rows in shared memory
size_t select_scratch_bytes(const Grid& g);
cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream);

}  // namespace vsa
