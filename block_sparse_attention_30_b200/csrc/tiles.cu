// tiles.cu -- cube-tile gather / scatter between grid order [B][N][heads][d]
// and cube-major [B][heads][nt][64][d] (bf16, bit-exact copies).
//
// The cube grouping is the tiling step behind "FastVideo 稀疏蒸馏技术深度解析"
// (omica.com.cn), section "2. 视频稀疏注意力VSA" (key blocks are spatio-temporal
// blocks of the video).  The fused forward path never materialises these
// layouts -- its TMA boxes cut cubes straight out of grid order -- but the
// copies are part of the library for callers that keep cube-major tensors.
//
// One thread moves one 16-byte vector (8 bf16); consecutive threads walk the
// d axis of one slot, then the slots of a cube, so every warp reads and writes
// whole 128-byte lines of both layouts.  HBM-bound.
#include <cuda_runtime.h>

#include "common.cuh"
#include "tiles.h"

namespace vsa {

template <bool GATHER>
__global__ void __launch_bounds__(256)
tile_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, const Grid g,
                 const long long total_vec) {
    const int vpr = g.d / 8;                     // vectors per (slot, head) row
    const int vol = g.tt * g.th * g.tw;
    for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < total_vec;
         v += (long long)gridDim.x * blockDim.x) {
        // cube-major index: (((b*heads + head)*nt + j)*vol + s)*vpr + c
        const int c = (int)(v % vpr);
        long long rest = v / vpr;
        const int s = (int)(rest % vol); rest /= vol;
        const int j = (int)(rest % g.nt); rest /= g.nt;
        const int head = (int)(rest % g.heads);
        const int b = (int)(rest / g.heads);
        const int it = j / (g.nh * g.nw), ih = (j / g.nw) % g.nh, iw = j % g.nw;
        const int dt = s / (g.th * g.tw), dh = (s / g.tw) % g.th, dw = s % g.tw;
        const int t = it * g.tt + dt, h = ih * g.th + dh, w = iw * g.tw + dw;
        const bool valid = t < g.T && h < g.H && w < g.W;
        const long long n = ((long long)t * g.H + h) * g.W + w;
        const long long gi = (((long long)b * g.N + n) * g.heads + head) * vpr + c;
        if (GATHER) {
            dst[v] = valid ? __ldg(src + gi) : make_uint4(0, 0, 0, 0);
        } else if (valid) {
            dst[gi] = __ldg(src + v);
        }
    }
}

static unsigned copy_blocks(long long total_vec) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (total_vec + 255) / 256;
    const long long cap = (long long)sms * 8;     // 8 resident CTAs of 256 threads per SM
    return (unsigned)(want < cap ? want : cap);
}

cudaError_t launch_gather(const Grid& g, const void* x, void* x_tiles, cudaStream_t stream) {
    const long long total = (long long)g.B * g.heads * g.nt * (g.tt * g.th * g.tw) * (g.d / 8);
    if (total == 0) return cudaSuccess;
    tile_copy_kernel<true><<<copy_blocks(total), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(x_tiles), g, total);
    return cudaGetLastError();
}

cudaError_t launch_scatter(const Grid& g, const void* x_tiles, void* x, cudaStream_t stream) {
    const long long total = (long long)g.B * g.heads * g.nt * (g.tt * g.th * g.tw) * (g.d / 8);
    if (total == 0) return cudaSuccess;
    tile_copy_kernel<false><<<copy_blocks(total), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(x_tiles), reinterpret_cast<uint4*>(x), g, total);
    return cudaGetLastError();
}

}  // namespace vsa
