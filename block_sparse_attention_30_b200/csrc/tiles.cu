// tiles.cu -- cube-tile gather / scatter between grid order [B][N][heads][d]
// and cube-major [B][heads][nt][64][d] (bf16, bit-exact copies).
//
// The cube grouping is the tiling step behind "FastVideo 稀疏蒸馏技术深度解析"
// (omica.com.cn), section "2. 视频稀疏注意力VSA" (key blocks are spatio-temporal
// blocks of the video).  The fused forward path never materialises these
// layouts -- its TMA boxes cut cubes straight out of grid order -- but the
// copies are part of the library for callers that keep cube-major tensors.
//
// HBM-bound copies: every byte is read once and written once.
#include <cuda_runtime.h>

#include "common.cuh"
#include "tiles.h"

namespace vsa {

// One CTA per (cube j, batch b, group of kSlotsPerCta slots).  For each of its
// slots the token row -- all heads, heads*d bf16, contiguous in grid order --
// is copied with 16-byte vectors; in cube-major order the same vector lands
// in row ((b*heads + head)*nt + j)*vol + slot.  Consecutive threads take
// consecutive vectors of one row, so reads cover whole 128-byte lines of grid
// order and writes whole d-wide rows of cube-major order.  Four slots are in
// flight per thread; splitting a cube's slots over several CTAs gives the
// small grids (a few hundred cubes) enough CTAs to fill every SM.
constexpr int kSlotsPerCta = 16;

template <bool GATHER, int VPR>     // VPR: 16-byte vectors per (slot, head) row = d/8
__global__ void __launch_bounds__(256)
tile_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, const Grid g) {
    const int j = blockIdx.x, b = blockIdx.y;
    const int vol = g.tt * g.th * g.tw;
    const int it = j / (g.nh * g.nw), ih = (j / g.nw) % g.nh, iw = j % g.nw;
    const int row_vec = g.heads * VPR;                       // vectors per token row
    const int s_end = min(vol, ((int)blockIdx.z + 1) * kSlotsPerCta);
    for (int s0 = blockIdx.z * kSlotsPerCta; s0 < s_end; s0 += 4) {
        long long n[4];
        bool valid[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            const int dt = s / (g.th * g.tw), dh = (s / g.tw) % g.th, dw = s % g.tw;
            const int t = it * g.tt + dt, h = ih * g.th + dh, w = iw * g.tw + dw;
            valid[u] = s < s_end && t < g.T && h < g.H && w < g.W;
            n[u] = ((long long)t * g.H + h) * g.W + w;
        }
        for (int v = threadIdx.x; v < row_vec; v += blockDim.x) {
            const int head = v / VPR, c = v % VPR;
            const long long tile_row = (((long long)b * g.heads + head) * g.nt + j) * vol;
            uint4 val[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const long long gi = ((long long)b * g.N + n[u]) * row_vec + v;
                const long long ti = (tile_row + s0 + u) * VPR + c;
                if (GATHER) val[u] = valid[u] ? __ldg(src + gi) : make_uint4(0, 0, 0, 0);
                else val[u] = valid[u] ? __ldg(src + ti) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (s0 + u >= s_end) continue;
                const long long gi = ((long long)b * g.N + n[u]) * row_vec + v;
                const long long ti = (tile_row + s0 + u) * VPR + c;
                if (GATHER) dst[ti] = val[u];
                else if (valid[u]) dst[gi] = val[u];
            }
        }
    }
}

template <bool GATHER>
static cudaError_t launch_copy(const Grid& g, const void* src, void* dst, cudaStream_t stream) {
    if ((long long)g.B * g.nt == 0) return cudaSuccess;
    const dim3 grid(g.nt, g.B, ceil_div_i(g.tt * g.th * g.tw, kSlotsPerCta));
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst);
    if (g.d == 128) tile_copy_kernel<GATHER, 16><<<grid, 256, 0, stream>>>(s, d, g);
    else tile_copy_kernel<GATHER, 8><<<grid, 256, 0, stream>>>(s, d, g);
    return cudaGetLastError();
}

cudaError_t launch_gather(const Grid& g, const void* x, void* x_tiles, cudaStream_t stream) {
    return launch_copy<true>(g, x, x_tiles, stream);
}

cudaError_t launch_scatter(const Grid& g, const void* x_tiles, void* x, cudaStream_t stream) {
    return launch_copy<false>(g, x_tiles, x, stream);
}

}  // namespace vsa
