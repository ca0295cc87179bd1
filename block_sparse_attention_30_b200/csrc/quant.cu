// quant.cu -- per-cube FP8 E4M3 quantisation of q and k for the
// low-precision fine pass.
//
// Source: TurboDiffusion article (dolphinsci.com), section
// "稀疏、蒸馏与全链路量化": sparse attention is orthogonal to low-bit tensor
// cores (SageSLA, built on SageAttention's quantised attention products).
// Reading: one fp32 scale per (b, head, cube) = amax / 448 over the cube's
// valid tokens and all d features (1 for an all-zero cube), codes =
// E4M3(x / scale) rounded to nearest-even with saturation at 448 (the largest
// finite E4M3 value), the division in IEEE fp32.  Codes keep the
// [B][N][heads][d] layout (one byte per element) so the fine kernel's 5-D
// TMA boxes cut cubes out of them exactly as out of the bf16 tensors.
//
// One CTA per (cube, batch, group of 4 heads, q|k), 256 threads: each thread
// holds its 16-byte vectors of the cube's tokens in registers, so the data is
// read once; the cube maximum of each head is reduced over the threads that
// share the head (shuffles, then shared memory across token groups).
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "quant.h"

namespace vsa {

template <int D>
struct QuantCfg {
    static constexpr int HG = 4;                       // heads per CTA
    static constexpr int VPT = D / 8;                  // 16-byte vectors per (token, head)
    static constexpr int VPR = HG * VPT;               // vectors per token row of the group
    static constexpr int TG = 256 / VPR;               // token groups
    static constexpr int TPT = 64 / TG;                // tokens per thread
};

// 8 floats -> 8 E4M3 codes (nearest-even, saturating), packed little-endian.
__device__ __forceinline__ uint2 to_e4m3x8(const float (&y)[8]) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(y[4 * h], y[4 * h + 1]), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(y[4 * h + 2], y[4 * h + 3]), __NV_SATFINITE, __NV_E4M3);
        w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    return make_uint2(w[0], w[1]);
}

template <int D>
__global__ void __launch_bounds__(256)
quant_e4m3_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const Grid g,
                  uint8_t* __restrict__ q8, uint8_t* __restrict__ k8, float* __restrict__ q_scale,
                  float* __restrict__ k_scale) {
    using C = QuantCfg<D>;
    __shared__ float part[C::TG][C::HG];
    const int j = blockIdx.x;
    const int hgroups = (g.heads + C::HG - 1) / C::HG;
    const int b = blockIdx.y / hgroups, h0 = (blockIdx.y % hgroups) * C::HG;
    const bool is_k = blockIdx.z != 0;
    const uint16_t* x = is_k ? k : q;
    uint8_t* x8 = is_k ? k8 : q8;
    float* scales = is_k ? k_scale : q_scale;
    const int tid = threadIdx.x;
    const int v = tid % C::VPR, tg = tid / C::VPR;     // vector of the row, token group
    const int hl = v / C::VPT, head = h0 + hl;         // head of this vector
    const bool head_ok = head < g.heads;
    const TileCoord c = tile_coord(g, j);
    const uint64_t valid = valid_slot_mask(g, c);

    uint4 raw[C::TPT];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < C::TPT; ++i) {
        const int s = tg + C::TG * i;                  // cube slot
        raw[i] = make_uint4(0, 0, 0, 0);
        if (head_ok && ((valid >> s) & 1ull)) {
            const int dt = s / (g.th * g.tw), dh = (s / g.tw) % g.th, dw = s % g.tw;
            const long long n = ((long long)(c.t0 + dt) * g.H + (c.h0 + dh)) * g.W + (c.w0 + dw);
            raw[i] = __ldg(reinterpret_cast<const uint4*>(x + ((b * g.N + n) * g.heads + head) * D) +
                           (v % C::VPT));
        }
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)),
                                     fabsf(__uint_as_float(w[e] & 0xffff0000u))));
    }
    // the VPT threads of a (token group, head) are consecutive lanes
#pragma unroll
    for (int o = C::VPT / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (v % C::VPT == 0) part[tg][hl] = amax;
    __syncthreads();
    float m = 0.f;
#pragma unroll
    for (int t = 0; t < C::TG; ++t) m = fmaxf(m, part[t][hl]);
    const float scale = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
    if (head_ok && tg == 0 && v % C::VPT == 0) scales[((long long)b * g.heads + head) * g.nt + j] = scale;
#pragma unroll
    for (int i = 0; i < C::TPT; ++i) {
        const int s = tg + C::TG * i;
        if (!head_ok || !((valid >> s) & 1ull)) continue;
        const int dt = s / (g.th * g.tw), dh = (s / g.tw) % g.th, dw = s % g.tw;
        const long long n = ((long long)(c.t0 + dt) * g.H + (c.h0 + dh)) * g.W + (c.w0 + dw);
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
        float y[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            y[2 * e] = __fdiv_rn(__uint_as_float(w[e] << 16), scale);
            y[2 * e + 1] = __fdiv_rn(__uint_as_float(w[e] & 0xffff0000u), scale);
        }
        reinterpret_cast<uint2*>(x8 + ((b * g.N + n) * g.heads + head) * D)[v % C::VPT] = to_e4m3x8(y);
    }
}

cudaError_t launch_quant_e4m3(const Grid& g, const void* q, const void* k, void* q8, void* k8,
                              float* q_scale, float* k_scale, cudaStream_t stream) {
    const dim3 grid((unsigned)g.nt, (unsigned)(g.B * ((g.heads + 3) / 4)), 2);
    if (g.d == 128)
        quant_e4m3_kernel<128><<<grid, 256, 0, stream>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), g,
            static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), q_scale, k_scale);
    else
        quant_e4m3_kernel<64><<<grid, 256, 0, stream>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), g,
            static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), q_scale, k_scale);
    return cudaGetLastError();
}

}  // namespace vsa
