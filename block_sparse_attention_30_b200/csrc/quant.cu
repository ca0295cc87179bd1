// quant.cu -- per-cube FP8 E4M3 quantisation of q and k for the
// low-precision fine pass.
//
// Source: TurboDiffusion article (dolphinsci.com), section
// "稀疏、蒸馏与全链路量化": sparse attention is orthogonal to low-bit tensor
// cores (SageSLA, built on SageAttention's quantised attention products).
// Reading: one fp32 scale per (b, head, cube) = amax / 448 over the cube's
// valid tokens and all d features (1 for an all-zero cube), codes =
// E4M3(x * inv) with inv = 1 / scale, both rounded to nearest fp32, the
// conversion rounded to nearest-even with saturation at 448 (the largest
// finite E4M3 value).  Codes keep the [B][N][heads][d] layout (one byte per
// element) so the fine kernel's 5-D TMA boxes cut cubes out of them exactly
// as out of the bf16 tensors.
//
// Each CTA holds its part of a cube in registers between the maximum and the
// conversion, so q and k are read from HBM once.  (A version that streamed
// each cube twice lost the second pass to L2 evictions: with every SM busy
// the data in flight between the passes exceeds L2.)
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "quant.h"

namespace vsa {

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

// Token of cube slot s (the cube's origin c), with a shift-only path for the
// 4 x 4 x 4 tile.
__device__ __forceinline__ long long slot_token(const Grid& g, const TileCoord& c, int s, bool t444) {
    int dt, dh, dw;
    if (t444) { dt = s >> 4; dh = (s >> 2) & 3; dw = s & 3; }
    else { dt = s / (g.th * g.tw); dh = (s / g.tw) % g.th; dw = s % g.tw; }
    return ((long long)(c.t0 + dt) * g.H + (c.h0 + dh)) * g.W + (c.w0 + dw);
}

// One CTA per (q|k, b, cube, group of HG heads), 256 threads: thread t holds
// vector t % 32 of the group's token-row chunk (HG heads x D/8 vectors, 512
// bytes, contiguous) for 8 of the cube's 64 slots in registers, so the data
// is read from HBM once and several CTAs fit on an SM.  The cube maximum of a
// head is reduced over its lanes (shuffles), then over the 8 token groups
// (shared memory).
template <int D>
struct QuantCfg {
    static constexpr int VPT = D / 8;                  // 16-byte vectors per (token, head)
    static constexpr int HG = 32 / VPT;                // heads per CTA (one warp-wide row chunk)
    static constexpr int TG = 256 / 32;                // token groups (one per warp)
    static constexpr int TPT = 64 / TG;                // slots per thread
};

template <int D>
__global__ void __launch_bounds__(256, 3)
quant_e4m3_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const Grid g,
                  uint8_t* __restrict__ q8, uint8_t* __restrict__ k8, float* __restrict__ q_scale,
                  float* __restrict__ k_scale, const int head_groups) {
    using C = QuantCfg<D>;
    __shared__ float part[C::TG][C::HG];
    const int lane = threadIdx.x & 31, tg = threadIdx.x >> 5;
    long long r = blockIdx.x;
    const int hgi = (int)(r % head_groups);
    r /= head_groups;
    const int j = (int)(r % g.nt);
    r /= g.nt;
    const int b = (int)(r % g.B);
    const bool is_k = r / g.B != 0;
    const int hl = lane / C::VPT, vec = lane % C::VPT;
    const int head = hgi * C::HG + hl;
    const bool head_ok = head < g.heads;
    const uint16_t* x = is_k ? k : q;
    uint8_t* x8 = is_k ? k8 : q8;
    float* scales = is_k ? k_scale : q_scale;
    const TileCoord c = tile_coord(g, j);
    const uint64_t valid = valid_slot_mask(g, c);
    const bool t444 = g.tt == 4 && g.th == 4 && g.tw == 4;

    uint4 raw[C::TPT];
    int tok[C::TPT];                                   // token of each slot, -1 if not held
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < C::TPT; ++i) {
        const int s = tg + C::TG * i;
        const bool ok = head_ok && ((valid >> s) & 1ull);
        tok[i] = ok ? (int)slot_token(g, c, s, t444) : -1;
        raw[i] = ok ? __ldg(reinterpret_cast<const uint4*>(x + ((b * g.N + tok[i]) * g.heads + head) * D) + vec)
                    : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < C::TPT; ++i) {
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)),
                                     fabsf(__uint_as_float(w[e] & 0xffff0000u))));
    }
    // the VPT lanes of a head are consecutive
#pragma unroll
    for (int o = C::VPT / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (vec == 0) part[tg][hl] = amax;
    __syncthreads();
    float m = 0.f;
#pragma unroll
    for (int t = 0; t < C::TG; ++t) m = fmaxf(m, part[t][hl]);
    const float scale = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
    const float inv = __frcp_rn(scale);
    if (head_ok && tg == 0 && vec == 0) scales[((long long)b * g.heads + head) * g.nt + j] = scale;
#pragma unroll
    for (int i = 0; i < C::TPT; ++i) {
        if (tok[i] < 0) continue;
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
        float y[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            y[2 * e] = __fmul_rn(__uint_as_float(w[e] << 16), inv);
            y[2 * e + 1] = __fmul_rn(__uint_as_float(w[e] & 0xffff0000u), inv);
        }
        reinterpret_cast<uint2*>(x8 + ((b * g.N + tok[i]) * g.heads + head) * D)[vec] = to_e4m3x8(y);
    }
}

cudaError_t launch_quant_e4m3(const Grid& g, const void* q, const void* k, void* q8, void* k8,
                              float* q_scale, float* k_scale, cudaStream_t stream) {
    const int hg = 32 / (g.d / 8);                             // heads per CTA
    const int head_groups = (g.heads + hg - 1) / hg;
    const unsigned ctas = (unsigned)(2ll * g.B * g.nt * head_groups);
    if (g.d == 128)
        quant_e4m3_kernel<128><<<ctas, 256, 0, stream>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), g,
            static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), q_scale, k_scale, head_groups);
    else
        quant_e4m3_kernel<64><<<ctas, 256, 0, stream>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), g,
            static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), q_scale, k_scale, head_groups);
    return cudaGetLastError();
}

}  // namespace vsa
