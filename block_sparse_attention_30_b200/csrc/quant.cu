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
// One CTA per (q|k, b, cube) (and chunk of heads when there are many), each
// warp a pair of heads (d = 128) or four (d = 64): a warp-wide load is one
// token's consecutive head rows, so the CTA reads whole token rows.  Each
// warp streams the cube twice: once for the per-head maximum (lane
// reductions), once to convert; the second pass is served from L1.
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

// One CTA per (q|k, b, cube, chunk of up to 64 heads); warp w of the CTA
// takes heads 2w and 2w + 1 of the chunk (HPW heads per warp: 32 lanes = HPW
// heads x VPT 16-byte vectors), so each warp-wide load is HPW consecutive
// head rows of one token and the CTA reads whole token rows.
template <int D>
__global__ void __launch_bounds__(1024)
quant_e4m3_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const Grid g,
                  uint8_t* __restrict__ q8, uint8_t* __restrict__ k8, float* __restrict__ q_scale,
                  float* __restrict__ k_scale, const int head_chunks) {
    constexpr int VPT = D / 8;                         // 16-byte vectors per (token, head)
    constexpr int HPW = 32 / VPT;                      // heads per warp
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long r = blockIdx.x;
    const int hc = (int)(r % head_chunks);
    r /= head_chunks;
    const int j = (int)(r % g.nt);
    r /= g.nt;
    const int b = (int)(r % g.B);
    const bool is_k = r / g.B != 0;
    const int head = hc * (32 * HPW) + warp * HPW + lane / VPT;   // 32 warps x HPW heads per chunk
    const bool head_ok = head < g.heads;
    const int vec = lane % VPT;
    const uint16_t* x = is_k ? k : q;
    uint8_t* x8 = is_k ? k8 : q8;
    float* scales = is_k ? k_scale : q_scale;
    const TileCoord c = tile_coord(g, j);
    const uint64_t valid = valid_slot_mask(g, c);
    const bool t444 = g.tt == 4 && g.th == 4 && g.tw == 4;

    float amax = 0.f;
#pragma unroll 8
    for (int s = 0; s < 64; ++s) {
        if (!head_ok || !((valid >> s) & 1ull)) continue;
        const long long n = slot_token(g, c, s, t444);
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x + ((b * g.N + n) * g.heads + head) * D) + vec);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)),
                                     fabsf(__uint_as_float(w[e] & 0xffff0000u))));
    }
    // the VPT lanes of a head are consecutive
#pragma unroll
    for (int o = VPT / 2; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const float inv = __frcp_rn(scale);
    if (head_ok && vec == 0) scales[((long long)b * g.heads + head) * g.nt + j] = scale;
#pragma unroll 8
    for (int s = 0; s < 64; ++s) {
        if (!head_ok || !((valid >> s) & 1ull)) continue;
        const long long n = slot_token(g, c, s, t444);
        const long long row = (b * g.N + n) * g.heads + head;
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x + row * D) + vec);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float y[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            y[2 * e] = __fmul_rn(__uint_as_float(w[e] << 16), inv);
            y[2 * e + 1] = __fmul_rn(__uint_as_float(w[e] & 0xffff0000u), inv);
        }
        reinterpret_cast<uint2*>(x8 + row * D)[vec] = to_e4m3x8(y);
    }
}

cudaError_t launch_quant_e4m3(const Grid& g, const void* q, const void* k, void* q8, void* k8,
                              float* q_scale, float* k_scale, cudaStream_t stream) {
    const int hpw = 32 / (g.d / 8);                            // heads per warp
    const int per_chunk = 32 * hpw;                            // heads per CTA (at most 32 warps)
    const int head_chunks = (g.heads + per_chunk - 1) / per_chunk;
    const int heads_in_cta = g.heads < per_chunk ? g.heads : per_chunk;
    const int threads = 32 * ((heads_in_cta + hpw - 1) / hpw);
    const unsigned ctas = (unsigned)(2ll * g.B * g.nt * head_chunks);
    if (g.d == 128)
        quant_e4m3_kernel<128><<<ctas, threads, 0, stream>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), g,
            static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), q_scale, k_scale, head_chunks);
    else
        quant_e4m3_kernel<64><<<ctas, threads, 0, stream>>>(
            static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), g,
            static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), q_scale, k_scale, head_chunks);
    return cudaGetLastError();
}

}  // namespace vsa
