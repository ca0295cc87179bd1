// linear.cu -- state of the linear-attention branch on sm_100a.
//
// Source: SparkDiffusion news item (bazainvestora.ru), paragraph 3 -- RoLA
// pairs the block-sparse branch with a low-rank linear branch that keeps
// global context -- and the TurboDiffusion article (dolphinsci.com), section
// "稀疏、蒸馏与全链路量化" -- SLA = sparse attention + linear attention.  With
// the feature map phi(x) = elu(x) + 1 the branch needs, per (b, head),
//     S = sum_n phi(k_n)^T v_n   (d x d)   and   z = sum_n phi(k_n)   (d),
// summed over every token of the grid, in fp32.
//
// One CTA per (chunk of 1024 tokens, b*heads): 32-token slices of phi(K) and
// V are staged in shared memory as fp32, each of the 256 threads accumulates
// a (d/16) x (d/16) block of S in registers, and the chunk's partial S and z
// are added into the (zeroed) outputs with fp32 atomics.  Summation order
// across chunks therefore varies from run to run at the fp32 rounding level.
#include <cuda_runtime.h>

#include "common.cuh"
#include "linear.h"

namespace vsa {

constexpr int kLinChunk = 1024;
constexpr int kLinSlice = 32;

__device__ __forceinline__ float phi_elu1(float x) { return x > 0.f ? x + 1.f : __expf(x); }

template <int D>
__global__ void __launch_bounds__(256)
linear_state_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, const Grid g,
                    float* __restrict__ S, float* __restrict__ z) {
    constexpr int R = D / 16;                       // rows / cols of S per thread
    __shared__ float sk[kLinSlice][D + 4];
    __shared__ float sv[kLinSlice][D + 4];
    const int bh = blockIdx.y, b = bh / g.heads, head = bh % g.heads;
    const long long n_begin = (long long)blockIdx.x * kLinChunk;
    const long long n_end = min(n_begin + kLinChunk, g.N);
    const int ta = threadIdx.x / 16, tc = threadIdx.x % 16;
    float acc[R][R];
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
        for (int c = 0; c < R; ++c) acc[a][c] = 0.f;
    float zacc = 0.f;
    for (long long n0 = n_begin; n0 < n_end; n0 += kLinSlice) {
        const int cnt = (int)min((long long)kLinSlice, n_end - n0);
        // stage: 8 bf16 per thread-step, phi applied to k
        for (int l = threadIdx.x; l < kLinSlice * (D / 8); l += 256) {
            const int tok = l / (D / 8), u = l % (D / 8);
            float kf[8], vf[8];
            if (tok < cnt) {
                const long long off = (((long long)b * g.N + n0 + tok) * g.heads + head) * D + u * 8;
                const uint4 rk = __ldg(reinterpret_cast<const uint4*>(k + off));
                const uint4 rv = __ldg(reinterpret_cast<const uint4*>(v + off));
                const uint32_t wk[4] = {rk.x, rk.y, rk.z, rk.w}, wv[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[2 * e] = phi_elu1(__uint_as_float(wk[e] << 16));
                    kf[2 * e + 1] = phi_elu1(__uint_as_float(wk[e] & 0xffff0000u));
                    vf[2 * e] = __uint_as_float(wv[e] << 16);
                    vf[2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) { kf[e] = 0.f; vf[e] = 0.f; }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) { sk[tok][u * 8 + e] = kf[e]; sv[tok][u * 8 + e] = vf[e]; }
        }
        __syncthreads();
        for (int t = 0; t < cnt; ++t) {
            float ka[R], vc[R];
#pragma unroll
            for (int a = 0; a < R; ++a) ka[a] = sk[t][ta * R + a];
#pragma unroll
            for (int c = 0; c < R; ++c) vc[c] = sv[t][tc * R + c];
#pragma unroll
            for (int a = 0; a < R; ++a)
#pragma unroll
                for (int c = 0; c < R; ++c) acc[a][c] = fmaf(ka[a], vc[c], acc[a][c]);
        }
        if (threadIdx.x < D)
            for (int t = 0; t < cnt; ++t) zacc += sk[t][threadIdx.x];
        __syncthreads();
    }
    float* Sb = S + (long long)bh * D * D;
#pragma unroll
    for (int a = 0; a < R; ++a)
#pragma unroll
        for (int c = 0; c < R; ++c) atomicAdd(Sb + (ta * R + a) * D + tc * R + c, acc[a][c]);
    if (threadIdx.x < D) atomicAdd(z + (long long)bh * D + threadIdx.x, zacc);
}

cudaError_t launch_linear_state(const Grid& g, const void* k, const void* v, float* S, float* z,
                                cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(S, 0, sizeof(float) * g.B * g.heads * g.d * g.d, stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(z, 0, sizeof(float) * g.B * g.heads * g.d, stream);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((g.N + kLinChunk - 1) / kLinChunk), g.B * g.heads);
    const uint16_t* kk = reinterpret_cast<const uint16_t*>(k);
    const uint16_t* vv = reinterpret_cast<const uint16_t*>(v);
    if (g.d == 128) linear_state_kernel<128><<<grid, 256, 0, stream>>>(kk, vv, g, S, z);
    else linear_state_kernel<64><<<grid, 256, 0, stream>>>(kk, vv, g, S, z);
    return cudaGetLastError();
}

}  // namespace vsa
