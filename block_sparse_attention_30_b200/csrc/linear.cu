// linear.cu -- state of the linear-attention branch on sm_100a.
//
// Source: SparkDiffusion news item (bazainvestora.ru), paragraph 3 -- RoLA
// pairs the block-sparse branch with a low-rank linear branch that keeps
// global context -- and the TurboDiffusion article (dolphinsci.com), section
// "稀疏、蒸馏与全链路量化" -- SLA = sparse attention + linear attention.  With
// the feature map phi(x) = elu(x) + 1 the branch needs, per (b, head),
//     S = sum_n phi(k_n)^T v_n   (d x d)   and   z = sum_n phi(k_n)   (d),
// summed over every token of the grid, with fp32 accumulation.
//
// S is a GEMM with a long reduction (the tokens), done on the tensor cores:
// per 64-token step, TMA brings K and V (box: 64 features x 64 tokens of one
// head, 128-byte swizzle); 128 threads turn K into phi(K) split into bf16
// hi + lo parts (phi(k) = hi + lo to ~2^-17) written in place of the tile's
// layout, and accumulate z in fp32; one thread issues
//     S(TMEM, M = d features a, N = d features c) += phi_hi^T V + phi_lo^T V
// (A = phi(K)^T and B = V, both read MN-major from shared memory, M = 128).
// Four 48 KB stages (phi hi overwrites K in place) keep three steps of loads
// in flight while step t is computed.  At the
// end each CTA adds its partial S (read from TMEM) and z into the zeroed
// outputs with fp32 atomics, so the summation order across CTAs varies from
// run to run at the fp32 rounding level.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "linear.h"
#include "sm100.cuh"

namespace vsa {
using namespace sm100;

template <int D>
struct LinCfg {
    static constexpr int NCH = D / 64;                    // 64-feature chunks
    static constexpr int TILE = 64 * D * 2;               // one 64-token tile (bf16)
    static constexpr int STAGE = 3 * TILE;                // K -> phi hi (in place), V, phi lo
    static constexpr int NST = 4;
    static constexpr int BAR_BYTES = 128;
    static constexpr int SMEM_BYTES = NST * STAGE + BAR_BYTES;
    static constexpr int TMEM_COLS = D < 32 ? 32 : D;     // fp32 accumulator, D columns
};

template <int D>
struct LinBars {
    uint64_t full[LinCfg<D>::NST];       // K and V of a stage landed
    uint64_t ready[LinCfg<D>::NST];      // phi hi/lo written (128 arrivals)
    uint64_t done[LinCfg<D>::NST];       // MMAs of a stage finished
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ float phi_elu1(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// Fire-and-forget vector add of four floats into global memory (16-byte aligned).
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// grid: (chunks, B*heads); 160 threads: warps 0-3 transform K, warp 4 = TMA + MMA.
template <int D>
__global__ void __launch_bounds__(160, 1)
linear_state_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                    const Grid g, const int tokens_per_cta, float* __restrict__ S,
                    float* __restrict__ z, int* status) {
    using C = LinCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    LinBars<D>* bars = reinterpret_cast<LinBars<D>*>(smem + C::NST * C::STAGE);
    volatile int* abort_flag = &bars->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y, b = bh / g.heads, head = bh % g.heads;
    const long long n_begin = (long long)blockIdx.x * tokens_per_cta;
    const long long n_end = min(n_begin + tokens_per_cta, g.N);
    const int n_steps = (int)((n_end - n_begin + 63) / 64);

    if (tid == 0) {
        bars->abort = 0;
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->ready[s], 128);
            mbar_init(&bars->done[s], 1);
        }
        fence_barrier_init();
    }
    if (warp == 4) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;
    auto stage_ptr = [&](int s, int part) { return smem + s * C::STAGE + part * C::TILE; };
    auto fail = [&]() { *abort_flag = 1; report(status, kStatusTimeout); };

    if (warp == 4) {
        if (lane == 0) {
            // ------------------------------------------------- loads + MMAs
            const uint32_t id = idesc_bf16_f32(D, D, true, true);
            bool ok = true;
            auto load = [&](int t) {
                const int s = t % C::NST;
                const int n0 = (int)(n_begin + 64ll * t);
                mbar_arrive_expect_tx(&bars->full[s], 2 * C::TILE);
                for (int c = 0; c < C::NCH; ++c) {
                    tma_load_3d(stage_ptr(s, 0) + c * 8192, &mk, &bars->full[s], head * D + 64 * c, n0, b);
                    tma_load_3d(stage_ptr(s, 1) + c * 8192, &mv, &bars->full[s], head * D + 64 * c, n0, b);
                }
            };
            for (int t = 0; t < min(C::NST, n_steps); ++t) load(t);
            for (int t = 0; t < n_steps && ok; ++t) {
                const int s = t % C::NST;
                const uint32_t ph = (uint32_t)((t / C::NST) & 1);
                if (!mbar_wait_spin(&bars->ready[s], ph, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t v_addr = smem_u32(stage_ptr(s, 1));
#pragma unroll
                for (int part = 0; part < 3; part += 2) {     // phi hi (part 0), phi lo (part 2)
                    const uint32_t a_addr = smem_u32(stage_ptr(s, part));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {         // 16 tokens per MMA
                        const uint64_t a = smem_desc_sw128(a_addr + kk * 2048, 8192, 1024);
                        const uint64_t bd = smem_desc_sw128(v_addr + kk * 2048, 8192, 1024);
                        mma_bf16_ss(tbase, a, bd, id, (t > 0 || part > 0 || kk > 0));
                    }
                }
                mma_commit(&bars->done[s]);
                // refill the stage of step t-1 (its MMAs ran before these) with step t-1+NST
                const int tr = t - 1 + C::NST;
                if (t >= 1 && tr < n_steps) {
                    const int sp = (t - 1) % C::NST;
                    if (!mbar_wait_spin(&bars->done[sp], (uint32_t)(((t - 1) / C::NST) & 1), abort_flag)) { ok = false; break; }
                    load(tr);
                }
            }
            if (!ok) fail();
            // all MMAs done (the last commit covers every earlier MMA)
            if (n_steps > 0) wait_noabort(&bars->done[(n_steps - 1) % C::NST], ((n_steps - 1) / C::NST) & 1);
        }
    } else {
        // ------------------------------------------- phi(K) hi/lo and z (fp32)
        // thread -> 16-byte column unit u (8 features) and token rows r0 + 8i
        const int u = tid % (D / 8), r0 = tid / (D / 8);
        const int rows_per_pass = 128 / (D / 8);           // 8 for D = 128, 16 for D = 64
        const int chunk = u / 8, uu = u % 8;
        float zacc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
        bool ok = true;
        for (int t = 0; t < n_steps; ++t) {
            const int s = t % C::NST;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->full[s], (t / C::NST) & 1, abort_flag))) { ok = false; break; }
            const int valid = (int)min(64ll, n_end - (n_begin + 64ll * t));
            const uint8_t* kt = stage_ptr(s, 0);
            uint8_t* hi = stage_ptr(s, 0);                  // in place: each thread rewrites its own units
            uint8_t* lo = stage_ptr(s, 2);
            for (int r = r0; r < 64; r += rows_per_pass) {
                const uint32_t off = chunk * 8192 + r * 128 + ((uu ^ (r & 7)) << 4);
                uint4 raw = *reinterpret_cast<const uint4*>(kt + off);
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t h[4], l[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // rows past the end of the grid hold zero-filled K: phi(0) = 1
                    // must not count, so their phi is forced to 0
                    const float f0 = r < valid ? phi_elu1(__uint_as_float(w[e] << 16)) : 0.f;
                    const float f1 = r < valid ? phi_elu1(__uint_as_float(w[e] & 0xffff0000u)) : 0.f;
                    zacc[2 * e] += f0;
                    zacc[2 * e + 1] += f1;
                    const uint32_t ph = pack_bf16x2(f0, f1);
                    h[e] = ph;
                    l[e] = pack_bf16x2(f0 - __uint_as_float(ph << 16), f1 - __uint_as_float(ph & 0xffff0000u));
                }
                *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->ready[s]);
            // the MMA thread reuses stage s only after its MMAs finished
        }
        if (!ok) fail();
        // z: add this thread's 8 partial sums
        float* zb = z + (long long)bh * D + u * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) atomicAdd(zb + e, zacc[e]);
        // S partial from TMEM: warp w reads lanes 32w..32w+31 (= feature a)
        if (ok && n_steps > 0) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->done[(n_steps - 1) % C::NST], ((n_steps - 1) / C::NST) & 1, abort_flag))) ok = false;
        }
        if (ok && n_steps > 0) {
            // M = 128: feature a in lane a; M = 64: feature a in lane (a % 16) + 32 (a / 16)
            tc_fence_after();
            const int a = D == 128 ? 32 * warp + lane : 16 * warp + lane;
            const bool mine = D == 128 || lane < 16;
            float* Sb = S + ((long long)bh * D + a) * D;
            for (int c0 = 0; c0 < D; c0 += 16) {
                float vals[16];
                tmem_ld_32x32b_x16(tbase + ((uint32_t)(32 * warp) << 16) + c0, vals);
                tmem_wait_ld();
                if (mine) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4) red_add_v4(Sb + c0 + e, vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 4) tmem_dealloc(tbase, C::TMEM_COLS);
}

// 3-D view (heads*d, N, B) of a [B][N][heads][d] bf16 tensor; box = 64
// features x 64 tokens of one batch, 128-byte swizzle; tokens past N are
// zero-filled.
static bool encode_token_map(CUtensorMap* m, const void* base, const Grid& g,
                             PFN_cuTensorMapEncodeTiled_v12000 fn) {
    const cuuint64_t row = (cuuint64_t)g.heads * g.d;
    cuuint64_t dims[3] = {row, (cuuint64_t)g.N, (cuuint64_t)g.B};
    cuuint64_t strides[2] = {row * 2, row * 2 * (cuuint64_t)g.N};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_linear_impl(const Grid& g, const void* k, const void* v, float* S,
                                      float* z, int* status, cudaStream_t stream,
                                      PFN_cuTensorMapEncodeTiled_v12000 enc) {
    using C = LinCfg<D>;
    static int configured_device = -1;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(linear_state_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    CUtensorMap mk, mv;
    if (!encode_token_map(&mk, k, g, enc) || !encode_token_map(&mv, v, g, enc)) return cudaErrorInvalidValue;
    e = cudaMemsetAsync(S, 0, sizeof(float) * g.B * g.heads * g.d * g.d, stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(z, 0, sizeof(float) * g.B * g.heads * g.d, stream);
    if (e != cudaSuccess) return e;
    // at most one wave (one CTA per SM) over all (b, head), whole 64-token steps per CTA
    const long long bh = (long long)g.B * g.heads;
    long long chunks = sms / bh > 0 ? sms / bh : 1;
    long long per = (g.N + chunks - 1) / chunks;
    per = ((per + 63) / 64) * 64;
    chunks = (g.N + per - 1) / per;
    linear_state_kernel<D><<<dim3((unsigned)chunks, (unsigned)bh), 160, C::SMEM_BYTES, stream>>>(
        mk, mv, g, (int)per, S, z, status);
    return cudaGetLastError();
}

cudaError_t launch_linear_state(const Grid& g, const void* k, const void* v, float* S, float* z,
                                int* status, cudaStream_t stream,
                                PFN_cuTensorMapEncodeTiled_v12000 enc) {
    if (g.d == 128) return launch_linear_impl<128>(g, k, v, S, z, status, stream, enc);
    return launch_linear_impl<64>(g, k, v, S, z, status, stream, enc);
}

}  // namespace vsa
