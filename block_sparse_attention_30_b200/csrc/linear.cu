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
    static constexpr int NST = D == 128 ? 4 : 8;          // 192 KB of stages
    static constexpr int NTW = 8;                         // transform warps
    static constexpr int THREADS = 32 * (NTW + 1);        // + one TMA / MMA warp
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_BYTES = NST * STAGE + BAR_BYTES;
    static constexpr int TMEM_COLS = D < 32 ? 32 : D;     // fp32 accumulator, D columns
    static constexpr int UPR = D / 8;                     // 16-byte units per token row
    static constexpr int ROWS_PER_PASS = 32 * NTW / UPR;  // token rows one pass covers
};

template <int D>
struct LinBars {
    uint64_t full[LinCfg<D>::NST];       // K and V of a stage landed
    uint64_t ready[LinCfg<D>::NST];      // phi hi/lo written (transform threads)
    uint64_t done[LinCfg<D>::NST];       // MMAs of a stage finished
    uint64_t seg_done;                   // MMAs of one (b, head) segment finished
    uint64_t mma_idle;                   // every MMA of the CTA finished
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(LinBars<64>) <= LinCfg<64>::BAR_BYTES, "barrier block");
static_assert(sizeof(LinBars<128>) <= LinCfg<128>::BAR_BYTES, "barrier block");

// Where 64-token step gs of the flattened (b*heads, step) space lives.
struct LinStep {
    int bh, st;       // (b, head) pair and 64-token step within it
    bool first, last; // first / last step of this CTA's segment of bh
};

// grid: one CTA per slice of the flattened (b*heads, 64-token step) space;
// warps 0..NTW-1 transform K, warp NTW = TMA + MMA.  A CTA's slice may cross
// (b, head) boundaries: at the end of each (b, head) segment the transform
// warps read the accumulator out of TMEM and add it to S (and z) with
// vector reductions, and the next segment starts a fresh accumulation.
template <int D>
__global__ void __launch_bounds__(LinCfg<D>::THREADS, 1)
linear_state_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                    const Grid g, const int steps_per_head, const long long total_steps,
                    const int steps_per_cta, float* __restrict__ S, float* __restrict__ z,
                    int* status) {
    using C = LinCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    LinBars<D>* bars = reinterpret_cast<LinBars<D>*>(smem + C::NST * C::STAGE);
    volatile int* abort_flag = &bars->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long gs0 = (long long)blockIdx.x * steps_per_cta;
    const int n_steps = (int)max(0ll, min((long long)steps_per_cta, total_steps - gs0));
    auto step_of = [&](int t) {
        LinStep x;
        const long long gs = gs0 + t;
        x.bh = (int)(gs / steps_per_head);
        x.st = (int)(gs - (long long)x.bh * steps_per_head);
        x.first = t == 0 || x.st == 0;
        x.last = t == n_steps - 1 || x.st == steps_per_head - 1;
        return x;
    };

    if (tid == 0) {
        bars->abort = 0;
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->ready[s], 32 * C::NTW);
            mbar_init(&bars->done[s], 1);
        }
        mbar_init(&bars->seg_done, 1);
        mbar_init(&bars->mma_idle, 1);
        fence_barrier_init();
    }
    if (warp == C::NTW) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;
    auto stage_ptr = [&](int s, int part) { return smem + s * C::STAGE + part * C::TILE; };
    auto fail = [&]() { *abort_flag = 1; report(status, kStatusTimeout); };

    if (warp == C::NTW) {
        if (lane == 0) {
            // ------------------------------------------------- loads + MMAs
            const uint32_t id = idesc_bf16_f32(D, D, true, true);
            bool ok = true;
            int issued = 0;
            auto load = [&](int t) {
                const int s = t % C::NST;
                const LinStep x = step_of(t);
                const int b = x.bh / g.heads, head = x.bh % g.heads;
                mbar_arrive_expect_tx(&bars->full[s], 2 * C::TILE);
                for (int c = 0; c < C::NCH; ++c) {
                    tma_load_3d(stage_ptr(s, 0) + c * 8192, &mk, &bars->full[s], head * D + 64 * c, 64 * x.st, b);
                    tma_load_3d(stage_ptr(s, 1) + c * 8192, &mv, &bars->full[s], head * D + 64 * c, 64 * x.st, b);
                }
                ++issued;
            };
            for (int t = 0; t < min(C::NST, n_steps); ++t) load(t);
            for (int t = 0; t < n_steps && ok; ++t) {
                const int s = t % C::NST;
                const LinStep x = step_of(t);
                if (!mbar_wait_spin(&bars->ready[s], (uint32_t)((t / C::NST) & 1), abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t v_addr = smem_u32(stage_ptr(s, 1));
#pragma unroll
                for (int part = 0; part < 3; part += 2) {     // phi hi (part 0), phi lo (part 2)
                    const uint32_t a_addr = smem_u32(stage_ptr(s, part));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {         // 16 tokens per MMA
                        const uint64_t a = smem_desc_sw128(a_addr + kk * 2048, 8192, 1024);
                        const uint64_t bd = smem_desc_sw128(v_addr + kk * 2048, 8192, 1024);
                        mma_bf16_ss(tbase, a, bd, id, !(x.first && part == 0 && kk == 0));
                    }
                }
                mma_commit(&bars->done[s]);
                if (x.last) mma_commit(&bars->seg_done);
                // refill the stage of step t-1 (its MMAs ran before these) with step t-1+NST
                const int tr = t - 1 + C::NST;
                if (t >= 1 && tr < n_steps) {
                    const int sp = (t - 1) % C::NST;
                    if (!mbar_wait_spin(&bars->done[sp], (uint32_t)(((t - 1) / C::NST) & 1), abort_flag)) { ok = false; break; }
                    load(tr);
                }
            }
            if (!ok) {
                fail();
                // drain: the last load issued into each stage must land before exit
                for (int n = max(0, issued - C::NST); n < issued; ++n)
                    wait_noabort(&bars->full[n % C::NST], (n / C::NST) & 1);
            }
            mma_commit(&bars->mma_idle);
            wait_noabort(&bars->mma_idle, 0);
        }
    } else {
        // ------------------------------------------- phi(K) hi/lo and z (fp32)
        // thread -> 16-byte column unit u (8 features) and token rows r0 + k*ROWS_PER_PASS
        const int u = tid % C::UPR, r0 = tid / C::UPR;
        const int chunk = u / 8, uu = u % 8;
        float zacc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
        const uint64_t one2 = f32x2(1.f, 1.f);
        const float log2e = 1.4426950408889634f;
        bool ok = true;
        int seg = 0;
        for (int t = 0; t < n_steps; ++t) {
            const int s = t % C::NST;
            const LinStep x = step_of(t);
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->full[s], (t / C::NST) & 1, abort_flag))) { ok = false; break; }
            const int valid = (int)min(64ll, g.N - 64ll * x.st);
            uint8_t* kt = stage_ptr(s, 0);                  // phi hi is written in place
            uint8_t* lo = stage_ptr(s, 2);
#pragma unroll
            for (int k = 0; k < 64 / C::ROWS_PER_PASS; ++k) {
                const int r = r0 + k * C::ROWS_PER_PASS;
                const uint32_t off = chunk * 8192 + r * 128 + ((uu ^ (r & 7)) << 4);
                const uint4 raw = *reinterpret_cast<const uint4*>(kt + off);
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t h[4], l[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // phi(x) = elu(x) + 1 = max(x + 1, e^min(x, 0)), because
                    // e^x >= 1 + x everywhere; zero-filled rows past the end
                    // of the grid would give phi(0) = 1 and are forced to 0
                    const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
                    float p0, p1;
                    unf32x2(add_f32x2(f32x2(x0, x1), one2), p0, p1);
                    float f0 = fmaxf(p0, ex2(fminf(x0, 0.f) * log2e));
                    float f1 = fmaxf(p1, ex2(fminf(x1, 0.f) * log2e));
                    if (r >= valid) { f0 = 0.f; f1 = 0.f; }
                    zacc[2 * e] += f0;
                    zacc[2 * e + 1] += f1;
                    const uint32_t ph = pack_bf16x2(f0, f1);
                    h[e] = ph;
                    float d0, d1;
                    unf32x2(add_f32x2(f32x2(f0, f1), f32x2(-__uint_as_float(ph << 16), -__uint_as_float(ph & 0xffff0000u))), d0, d1);
                    l[e] = pack_bf16x2(d0, d1);
                }
                *reinterpret_cast<uint4*>(kt + off) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
            }
            fence_proxy_async_smem();
            if (x.last) {
                // z of this segment: lanes with the same unit u sum first
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float v = zacc[e];
                    for (int m = C::UPR; m < 32; m <<= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
                    zacc[e] = v;
                }
                if (lane < C::UPR) {
                    float* zb = z + (long long)x.bh * D + u * 8;
                    red_add_v4(zb, zacc[0], zacc[1], zacc[2], zacc[3]);
                    red_add_v4(zb + 4, zacc[4], zacc[5], zacc[6], zacc[7]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
            }
            mbar_arrive(&bars->ready[s]);
            if (x.last) {
                // the segment's accumulator: wait for its MMAs, add it to S
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->seg_done, seg & 1, abort_flag))) { ok = false; break; }
                ++seg;
                tc_fence_after();
                // M = 128: feature a in lane a; M = 64: feature a in lane (a % 16) + 32 (a / 16).
                // Warps w and w + 4 share sub-partition w % 4 and split the columns.
                const int sp = warp % 4, part = warp / 4;
                const int a = D == 128 ? 32 * sp + lane : 16 * sp + lane;
                const bool mine = D == 128 || lane < 16;
                float* Sb = S + ((long long)x.bh * D + a) * D;
                constexpr int COLS = D / (C::NTW / 4);
#pragma unroll
                for (int c0 = part * COLS; c0 < (part + 1) * COLS; c0 += 16) {
                    float vals[16];
                    tmem_ld_32x32b_x16(tbase + ((uint32_t)(32 * sp) << 16) + c0, vals);
                    tmem_wait_ld();
                    if (mine) {
#pragma unroll
                        for (int e = 0; e < 16; e += 4) red_add_v4(Sb + c0 + e, vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
                    }
                }
                // TMEM reads complete before the next segment's first MMA overwrites
                tc_fence_before();
            }
        }
        if (!ok) fail();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::NTW) tmem_dealloc(tbase, C::TMEM_COLS);
}

// 3-D view (heads*d, N, B) of a [B][N][heads][d] bf16 tensor; box = 64
// features x 64 tokens of one batch, 128-byte swizzle; tokens past N are
// zero-filled.
bool encode_token_map(CUtensorMap* m, const void* base, const Grid& g,
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
    // one wave (one CTA per SM): the flattened (b*heads, 64-token step)
    // space cut into equal slices of whole steps
    const int steps_per_head = (int)((g.N + 63) / 64);
    const long long total = (long long)g.B * g.heads * steps_per_head;
    const long long per = (total + sms - 1) / sms;
    const long long ctas = (total + per - 1) / per;
    linear_state_kernel<D><<<(unsigned)ctas, C::THREADS, C::SMEM_BYTES, stream>>>(
        mk, mv, g, steps_per_head, total, (int)per, S, z, status);
    return cudaGetLastError();
}

// ------------------------------------------------ operand image of (S, z)
// The fine kernel applies the branch as phi(Q) S on the tensor cores with S
// split into bf16 hi + lo parts (S = hi + lo to ~2^-17 relative).  This
// kernel writes, per (b, head), the shared-memory image the fine kernel
// copies in one piece:
//   [S hi | S lo | z], S parts as the MN-major B operand with a 128-byte
//   swizzle: 64-wide chunks of output features c, in each chunk one
//   128-byte row per input feature a, 16-byte unit u of row a stored at
//   unit position u ^ (a & 7); z as d fp32 values.
// One thread per 16-byte unit of S (8 consecutive c of one row a).
__global__ void __launch_bounds__(256)
linear_pack_kernel(const float* __restrict__ S, const float* __restrict__ z, uint8_t* __restrict__ image,
                   int d, long long bh_count) {
    const long long units_per_bh = (long long)d * d / 8;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long bh = gid / units_per_bh;
    if (bh >= bh_count) return;
    const int unit = (int)(gid % units_per_bh);
    const int a = unit / (d / 8), cu = unit % (d / 8);
    const int ch = cu / 8, uu = cu % 8;
    const float* src = S + (bh * d + a) * d + cu * 8;
    const float4 x0 = __ldg(reinterpret_cast<const float4*>(src));
    const float4 x1 = __ldg(reinterpret_cast<const float4*>(src + 4));
    const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        hi[e] = pack_bf16x2(xs[2 * e], xs[2 * e + 1]);
        lo[e] = pack_bf16x2(xs[2 * e] - __uint_as_float(hi[e] << 16),
                            xs[2 * e + 1] - __uint_as_float(hi[e] & 0xffff0000u));
    }
    uint8_t* img = image + bh * linear_image_bytes(d);
    const int off = ch * (d * 128) + a * 128 + ((uu ^ (a & 7)) << 4);
    *reinterpret_cast<uint4*>(img + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(img + d * d * 2 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    if (unit < d / 4)       // z: d floats = d/4 16-byte units
        reinterpret_cast<float4*>(img + 4 * d * d)[unit] = __ldg(reinterpret_cast<const float4*>(z + bh * d) + unit);
}

cudaError_t launch_linear_pack(const Grid& g, const float* S, const float* z, void* image,
                               cudaStream_t stream) {
    const long long bh = (long long)g.B * g.heads;
    const long long threads = bh * g.d * g.d / 8;
    linear_pack_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(
        S, z, static_cast<uint8_t*>(image), g.d, bh);
    return cudaGetLastError();
}

cudaError_t launch_linear_state(const Grid& g, const void* k, const void* v, float* S, float* z,
                                int* status, cudaStream_t stream,
                                PFN_cuTensorMapEncodeTiled_v12000 enc) {
    if (g.d == 128) return launch_linear_impl<128>(g, k, v, S, z, status, stream, enc);
    return launch_linear_impl<64>(g, k, v, S, z, status, stream, enc);
}

}  // namespace vsa
