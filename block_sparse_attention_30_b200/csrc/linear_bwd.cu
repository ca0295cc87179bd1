// linear_bwd.cu -- backward of the linear-attention branch on sm_100a.
//
// Source: SparkDiffusion news item (bazainvestora.ru), paragraph 3 (RoLA: a
// low-rank linear branch beside the block-sparse one) and the TurboDiffusion
// article (dolphinsci.com), section "稀疏、蒸馏与全链路量化" (SLA: the sparse
// and the linear branch are trained together).  With phi = elu + 1, per
// (b, head): lin_n = phi(q_n) S / den_n, den_n = phi(q_n).z,
// S = sum_m phi(k_m)^T v_m, z = sum_m phi(k_m).  For the output gradient g_n,
// write u_n = S g_n (u_n[a] = sum_c S[a][c] g_n[c]); the chain rule gives
//     g_n.lin_n = phi(q_n).u_n / den_n,   e_n = -phi(q_n).u_n / den_n^2
//     dq_n = (u_n / den_n + e_n z) o phi'(q_n)
//     dS   = sum_n (phi(q_n) / den_n)^T g_n,        dz = sum_n e_n phi(q_n)
//     dk_m = (dS v_m + dz) o phi'(k_m),             dv_m = phi(k_m) dS
// with phi'(x) = 1 for x > 0 and e^x otherwise.  Nothing per token has to be
// kept from the forward pass: S and z are its only state.
//
// Two kernels, each one CTA per SM over 128-token steps of the flattened
// (b*heads, step) space, with G epilogue threads per token (each owning D/G
// features; G = 2 on the query side, 4 on the key side) and one TMA + MMA warp:
//  * query side: U = dO S^T on the tensor cores (dO = dout is exact in bf16,
//    S enters as bf16 hi + lo, so u is good to ~2^-17), the per-token terms on
//    the CUDA cores, then dS += (phi(Q)/den)^T dO (phi/den as hi + lo) into a
//    TMEM accumulator that is added to a global fp32 dS at the end of each
//    (b, head) segment; dz by warp reductions.
//  * key side: U' = V dS^T (dS hi + lo) and dV = phi(K) dS (three products:
//    hi.hi, lo.hi, hi.lo), dk and dv written per token.
// Tiles are double-buffered so the next step's loads overlap the current
// step; the (b, head) operand image (S or dS as bf16 hi/lo, plus z or dz)
// sits in shared memory and is reloaded when a CTA's slice crosses into the
// next (b, head).
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "linear.h"
#include "sm100.cuh"

namespace vsa {
using namespace sm100;

// G epilogue threads per token, each owning D/G consecutive features.
template <int D, int G>
struct LbCfg {
    static constexpr int ROWS = 128;                     // tokens per step
    static constexpr int CHUNK = ROWS * 128;             // one 64-feature chunk of a step tile
    static constexpr int TILE = (D / 64) * CHUNK;        // one tensor's step tile
    static constexpr int IMG = (int)linear_image_bytes(D);  // S hi, S lo (1024-aligned), z
    static constexpr int LO_OFF = 4 * TILE;              // [X0 | Y0 | X1 | Y1 | LO | IMG | bars | xch]
    static constexpr int IMG_OFF = 5 * TILE;
    static constexpr int BAR_OFF = IMG_OFF + IMG;
    static constexpr int XCH_OFF = BAR_OFF + 256;        // per-token partial sums (query side)
    static constexpr int XCH_BYTES = G * 2 * ROWS * 4;
    static constexpr int EPI = ROWS * G;                 // epilogue threads
    static constexpr int MMA_WARP = EPI / 32;            // TMA + MMA warp
    static constexpr int THREADS = EPI + 32;
    static constexpr int FC = D / G;                     // features per epilogue thread
    static constexpr int NC = FC / 16;                   // 16-feature chunks per epilogue thread
    static constexpr int ACC2 = 128;                     // TMEM column of the second accumulator
    static constexpr int TMEM_COLS = 256;
};
// query side: 2 threads per token and the exchange area; key side: 4, none
constexpr int kQueryG = 2, kKeyG = 4;
static_assert(LbCfg<128, kQueryG>::XCH_OFF + LbCfg<128, kQueryG>::XCH_BYTES <= 232448, "shared memory");
static_assert(LbCfg<128, kKeyG>::XCH_OFF <= 232448, "shared memory");
static_assert(LbCfg<64, kKeyG>::NC >= 1, "at least one chunk per thread");

struct LbBars {
    uint64_t full[2];     // X and Y tiles of buffer b landed
    uint64_t done[2];     // (query side) MMAs reading buffer b finished
    uint64_t img_full;    // operand image landed (once per segment)
    uint64_t acc_full;    // the step's accumulator(s) written
    uint64_t ready;       // epilogue warps finished a step (all epilogue threads)
    uint64_t kready;      // (key side) phi(K) hi/lo written (all epilogue threads)
    uint64_t pair[4];     // (query side) all warps of a token group finished pass 1
    uint64_t seg_done;    // (query side) dS accumulation of a segment finished
    uint64_t mma_idle;    // every MMA of the CTA finished
    uint32_t tmem_base;
    int abort;
};

struct LbStep {
    int bh, st;        // (b, head) pair and 128-token step within it
    bool first, last;  // first / last step of this CTA's segment of bh
};

__device__ __forceinline__ LbStep lb_step(long long gs0, int t, int n_steps, int steps_per_head) {
    LbStep x;
    const long long gs = gs0 + t;
    x.bh = (int)(gs / steps_per_head);
    x.st = (int)(gs - (long long)x.bh * steps_per_head);
    x.first = t == 0 || x.st == 0;
    x.last = t == n_steps - 1 || x.st == steps_per_head - 1;
    return x;
}

// phi(x) = elu(x) + 1 = max(x + 1, e^min(x, 0)), since e^x >= 1 + x.
__device__ __forceinline__ float phi_elu1(float x) {
    return fmaxf(x + 1.f, ex2(fminf(x, 0.f) * 1.4426950408889634f));
}

// 8 bf16 of a 16-byte unit -> floats.
__device__ __forceinline__ void unpack8(const uint4 w, float* f) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(a[e] << 16);
        f[2 * e + 1] = __uint_as_float(a[e] & 0xffff0000u);
    }
}

// Splits 8 floats into bf16 hi and lo units (x = hi + lo to ~2^-17).
__device__ __forceinline__ void split8(const float* f, uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        h[e] = pack_bf16x2(f[2 * e], f[2 * e + 1]);
        l[e] = pack_bf16x2(f[2 * e] - __uint_as_float(h[e] << 16),
                           f[2 * e + 1] - __uint_as_float(h[e] & 0xffff0000u));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Stores 8 floats as bf16 at p (16-byte aligned); with `acc`, adds the bf16
// values already there first (one rounding of the sum).
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* f, bool acc) {
    float s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = f[e];
    if (acc) {
        float o[8];
        unpack8(*reinterpret_cast<const uint4*>(p), o);
#pragma unroll
        for (int e = 0; e < 8; ++e) s[e] += o[e];
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(s[0], s[1]), pack_bf16x2(s[2], s[3]),
                                              pack_bf16x2(s[4], s[5]), pack_bf16x2(s[6], s[7]));
}

// Sum over the 32 lanes of 16 per-lane values, scattered: lane l returns the
// warp total of value (l >> 1).  Recursive halving: 16 shuffles in all.
__device__ __forceinline__ float warp_reduce_scatter16(float (&v)[16], int lane) {
#pragma unroll
    for (int lv = 0; lv < 4; ++lv) {
        const int s = 16 >> lv, half = 8 >> lv;
        const bool up = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// Ties 16 values to this point of the program: placed right after
// tcgen05.wait::ld, it keeps the compiler from touching registers that an
// asynchronous TMEM load is still writing before the wait.
__device__ __forceinline__ void reg_fence16(float (&v)[16]) {
    asm volatile("" : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                      "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                      "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]));
}

// Byte offset of 16-byte unit u (8 features) of 64-feature chunk ch of token
// row r in a step tile (TMA 128-byte swizzle).
__device__ __forceinline__ uint32_t unit_off(int ch, int u, int r) {
    return ch * (128 * 128) + r * 128 + ((u ^ (r & 7)) << 4);
}

// Shared setup: barriers and TMEM.
template <int D, int G>
__device__ __forceinline__ LbBars* lb_setup(uint8_t* smem, int warp) {
    using C = LbCfg<D, G>;
    LbBars* bars = reinterpret_cast<LbBars*>(smem + C::BAR_OFF);
    if (threadIdx.x == 0) {
        bars->abort = 0;
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->full[b], 1);
            mbar_init(&bars->done[b], 1);
        }
        mbar_init(&bars->img_full, 1);
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->ready, C::EPI);
        mbar_init(&bars->kready, C::EPI);
        for (int i = 0; i < 4; ++i) mbar_init(&bars->pair[i], 32 * G);
        mbar_init(&bars->seg_done, 1);
        mbar_init(&bars->mma_idle, 1);
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return bars;
}

// Loads of one step (two tensors, 128 tokens, all features) into buffer b.
template <int D, int G>
__device__ __forceinline__ void lb_load_step(uint8_t* smem, LbBars* bars, const CUtensorMap* mx,
                                             const CUtensorMap* my, const Grid& g, const LbStep& x,
                                             int b) {
    using C = LbCfg<D, G>;
    const int bb = x.bh / g.heads, head = x.bh % g.heads;
    uint8_t* xb = smem + (2 * b) * C::TILE;
    uint8_t* yb = smem + (2 * b + 1) * C::TILE;
    mbar_arrive_expect_tx(&bars->full[b], 2 * C::TILE);
    for (int ch = 0; ch < D / 64; ++ch)
        for (int h = 0; h < 2; ++h) {
            const int tok = 128 * x.st + 64 * h;
            tma_load_3d(xb + ch * C::CHUNK + h * 8192, mx, &bars->full[b], head * D + 64 * ch, tok, bb);
            tma_load_3d(yb + ch * C::CHUNK + h * 8192, my, &bars->full[b], head * D + 64 * ch, tok, bb);
        }
}

template <int D, int G>
__device__ __forceinline__ void lb_load_image(uint8_t* smem, LbBars* bars, const uint8_t* image, int bh) {
    mbar_arrive_expect_tx(&bars->img_full, (uint32_t)linear_image_bytes(D));
    bulk_load(smem + LbCfg<D, G>::IMG_OFF, image + (long long)bh * linear_image_bytes(D),
              (uint32_t)linear_image_bytes(D), &bars->img_full);
}

// ------------------------------------------------------------- query side
// X = Q (overwritten in place by (phi(q)/den) hi), Y = dO (dout).
template <int D>
__global__ void __launch_bounds__(LbCfg<D, kQueryG>::THREADS, 1)
linear_bwd_query_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mg,
                        const Grid g, const int steps_per_head, const long long total_steps,
                        const int steps_per_cta, const uint8_t* __restrict__ image,
                        __nv_bfloat16* __restrict__ dq, const int accumulate, float* __restrict__ dS,
                        float* __restrict__ dz, int* status) {
    using C = LbCfg<D, kQueryG>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    LbBars* bars = lb_setup<D, kQueryG>(smem, warp);
    volatile int* abort_flag = &bars->abort;
    const uint32_t tbase = bars->tmem_base;
    const long long gs0 = (long long)blockIdx.x * steps_per_cta;
    const int n_steps = (int)max(0ll, min((long long)steps_per_cta, total_steps - gs0));
    auto fail = [&]() { *abort_flag = 1; report(status, kStatusTimeout); };

    if (warp == C::MMA_WARP) {
        if (lane == 0 && n_steps > 0) {
            // ------------------------------------------------ loads + MMAs
            const uint32_t id_u = idesc_bf16_f32(128, D, false, false);   // U = dO S^T
            const uint32_t id_s = idesc_bf16_f32(D, D, true, true);       // dS += W^T dO
            const uint32_t img = smem_u32(smem + C::IMG_OFF);
            auto mma_u = [&](int t) {
                const uint32_t ga = smem_u32(smem + (2 * (t & 1) + 1) * C::TILE);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = smem_desc_sw128(ga + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(img + part * D * D * 2 + (kk >> 2) * (D * 128) + (kk & 3) * 32, 16, 1024);
                        mma_bf16_ss(tbase, a, bd, id_u, part | kk);
                    }
                mma_commit(&bars->acc_full);
            };
            auto mma_s = [&](int t, bool first) {
                const uint32_t wa = smem_u32(smem + (2 * (t & 1)) * C::TILE);
                const uint32_t lo = smem_u32(smem + C::LO_OFF);
                const uint32_t ga = smem_u32(smem + (2 * (t & 1) + 1) * C::TILE);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {     // 16 tokens per MMA
                        const uint64_t a = smem_desc_sw128((part ? lo : wa) + kk * 2048, C::CHUNK, 1024);
                        const uint64_t bd = smem_desc_sw128(ga + kk * 2048, C::CHUNK, 1024);
                        mma_bf16_ss(tbase + C::ACC2, a, bd, id_s, !(first && part == 0 && kk == 0));
                    }
                mma_commit(&bars->done[t & 1]);
            };
            bool ok = true;
            int issued = 0, seg = 0;
            lb_load_image<D, kQueryG>(smem, bars, image, lb_step(gs0, 0, n_steps, steps_per_head).bh);
            for (int t = 0; t < min(2, n_steps); ++t) {
                lb_load_step<D, kQueryG>(smem, bars, &mq, &mg, g, lb_step(gs0, t, n_steps, steps_per_head), t);
                ++issued;
            }
            if (!mbar_wait_spin(&bars->img_full, 0, abort_flag) || !mbar_wait_spin(&bars->full[0], 0, abort_flag)) ok = false;
            if (ok) { tc_fence_after(); mma_u(0); }
            for (int t = 0; t < n_steps && ok; ++t) {
                const LbStep x = lb_step(gs0, t, n_steps, steps_per_head);
                if (!mbar_wait_spin(&bars->ready, t & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                mma_s(t, x.first);
                if (x.last) mma_commit(&bars->seg_done);
                if (t + 1 < n_steps) {
                    const LbStep x1 = lb_step(gs0, t + 1, n_steps, steps_per_head);
                    if (x1.first) {
                        // U(t) was read (ready), so the old image is free
                        ++seg;
                        lb_load_image<D, kQueryG>(smem, bars, image, x1.bh);
                        if (!mbar_wait_spin(&bars->img_full, seg & 1, abort_flag)) { ok = false; break; }
                    }
                    if (!mbar_wait_spin(&bars->full[(t + 1) & 1], ((t + 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    mma_u(t + 1);
                }
                if (t + 2 < n_steps) {
                    if (!mbar_wait_spin(&bars->done[t & 1], (t >> 1) & 1, abort_flag)) { ok = false; break; }
                    lb_load_step<D, kQueryG>(smem, bars, &mq, &mg, g, lb_step(gs0, t + 2, n_steps, steps_per_head), t & 1);
                    ++issued;
                }
            }
            if (!ok) {
                fail();
                for (int n = max(0, issued - 2); n < issued; ++n) wait_noabort(&bars->full[n & 1], (n >> 1) & 1);
                wait_noabort(&bars->img_full, seg & 1);
            }
            mma_commit(&bars->mma_idle);
            wait_noabort(&bars->mma_idle, 0);
        }
    } else {
        // ------------------------------------------ G threads per token
        // warps w, w + 4, ... share TMEM sub-partition w % 4 (tokens 32 (w % 4)
        // + lane) and split the features: warp w owns the NC 16-feature chunks
        // from (w / 4) NC.  The per-token dot products are summed from the parts
        // through shared memory.
        constexpr int NC = C::NC;
        const int sp = warp & 3, part = warp >> 2;
        const int r = 32 * sp + lane;                        // row of the step tile
        const uint32_t lanes = (uint32_t)(32 * sp) << 16;    // this warp's TMEM lanes
        const int c_lo = part * NC;
        const float* zs = reinterpret_cast<const float*>(smem + C::IMG_OFF + 4 * D * D);
        float* xch = reinterpret_cast<float*>(smem + C::XCH_OFF);   // [G][den, gu][128 rows]
        float dzacc[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) dzacc[c] = 0.f;
        bool ok = true;
        int seg = -1;
        for (int t = 0; t < n_steps; ++t) {
            const LbStep x = lb_step(gs0, t, n_steps, steps_per_head);
            const int b = t & 1;
            if (x.first) {
                ++seg;
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->img_full, seg & 1, abort_flag))) { ok = false; break; }
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->full[b], (t >> 1) & 1, abort_flag))) { ok = false; break; }
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_full, t & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            const int bb = x.bh / g.heads, head = x.bh % g.heads;
            const long long n = 128ll * x.st + r;
            const bool valid = n < g.N;
            uint8_t* qt = smem + (2 * b) * C::TILE;
            uint8_t* lot = smem + C::LO_OFF;

            // pass 1 (own features): partial den = phi(q).z and gu = phi(q).u;
            // the TMEM read of chunk i + 1 overlaps the arithmetic of chunk i
            float den = 0.f, gu = 0.f;
            {
                float ub[2][16];
                tmem_ld_32x32b_x16(tbase + lanes + 16 * c_lo, ub[0]);
                tmem_wait_ld();
                reg_fence16(ub[0]);
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    const int c16 = c_lo + i;
                    if (i + 1 < NC) tmem_ld_32x32b_x16(tbase + lanes + 16 * (c16 + 1), ub[(i + 1) & 1]);
                    float qf[16];
                    const int ch = c16 >> 2, u0 = 2 * (c16 & 3);
                    unpack8(*reinterpret_cast<const uint4*>(qt + unit_off(ch, u0, r)), qf);
                    unpack8(*reinterpret_cast<const uint4*>(qt + unit_off(ch, u0 + 1, r)), qf + 8);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float p = phi_elu1(qf[e]);
                        den = fmaf(p, zs[16 * c16 + e], den);
                        gu = fmaf(p, ub[i & 1][e], gu);
                    }
                    if (i + 1 < NC) { tmem_wait_ld(); reg_fence16(ub[(i + 1) & 1]); }
                }
            }
            xch[(2 * part) * 128 + r] = den;
            xch[(2 * part + 1) * 128 + r] = gu;
            // the parts are shared, and pass 2 overwrites this part of the Q
            // tile that the other warps' pass 1 reads: all finish pass 1 first
            mbar_arrive(&bars->pair[sp]);
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->pair[sp], t & 1, abort_flag))) { ok = false; break; }
            den = 0.f;
            gu = 0.f;
#pragma unroll
            for (int p2 = 0; p2 < kQueryG; ++p2) {     // same order in every warp
                den += xch[(2 * p2) * 128 + r];
                gu += xch[(2 * p2 + 1) * 128 + r];
            }
            const float rden = valid ? 1.f / den : 0.f;
            const float ecoef = -gu * rden * rden;

            // pass 2 (own features): dq, (phi/den) hi/lo for the dS product, dz
            __nv_bfloat16* dqrow = dq + (((long long)bb * g.N + n) * g.heads + head) * D;
            {
                float ub[2][16];
                tmem_ld_32x32b_x16(tbase + lanes + 16 * c_lo, ub[0]);
                tmem_wait_ld();
                reg_fence16(ub[0]);
#pragma unroll
                for (int i = 0; i < NC; ++i) {
                    const int c16 = c_lo + i;
                    if (i + 1 < NC) tmem_ld_32x32b_x16(tbase + lanes + 16 * (c16 + 1), ub[(i + 1) & 1]);
                    float qf[16];
                    const int ch = c16 >> 2, u0 = 2 * (c16 & 3);
                    const uint32_t o0 = unit_off(ch, u0, r), o1 = unit_off(ch, u0 + 1, r);
                    unpack8(*reinterpret_cast<const uint4*>(qt + o0), qf);
                    unpack8(*reinterpret_cast<const uint4*>(qt + o1), qf + 8);
                    float dqv[16], w[16], zc[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float p = valid ? phi_elu1(qf[e]) : 0.f;
                        const float dphi = fmaf(ub[i & 1][e], rden, ecoef * zs[16 * c16 + e]);
                        dqv[e] = dphi * (qf[e] > 0.f ? 1.f : p);
                        w[e] = p * rden;
                        zc[e] = ecoef * p;
                    }
                    uint4 h0, l0, h1, l1;
                    split8(w, h0, l0);
                    split8(w + 8, h1, l1);
                    *reinterpret_cast<uint4*>(qt + o0) = h0;
                    *reinterpret_cast<uint4*>(qt + o1) = h1;
                    *reinterpret_cast<uint4*>(lot + o0) = l0;
                    *reinterpret_cast<uint4*>(lot + o1) = l1;
                    if (valid) {
                        store8(dqrow + 16 * c16, dqv, accumulate != 0);
                        store8(dqrow + 16 * c16 + 8, dqv + 8, accumulate != 0);
                    }
                    dzacc[i] += warp_reduce_scatter16(zc, lane);
                    if (i + 1 < NC) { tmem_wait_ld(); reg_fence16(ub[(i + 1) & 1]); }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ready);

            if (x.last) {
                // dz of the segment: lane 2j holds feature 16 c + j of each chunk c
                if ((lane & 1) == 0) {
#pragma unroll
                    for (int c = 0; c < NC; ++c)
                        atomicAdd(dz + (long long)x.bh * D + 16 * (c_lo + c) + (lane >> 1), dzacc[c]);
                }
#pragma unroll
                for (int c = 0; c < NC; ++c) dzacc[c] = 0.f;
                // dS of the segment: M = 128 puts feature a in lane a; M = 64
                // puts it in lane (a % 16) + 32 (a / 16)
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->seg_done, seg & 1, abort_flag))) { ok = false; break; }
                tc_fence_after();
                const int a = D == 128 ? 32 * sp + lane : 16 * sp + lane;
                const bool mine = D == 128 || lane < 16;
                float* Sb = dS + ((long long)x.bh * D + a) * D;
#pragma unroll 1
                for (int c0 = part * C::FC; c0 < (part + 1) * C::FC; c0 += 16) {
                    float vals[16];
                    tmem_ld_32x32b_x16(tbase + lanes + C::ACC2 + c0, vals);
                    tmem_wait_ld();
                    if (mine) {
#pragma unroll
                        for (int e = 0; e < 16; e += 4) red_add_v4(Sb + c0 + e, vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
                    }
                }
                tc_fence_before();
            }
        }
        if (!ok) fail();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::MMA_WARP) tmem_dealloc(tbase, C::TMEM_COLS);
}

// --------------------------------------------------------------- key side
// X = K (overwritten in place by phi(k) hi), Y = V.
template <int D>
__global__ void __launch_bounds__(LbCfg<D, kKeyG>::THREADS, 1)
linear_bwd_key_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                      const Grid g, const int steps_per_head, const long long total_steps,
                      const int steps_per_cta, const uint8_t* __restrict__ image,
                      __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                      const int accumulate, int* status) {
    using C = LbCfg<D, kKeyG>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    LbBars* bars = lb_setup<D, kKeyG>(smem, warp);
    volatile int* abort_flag = &bars->abort;
    const uint32_t tbase = bars->tmem_base;
    const long long gs0 = (long long)blockIdx.x * steps_per_cta;
    const int n_steps = (int)max(0ll, min((long long)steps_per_cta, total_steps - gs0));
    auto fail = [&]() { *abort_flag = 1; report(status, kStatusTimeout); };

    if (warp == C::MMA_WARP) {
        if (lane == 0 && n_steps > 0) {
            const uint32_t id_u = idesc_bf16_f32(128, D, false, false);   // U' = V dS^T
            const uint32_t id_v = idesc_bf16_f32(128, D, false, true);    // dV = phi(K) dS
            const uint32_t img = smem_u32(smem + C::IMG_OFF);
            const uint32_t lo = smem_u32(smem + C::LO_OFF);
            bool ok = true;
            int issued = 0, seg = 0;
            lb_load_image<D, kKeyG>(smem, bars, image, lb_step(gs0, 0, n_steps, steps_per_head).bh);
            for (int t = 0; t < min(2, n_steps); ++t) {
                lb_load_step<D, kKeyG>(smem, bars, &mk, &mv, g, lb_step(gs0, t, n_steps, steps_per_head), t);
                ++issued;
            }
            for (int t = 0; t < n_steps; ++t) {
                const LbStep x = lb_step(gs0, t, n_steps, steps_per_head);
                if (t > 0) {
                    // epilogue(t-1) is done with TMEM, its K buffer, LO and the image
                    if (!mbar_wait_spin(&bars->ready, (t - 1) & 1, abort_flag)) { ok = false; break; }
                    if (x.first) { ++seg; lb_load_image<D, kKeyG>(smem, bars, image, x.bh); }
                    if (t + 1 < n_steps) {
                        lb_load_step<D, kKeyG>(smem, bars, &mk, &mv, g, lb_step(gs0, t + 1, n_steps, steps_per_head), (t + 1) & 1);
                        ++issued;
                    }
                }
                if (x.first && !mbar_wait_spin(&bars->img_full, seg & 1, abort_flag)) { ok = false; break; }
                if (!mbar_wait_spin(&bars->kready, t & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t xa = smem_u32(smem + (2 * (t & 1)) * C::TILE);
                const uint32_t ya = smem_u32(smem + (2 * (t & 1) + 1) * C::TILE);
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = smem_desc_sw128(ya + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(img + part * D * D * 2 + (kk >> 2) * (D * 128) + (kk & 3) * 32, 16, 1024);
                        mma_bf16_ss(tbase, a, bd, id_u, part | kk);
                    }
#pragma unroll
                for (int part = 0; part < 3; ++part)      // (phi hi, dS hi), (phi lo, dS hi), (phi hi, dS lo)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t ab = part == 1 ? lo : xa;
                        const uint64_t a = smem_desc_sw128(ab + (kk >> 2) * C::CHUNK + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(img + (part == 2 ? D * D * 2 : 0) + kk * 2048, D * 128, 1024);
                        mma_bf16_ss(tbase + C::ACC2, a, bd, id_v, part | kk);
                    }
                mma_commit(&bars->acc_full);
            }
            if (!ok) {
                fail();
                for (int n = max(0, issued - 2); n < issued; ++n) wait_noabort(&bars->full[n & 1], (n >> 1) & 1);
                wait_noabort(&bars->img_full, seg & 1);
            }
            mma_commit(&bars->mma_idle);
            wait_noabort(&bars->mma_idle, 0);
        }
    } else {
        // G threads per token: warps w, w + 4, ... take tokens 32 (w % 4) +
        // lane and split the features (NU 16-byte units, NC 16-feature chunks
        // each); no value crosses warps
        constexpr int NC = C::NC, NU = D / 8 / kKeyG;
        const int sp = warp & 3, part = warp >> 2;
        const int r = 32 * sp + lane;
        const uint32_t lanes = (uint32_t)(32 * sp) << 16;
        const int c_lo = part * NC;
        const float* dzs = reinterpret_cast<const float*>(smem + C::IMG_OFF + 4 * D * D);
        bool ok = true;
        int seg = -1;
        for (int t = 0; t < n_steps; ++t) {
            const LbStep x = lb_step(gs0, t, n_steps, steps_per_head);
            const int b = t & 1;
            const int bb = x.bh / g.heads, head = x.bh % g.heads;
            const long long n = 128ll * x.st + r;
            const bool valid = n < g.N;
            uint8_t* kt = smem + (2 * b) * C::TILE;
            uint8_t* lot = smem + C::LO_OFF;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->full[b], (t >> 1) & 1, abort_flag))) { ok = false; break; }
            // phi(K) hi in place, lo beside it; zero past the end of the grid
#pragma unroll
            for (int i = 0; i < NU; ++i) {
                const int u = part * NU + i;
                const uint32_t o = unit_off(u >> 3, u & 7, r);
                float f[8];
                unpack8(*reinterpret_cast<const uint4*>(kt + o), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = valid ? phi_elu1(f[e]) : 0.f;
                uint4 h, l;
                split8(f, h, l);
                *reinterpret_cast<uint4*>(kt + o) = h;
                *reinterpret_cast<uint4*>(lot + o) = l;
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->kready);
            if (x.first) {
                ++seg;
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->img_full, seg & 1, abort_flag))) { ok = false; break; }
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_full, t & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            __nv_bfloat16* dkrow = dk + (((long long)bb * g.N + n) * g.heads + head) * D;
            __nv_bfloat16* dvrow = dv + (((long long)bb * g.N + n) * g.heads + head) * D;
            // the TMEM reads of chunk i + 1 overlap the arithmetic of chunk i
            float ub[2][16], wb[2][16];
            tmem_ld_32x32b_x16(tbase + lanes + 16 * c_lo, ub[0]);
            tmem_ld_32x32b_x16(tbase + lanes + C::ACC2 + 16 * c_lo, wb[0]);
            tmem_wait_ld();
            reg_fence16(ub[0]);
            reg_fence16(wb[0]);
#pragma unroll
            for (int i = 0; i < NC; ++i) {
                const int c16 = c_lo + i;
                if (i + 1 < NC) {
                    tmem_ld_32x32b_x16(tbase + lanes + 16 * (c16 + 1), ub[(i + 1) & 1]);
                    tmem_ld_32x32b_x16(tbase + lanes + C::ACC2 + 16 * (c16 + 1), wb[(i + 1) & 1]);
                }
                const int ch = c16 >> 2, u0 = 2 * (c16 & 3);
                float ph[16], pl[16];
                unpack8(*reinterpret_cast<const uint4*>(kt + unit_off(ch, u0, r)), ph);
                unpack8(*reinterpret_cast<const uint4*>(kt + unit_off(ch, u0 + 1, r)), ph + 8);
                unpack8(*reinterpret_cast<const uint4*>(lot + unit_off(ch, u0, r)), pl);
                unpack8(*reinterpret_cast<const uint4*>(lot + unit_off(ch, u0 + 1, r)), pl + 8);
                float dkv[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    // phi'(k) = 1 for k > 0 (phi > 1) and phi(k) = e^k otherwise
                    dkv[e] = (ub[i & 1][e] + dzs[16 * c16 + e]) * fminf(ph[e] + pl[e], 1.f);
                }
                if (valid) {
                    store8(dkrow + 16 * c16, dkv, accumulate != 0);
                    store8(dkrow + 16 * c16 + 8, dkv + 8, accumulate != 0);
                    store8(dvrow + 16 * c16, wb[i & 1], accumulate != 0);
                    store8(dvrow + 16 * c16 + 8, wb[i & 1] + 8, accumulate != 0);
                }
                if (i + 1 < NC) {
                    tmem_wait_ld();
                    reg_fence16(ub[(i + 1) & 1]);
                    reg_fence16(wb[(i + 1) & 1]);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->ready);
        }
        if (!ok) fail();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::MMA_WARP) tmem_dealloc(tbase, C::TMEM_COLS);
}

long long linear_bwd_scratch_bytes(const Grid& g) {
    const long long part = ((long long)g.B * g.heads * linear_image_bytes(g.d) + 255) / 256 * 256;
    return 3 * part;
}

template <int D>
static cudaError_t launch_linear_bwd_impl(const Grid& g, const void* q, const void* k, const void* v,
                                          const void* dout, const float* S, const float* z, void* dq,
                                          void* dk, void* dv, int accumulate, uint8_t* scratch,
                                          int* status, cudaStream_t stream,
                                          PFN_cuTensorMapEncodeTiled_v12000 enc) {
    using CQ = LbCfg<D, kQueryG>;
    using CK = LbCfg<D, kKeyG>;
    constexpr int smem_q = CQ::XCH_OFF + CQ::XCH_BYTES, smem_k = CK::XCH_OFF;
    static int configured_device = -1;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(linear_bwd_query_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(linear_bwd_key_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_k);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv, mg;
    if (!encode_token_map(&mq, q, g, enc) || !encode_token_map(&mk, k, g, enc) ||
        !encode_token_map(&mv, v, g, enc) || !encode_token_map(&mg, dout, g, enc))
        return cudaErrorInvalidValue;
    const long long part = linear_bwd_scratch_bytes(g) / 3;
    const long long bh = (long long)g.B * g.heads;
    uint8_t* img_s = scratch;
    float* dS = reinterpret_cast<float*>(scratch + part);
    float* dz = dS + bh * D * D;
    uint8_t* img_ds = scratch + 2 * part;
    e = launch_linear_pack(g, S, z, img_s, stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(dS, 0, sizeof(float) * bh * (D * D + D), stream);
    if (e != cudaSuccess) return e;
    const int steps_per_head = (int)((g.N + 127) / 128);
    const long long total = bh * steps_per_head;
    const long long per = (total + sms - 1) / sms;
    const long long ctas = (total + per - 1) / per;
    linear_bwd_query_kernel<D><<<(unsigned)ctas, CQ::THREADS, smem_q, stream>>>(
        mq, mg, g, steps_per_head, total, (int)per, img_s, static_cast<__nv_bfloat16*>(dq), accumulate,
        dS, dz, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_linear_pack(g, dS, dz, img_ds, stream);
    if (e != cudaSuccess) return e;
    linear_bwd_key_kernel<D><<<(unsigned)ctas, CK::THREADS, smem_k, stream>>>(
        mk, mv, g, steps_per_head, total, (int)per, img_ds, static_cast<__nv_bfloat16*>(dk),
        static_cast<__nv_bfloat16*>(dv), accumulate, status);
    return cudaGetLastError();
}

cudaError_t launch_linear_bwd(const Grid& g, const void* q, const void* k, const void* v,
                              const void* dout, const float* S, const float* z, void* dq, void* dk,
                              void* dv, int accumulate, uint8_t* scratch, int* status,
                              cudaStream_t stream, PFN_cuTensorMapEncodeTiled_v12000 enc) {
    if (g.d == 128)
        return launch_linear_bwd_impl<128>(g, q, k, v, dout, S, z, dq, dk, dv, accumulate, scratch, status, stream, enc);
    return launch_linear_bwd_impl<64>(g, q, k, v, dout, S, z, dq, dk, dv, accumulate, scratch, status, stream, enc);
}

}  // namespace vsa
