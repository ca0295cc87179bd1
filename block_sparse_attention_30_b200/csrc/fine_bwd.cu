// fine_bwd.cu -- backward pass of the fine block-sparse attention on sm_100a.
//
// The sparse branch is trainable ("FastVideo 稀疏蒸馏技术深度解析",
// omica.com.cn, section "2. 视频稀疏注意力VSA"; TurboDiffusion article,
// dolphinsci.com, section "稀疏、蒸馏与全链路量化").  With the selection held
// fixed and P the softmax of the scaled scores over the kept keys,
//     dV = P^T dO,   dP = dO V^T,   dS = P o (dP - D),   D = rowsum(dO o O),
//     dQ = dS K / sqrt(d),          dK = dS^T Q / sqrt(d).
// P is recomputed from the forward's per-row log2 normaliser (lse).
//
// Kernels:
//   delta_kernel   D per cube slot, fp32 (0 for padded slots).
//   csr_bitmap_kernel  the transpose of the block index: for every key cube
//                  the ascending list of query cubes that kept it
//                  (deterministic; a shared-memory bitmap per (b, head)).
//   dq_body        one CTA per query cube: per kept key cube, S = Q K^T
//                  (TMEM lanes 0-15) and dP = dO V^T (lanes 16-31 of the same
//                  columns) on the tensor cores, dS written as bf16 over S by
//                  the softmax warps, then dQ += dS K (A = dS from TMEM).
//   dkdv_body      one CTA per key cube: per query cube that kept it,
//                  S^T = K Q^T and dP^T = V dO^T, P^T and dS^T written as bf16
//                  over them, then dV += P^T dO (lanes 0-15) and
//                  dK += dS^T Q (lanes 16-31) accumulate in TMEM.
// Both walk single cubes: two ring slots for the streamed cubes and two S
// buffers (the two 64-column halves of the S region) let the loads and the
// softmax of one step overlap the tensor-core work of the next.
// Both run in one launch (bwd_kernel: even CTAs dQ, odd CTAs dK/dV).  One
// K/Q tile serves as the K-major operand of one product and the MN-major
// operand of the other, as V does in the forward.  Every wait is bounded.
#include <algorithm>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "fine_bwd.h"
#include "sm100.cuh"

namespace vsa {
using namespace sm100;

// ------------------------------------------------------------------ delta
// One warp per cube slot: D = sum_c dO[n][c] O[n][c] over the slot's token row,
// with the forward's fp32 output (its bf16 rounding, 2^-9 relative, would
// otherwise enter dQ as -dD sum_m P_m k_m / sqrt(d), which does not shrink
// with dQ when the kept keys share a large common component).  Each lane
// reads 4 features at a time (16 bytes of O, 8 bytes of dO), 8 slots per warp.
__global__ void __launch_bounds__(256)
delta_kernel(const float* __restrict__ o, const __nv_bfloat16* __restrict__ dout, const Grid g,
             float* __restrict__ delta) {
    // one warp per 8 consecutive slots of one cube (8 token rows in flight)
    const long long grp = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)g.B * g.heads * g.nt;
    if (grp >= rows * 8) return;
    const long long row = grp / 8;
    const int s0 = (int)(grp % 8) * 8;
    const int i = (int)(row % g.nt), bh = (int)(row / g.nt);
    const int head = bh % g.heads, b = bh / g.heads;
    const TileCoord c = tile_coord(g, i);
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int s = s0 + u;
        const int dt = s / (g.th * g.tw), dh = (s / g.tw) % g.th, dw = s % g.tw;
        acc[u] = 0.f;
        if (dt < c.vt && dh < c.vh && dw < c.vw) {
            const long long n = ((long long)(c.t0 + dt) * g.H + (c.h0 + dh)) * g.W + (c.w0 + dw);
            const long long base = (((long long)b * g.N + n) * g.heads + head) * g.d;
            for (int e = lane * 4; e < g.d; e += 128) {
                const float4 x = *reinterpret_cast<const float4*>(o + base + e);
                const uint2 yr = *reinterpret_cast<const uint2*>(dout + base + e);
                acc[u] = fmaf(x.x, __uint_as_float(yr.x << 16), acc[u]);
                acc[u] = fmaf(x.y, __uint_as_float(yr.x & 0xffff0000u), acc[u]);
                acc[u] = fmaf(x.z, __uint_as_float(yr.y << 16), acc[u]);
                acc[u] = fmaf(x.w, __uint_as_float(yr.y & 0xffff0000u), acc[u]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
    if (lane < 8) {
        float v = acc[0];
#pragma unroll
        for (int u = 1; u < 8; ++u) v = lane == u ? acc[u] : v;
        delta[row * 64 + s0 + lane] = v;
    }
}

// ---------------------------------------------------------------- transpose
// The transpose of the block index, one CTA per (b, head): bit (j, i) of a
// shared-memory bitmap is set when query cube i kept key cube j, for key
// cubes j0 .. j0 + chunk - 1 at a time (the head's index rows are read once
// per chunk); the set bits of row j in ascending i are key cube j's list
// (deterministic, and a cube listed twice in one row counts once), off[j + 1]
// the running count.  Entries outside 0 .. nt-1 are skipped (the dQ body
// reports them).  chunk <= kCsrThreads: one thread per bitmap row for the
// counts and the writes.
constexpr int kCsrThreads = 512;
constexpr int kCsrSmemBytes = 40 * 1024;             // dynamic shared memory, below the default limit

__global__ void __launch_bounds__(kCsrThreads)
csr_bitmap_kernel(const int32_t* __restrict__ idx, const Grid g, const int k, const int chunk,
                  int32_t* __restrict__ off, int32_t* __restrict__ entries) {
    extern __shared__ uint32_t bm[];                 // [chunk][words]
    __shared__ int32_t wsum[kCsrThreads / 32];
    __shared__ int32_t carry;
    const int words = (g.nt + 31) / 32;
    const long long bh = blockIdx.x;
    const int32_t* rows = idx + bh * g.nt * k;
    int32_t* o = off + bh * (g.nt + 1);
    int32_t* e = entries + bh * g.nt * k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long total = (long long)g.nt * k;
    if (tid == 0) { carry = 0; o[0] = 0; }
    for (int j0 = 0; j0 < g.nt; j0 += chunk) {
        const int nj = min(chunk, g.nt - j0);
        for (int w = tid; w < nj * words; w += kCsrThreads) bm[w] = 0u;
        __syncthreads();
#pragma unroll 4
        for (long long t = tid; t < total; t += kCsrThreads) {
            const int j = __ldg(rows + t);
            if (j >= j0 && j < j0 + nj) {
                const int i = (int)(t / k);
                atomicOr(&bm[(j - j0) * words + (i >> 5)], 1u << (i & 31));
            }
        }
        __syncthreads();
        // row tid: its count, then an exclusive scan over the chunk's rows
        int cnt = 0;
        if (tid < nj)
            for (int w = 0; w < words; ++w) cnt += __popc(bm[tid * words + w]);
        int incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int w = lane < kCsrThreads / 32 ? wsum[lane] : 0;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, d);
                if (lane >= d) w += y;
            }
            if (lane < kCsrThreads / 32) wsum[lane] = w;
        }
        __syncthreads();
        const int base = carry + (warp > 0 ? wsum[warp - 1] : 0) + incl - cnt;
        if (tid < nj) {
            o[j0 + tid + 1] = base + cnt;
            int n = base;
            for (int w = 0; w < words; ++w) {
                uint32_t bits = bm[tid * words + w];
                while (bits) {
                    e[n++] = 32 * w + __ffs(bits) - 1;
                    bits &= bits - 1u;
                }
            }
        }
        __syncthreads();
        if (tid == 0) carry += wsum[kCsrThreads / 32 - 1];
        __syncthreads();
    }
}

// ---------------------------------------------------------- shared layout
// Both bodies walk single cubes (64 keys or 64 queries per step) so that the
// streamed cubes get two ring slots (three for the dQ body's K cubes) and S
// two TMEM buffers within the budget of two CTAs per SM; step t uses S
// buffer t % 2 and ring slot t mod the ring's depth.
template <int D>
struct BwdCfg {
    static constexpr int NCH = D / 64;
    static constexpr int CUBE_BYTES = 64 * D * 2;        // one cube of one tensor (bf16), chunks 8 KB apart
    static constexpr int TMEM_COLS = 256;
    static constexpr int ACC_COL = 0;                    // dQ | dV (lanes 0-15), dK (lanes 16-31)
    static constexpr int S_COL = 128;                    // S buffer b at S_COL + 64 b: S / P (lanes 0-15),
                                                         // dP / dS (lanes 16-31)
    // dQ body: own Q, dO + 3 K slots + 2 V slots; dK/dV body: own K, V + 2 Q
    // slots + 2 dO slots + their lse / D; barriers after either
    static constexpr int SMEM_DQ = 7 * CUBE_BYTES;
    static constexpr int SMEM_DKDV = 6 * CUBE_BYTES + 1024;
    static constexpr int SMEM = (SMEM_DQ > SMEM_DKDV ? SMEM_DQ : SMEM_DKDV) + 256;
    static constexpr int NK = 3;                         // dQ body's K slots
};

static_assert(BwdCfg<128>::SMEM <= 232448 / 2 - 1024, "two CTAs per SM");

struct BwdBars {
    uint64_t a_full;                 // the CTA's own cubes: Q + dO, or K + V
    uint64_t x_full[3], x_empty[3];  // ring 1 (K cubes: 3 slots / Q cubes + lse: 2 slots)
    uint64_t y_full[2], y_empty[2];  // ring 2 (V cubes / dO cubes + D)
    uint64_t s_full[2], ds_full[2], mma_done;
    uint32_t tmem_base;
    int abort;
};

template <int D>
__device__ __forceinline__ void load_cube(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, const Grid& g,
                                          int j, int head, int b) {
    const TileCoord c = tile_coord(g, j);
    for (int ch = 0; ch < D / 64; ++ch)
        tma_load_5d(dst + ch * 8192, map, bar, head * D + 64 * ch, c.w0, c.h0, c.t0, b);
}

// Writes half a row (D/2 features) of an fp32 TMEM accumulator, times `scale`,
// as bf16 to grid order.
template <int D>
__device__ __forceinline__ void store_half_row(uint32_t taddr, float scale, __nv_bfloat16* dst, bool valid) {
#pragma unroll
    for (int c0 = 0; c0 < D / 2; c0 += 16) {
        float o[16];
        tmem_ld_16x32bx2_x16<D / 2>(taddr + c0, o);
        tmem_wait_ld();
        uint4 w0, w1;
        w0.x = pack_bf16x2(o[0] * scale, o[1] * scale);
        w0.y = pack_bf16x2(o[2] * scale, o[3] * scale);
        w0.z = pack_bf16x2(o[4] * scale, o[5] * scale);
        w0.w = pack_bf16x2(o[6] * scale, o[7] * scale);
        w1.x = pack_bf16x2(o[8] * scale, o[9] * scale);
        w1.y = pack_bf16x2(o[10] * scale, o[11] * scale);
        w1.z = pack_bf16x2(o[12] * scale, o[13] * scale);
        w1.w = pack_bf16x2(o[14] * scale, o[15] * scale);
        if (valid) {
            reinterpret_cast<uint4*>(dst + c0)[0] = w0;
            reinterpret_cast<uint4*>(dst + c0)[1] = w1;
        }
    }
}

__device__ __forceinline__ void store_zero_half_row(int half, __nv_bfloat16* dst, bool valid) {
    if (!valid) return;
    for (int c = 0; c < half; c += 8) *reinterpret_cast<uint4*>(dst + c) = make_uint4(0, 0, 0, 0);
}

// One 64 x 64 product pair into S buffer `sb`: S (lanes 0-15) = A1 B1^T and
// dP (lanes 16-31) = A2 B2^T, all operands cubes in smem (K-major), K = D.
template <int D>
__device__ __forceinline__ void issue_s_dp(uint32_t sb, uint32_t a1, uint32_t b1, uint32_t a2, uint32_t b2) {
    const uint32_t id = idesc_bf16_f32(64, 64, false, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t o = (kk >> 2) * 8192 + (kk & 3) * 32;
        mma_bf16_ss(sb, smem_desc_sw128(a1 + o, 16, 1024), smem_desc_sw128(b1 + o, 16, 1024), id, kk > 0);
        mma_bf16_ss(sb + (16u << 16), smem_desc_sw128(a2 + o, 16, 1024), smem_desc_sw128(b2 + o, 16, 1024), id,
                    kk > 0);
    }
}

// acc += T (TMEM, 64 x 64 bf16 at `t`) x cube (smem, 64 rows x D, as the
// MN-major B operand), 4 MMAs of K = 16.
template <int D>
__device__ __forceinline__ void issue_acc(uint32_t acc, uint32_t t, uint32_t cube, bool accumulate) {
    const uint32_t id = idesc_bf16_f32(64, D, false, true);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ts(acc, t + kk * 8, smem_desc_sw128(cube + kk * 2048, 8192, 1024), id, accumulate || kk > 0);
}

// -------------------------------------------------------------------- dQ
// 224 threads: warps 0-3 softmax (rows 16w..16w+15 of the query cube, each
// row split over lanes t and t+16: keys 0-31 and 32-63 of the step's cube),
// warp 4 Q + dO + K cubes, warp 5 MMA, warp 6 V cubes.
template <int D>
__device__ __forceinline__ void dq_body(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                        const CUtensorMap& mg, const Grid& g,
                                        const int32_t* __restrict__ block_idx, const int topk,
                                        const float scale_log2, const int ragged,
                                        const float* __restrict__ lse, const float* __restrict__ delta,
                                        __nv_bfloat16* __restrict__ dq, int* status, uint8_t* smem,
                                        const long long row_id) {
    using C = BwdCfg<D>;
    uint8_t* sQ = smem;
    uint8_t* sG = sQ + C::CUBE_BYTES;
    uint8_t* sK = sG + C::CUBE_BYTES;                 // NK = 3 slots: a K cube is read by S and,
                                                      // after the softmax, by dQ
    uint8_t* sV = sK + C::NK * C::CUBE_BYTES;         // 2 slots (read by dP only)
    BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::SMEM_DQ);
    volatile int* abort_flag = &bars->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = (int)(row_id % g.nt);
    const int bh = (int)(row_id / g.nt);
    const int head = bh % g.heads, b = bh / g.heads;
    const int32_t* my_idx = block_idx + row_id * topk;

    if (tid == 0) {
        bars->abort = 0;
        mbar_init(&bars->a_full, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->y_full[x], 1); mbar_init(&bars->y_empty[x], 1);
            mbar_init(&bars->s_full[x], 1); mbar_init(&bars->ds_full[x], 128);
        }
        for (int x = 0; x < C::NK; ++x) { mbar_init(&bars->x_full[x], 1); mbar_init(&bars->x_empty[x], 1); }
        mbar_init(&bars->mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 5) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;
    auto fail = [&]() { *abort_flag = 1; report(status, kStatusTimeout); };

    if (warp == 4 || warp == 6) {
        if (lane == 0) {
            // step t uses K slot t % 3 (released by dQ of step t - 3) and V
            // slot t % 2 (released by dP of step t - 2)
            const bool is_k = warp == 4;
            const int nslot = is_k ? C::NK : 2;
            uint64_t* full = is_k ? bars->x_full : bars->y_full;
            uint64_t* empty = is_k ? bars->x_empty : bars->y_empty;
            uint8_t* ring = is_k ? sK : sV;
            const CUtensorMap* map = is_k ? &mk : &mv;
            if (is_k) {
                mbar_arrive_expect_tx(&bars->a_full, 2 * C::CUBE_BYTES);
                load_cube<D>(sQ, &mq, &bars->a_full, g, i, head, b);
                load_cube<D>(sG, &mg, &bars->a_full, g, i, head, b);
            }
            int issued = 0;
            for (int t = 0; t < topk; ++t) {
                int j = __ldg(my_idx + t);
                if (j < 0 || j >= g.nt) { if (is_k) report(status, kStatusBadIndex); j = 0; }
                const int x = t % nslot;
                if (t >= nslot && !mbar_wait(&empty[x], ((t / nslot) - 1) & 1, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(&full[x], C::CUBE_BYTES);
                load_cube<D>(ring + x * C::CUBE_BYTES, map, &full[x], g, j, head, b);
                ++issued;
            }
            if (*abort_flag) {
                if (is_k) wait_noabort(&bars->a_full, 0);
                for (int n = issued > nslot ? issued - nslot : 0; n < issued; ++n)
                    wait_noabort(&full[n % nslot], (n / nslot) & 1);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t q_addr = smem_u32(sQ), g_addr = smem_u32(sG);
            const uint32_t tAcc = tbase + C::ACC_COL;
            auto sbuf = [&](int x) { return tbase + C::S_COL + 64 * x; };
            // Two streams of MMAs, issued as their inputs arrive: S/dP of step
            // s (its K and V cubes loaded; S buffer s % 2 free once dQ of step
            // s - 2 is issued, as MMAs run in issue order) and dQ of step a
            // (its dS written).
            int s = 0, a = 0;
            bool ok = mbar_wait(&bars->a_full, 0, abort_flag);
            unsigned long long t0 = clock64();
            while (ok && a < topk) {
                if (s < topk && s <= a + 1 && mbar_test_wait(&bars->x_full[s % C::NK], (s / C::NK) & 1) &&
                    mbar_test_wait(&bars->y_full[s & 1], (s >> 1) & 1)) {
                    const int x = s & 1, xk = s % C::NK;
                    tc_fence_after();
                    issue_s_dp<D>(sbuf(x), q_addr, smem_u32(sK + xk * C::CUBE_BYTES), g_addr,
                                  smem_u32(sV + x * C::CUBE_BYTES));
                    mma_commit(&bars->s_full[x]);
                    mma_commit(&bars->y_empty[x]);         // V cube read by dP only
                    ++s;
                    t0 = clock64();
                } else if (a < s && mbar_test_wait(&bars->ds_full[a & 1], (a >> 1) & 1)) {
                    tc_fence_after();
                    issue_acc<D>(tAcc, sbuf(a & 1), smem_u32(sK + (a % C::NK) * C::CUBE_BYTES), a > 0);   // dQ += dS K
                    mma_commit(&bars->x_empty[a % C::NK]);
                    ++a;
                    t0 = clock64();
                } else if (*abort_flag || clock64() - t0 > VSA_WAIT_LIMIT_CYCLES) {
                    ok = false;
                }
            }
            if (!ok) fail();
            mma_commit(&bars->mma_done);
            wait_noabort(&bars->mma_done, 0);
        }
    } else {
        // softmax warps: P = exp2(s * scale_log2 - lse), dS = P (dP - D)
        const int r = 16 * warp + (lane & 15), hf = lane >> 4;
        const uint32_t lane_base = tbase + ((uint32_t)(32 * warp) << 16);
        const float l2 = __ldg(lse + row_id * 64 + r);
        const float dl = __ldg(delta + row_id * 64 + r);
        bool ok = true;
        for (int t = 0; t < topk; ++t) {
            const int x = t & 1;
            uint32_t vmask = 0xffffffffu;                 // keys 32 hf .. 32 hf + 31 of the cube
            if (ragged) {
                int j = __ldg(my_idx + t);
                if (j < 0 || j >= g.nt) j = 0;
                vmask = (uint32_t)(valid_slot_mask(g, tile_coord(g, j)) >> (32 * hf));
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[x], (t >> 1) & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = lane_base + C::S_COL + 64 * x, tP = tS + (16u << 16);
            float s[32], dp[32];
            tmem_ld_16x32bx2_x16<32>(tS, *reinterpret_cast<float(*)[16]>(&s[0]));
            tmem_ld_16x32bx2_x16<32>(tS + 16, *reinterpret_cast<float(*)[16]>(&s[16]));
            tmem_ld_16x32bx2_x16<32>(tP, *reinterpret_cast<float(*)[16]>(&dp[0]));
            tmem_ld_16x32bx2_x16<32>(tP + 16, *reinterpret_cast<float(*)[16]>(&dp[16]));
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const bool v0 = (vmask >> (2 * e)) & 1u, v1 = (vmask >> (2 * e + 1)) & 1u;
                const float p0 = v0 ? ex2(fmaf(s[2 * e], scale_log2, -l2)) : 0.f;
                const float p1 = v1 ? ex2(fmaf(s[2 * e + 1], scale_log2, -l2)) : 0.f;
                pk[e] = pack_bf16x2(p0 * (dp[2 * e] - dl), p1 * (dp[2 * e + 1] - dl));
            }
            tmem_st_16x32bx2_x16u<16>(tS, pk);            // dS over S: keys 32 hf.. -> columns 16 hf..
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->ds_full[x]);
        }
        if (ok && !__all_sync(0xffffffffu, mbar_wait(&bars->mma_done, 0, abort_flag))) ok = false;
        if (!ok) fail();
        if (ok) {
            tc_fence_after();
            const TileCoord qc = tile_coord(g, i);
            const int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;
            const bool valid = dt < qc.vt && dh < qc.vh && dw < qc.vw;
            const long long n = ((long long)(qc.t0 + dt) * g.H + (qc.h0 + dh)) * g.W + (qc.w0 + dw);
            __nv_bfloat16* drow = dq + (((long long)b * g.N + n) * g.heads + head) * D + hf * (D / 2);
            // scale_log2 / log2(e) = 1/sqrt(d)
            store_half_row<D>(lane_base + C::ACC_COL, scale_log2 * 0.6931471805599453f, drow, valid);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tbase, C::TMEM_COLS);
}

// ------------------------------------------------------------------ dK, dV
// One CTA per key cube: warps 0-3 softmax (key rows 16w..16w+15; lanes t and
// t+16 hold queries 0-31 and 32-63 of the step's query cube), warp 4 K + V
// cubes and the Q cubes (+ their lse), warp 5 MMA, warp 6 the dO cubes (+ D).
template <int D>
__device__ __forceinline__ void dkdv_body(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                          const CUtensorMap& mg, const Grid& g, const int topk,
                                          const float scale_log2, const int32_t* __restrict__ off,
                                          const int32_t* __restrict__ entries, const float* __restrict__ lse,
                                          const float* __restrict__ delta, __nv_bfloat16* __restrict__ dk,
                                          __nv_bfloat16* __restrict__ dv, int* status, uint8_t* smem,
                                          const long long row_id) {
    using C = BwdCfg<D>;
    uint8_t* sK = smem;
    uint8_t* sV = sK + C::CUBE_BYTES;
    uint8_t* sQ = sV + C::CUBE_BYTES;                 // 2 slots
    uint8_t* sG = sQ + 2 * C::CUBE_BYTES;             // 2 slots
    float* sL = reinterpret_cast<float*>(smem + 6 * C::CUBE_BYTES);   // lse of the slots' query cubes [2][64]
    float* sD = sL + 128;                                              // D of the slots' query cubes [2][64]
    BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::SMEM_DKDV);
    volatile int* abort_flag = &bars->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = (int)(row_id % g.nt);           // row_id = (b*heads + head)*nt + j
    const int bh = (int)(row_id / g.nt);
    const int head = bh % g.heads, b = bh / g.heads;
    const int32_t* o = off + (long long)bh * (g.nt + 1);
    const int e0 = __ldg(o + j), nq = __ldg(o + j + 1) - e0;
    const int32_t* my_q = entries + (long long)bh * g.nt * topk + e0;    // ascending query cubes
    const long long qrow0 = (long long)bh * g.nt;                          // row id of query cube 0

    if (tid == 0) {
        bars->abort = 0;
        mbar_init(&bars->a_full, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->x_full[x], 1); mbar_init(&bars->x_empty[x], 1);
            mbar_init(&bars->y_full[x], 1); mbar_init(&bars->y_empty[x], 1);
            mbar_init(&bars->s_full[x], 1); mbar_init(&bars->ds_full[x], 128);
        }
        mbar_init(&bars->mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 5) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;
    auto fail = [&]() { *abort_flag = 1; report(status, kStatusTimeout); };

    if (warp == 4 || warp == 6) {
        if (lane == 0) {
            const bool is_q = warp == 4;
            uint64_t* full = is_q ? bars->x_full : bars->y_full;
            uint64_t* empty = is_q ? bars->x_empty : bars->y_empty;
            uint8_t* ring = is_q ? sQ : sG;
            float* side = is_q ? sL : sD;
            const float* side_src = is_q ? lse : delta;
            const CUtensorMap* map = is_q ? &mq : &mg;
            if (is_q) {
                mbar_arrive_expect_tx(&bars->a_full, 2 * C::CUBE_BYTES);
                load_cube<D>(sK, &mk, &bars->a_full, g, j, head, b);
                load_cube<D>(sV, &mv, &bars->a_full, g, j, head, b);
            }
            int issued = 0;
            for (int t = 0; t < nq; ++t) {
                int it = __ldg(my_q + t);
                if (it < 0 || it >= g.nt) { report(status, kStatusBadIndex); it = 0; }
                const int x = t & 1;
                if (t >= 2 && !mbar_wait(&empty[x], ((t >> 1) - 1) & 1, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(&full[x], C::CUBE_BYTES + 256);
                load_cube<D>(ring + x * C::CUBE_BYTES, map, &full[x], g, it, head, b);
                bulk_load(side + 64 * x, side_src + (qrow0 + it) * 64, 256, &full[x]);
                ++issued;
            }
            if (*abort_flag) {
                if (is_q) wait_noabort(&bars->a_full, 0);
                for (int n = issued > 2 ? issued - 2 : 0; n < issued; ++n) wait_noabort(&full[n & 1], (n >> 1) & 1);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
            const uint32_t tdV = tbase + C::ACC_COL, tdK = tbase + C::ACC_COL + (16u << 16);
            auto sbuf = [&](int x) { return tbase + C::S_COL + 64 * x; };
            // Two streams of MMAs, issued as their inputs arrive: S/dP of step
            // s (its Q and dO cubes loaded; S buffer s % 2 free once the dV/dK
            // MMAs of step s - 2 are issued, as MMAs run in issue order) and
            // dV/dK of step a (its P / dS written).  The Q and dO slots of
            // step s + 2 are refilled only when dV/dK of step s complete, so a
            // fixed order (dV/dK of t, then S of t + 2) would hold dV/dK of
            // t + 1 behind that refill; here they go first when ready.
            int s = 0, a = 0;
            bool ok = mbar_wait(&bars->a_full, 0, abort_flag);
            unsigned long long t0 = clock64();
            while (ok && a < nq) {
                if (s < nq && s <= a + 1 && mbar_test_wait(&bars->x_full[s & 1], (s >> 1) & 1) &&
                    mbar_test_wait(&bars->y_full[s & 1], (s >> 1) & 1)) {
                    const int x = s & 1;
                    tc_fence_after();
                    // S^T = K Q^T (lanes 0-15), dP^T = V dO^T (lanes 16-31)
                    issue_s_dp<D>(sbuf(x), k_addr, smem_u32(sQ + x * C::CUBE_BYTES), v_addr,
                                  smem_u32(sG + x * C::CUBE_BYTES));
                    mma_commit(&bars->s_full[x]);
                    ++s;
                    t0 = clock64();
                } else if (a < s && mbar_test_wait(&bars->ds_full[a & 1], (a >> 1) & 1)) {
                    const int x = a & 1;
                    tc_fence_after();
                    issue_acc<D>(tdV, sbuf(x), smem_u32(sG + x * C::CUBE_BYTES), a > 0);                   // dV += P^T dO
                    issue_acc<D>(tdK, sbuf(x) + (16u << 16), smem_u32(sQ + x * C::CUBE_BYTES), a > 0);     // dK += dS^T Q
                    mma_commit(&bars->x_empty[x]);
                    mma_commit(&bars->y_empty[x]);
                    ++a;
                    t0 = clock64();
                } else if (*abort_flag || clock64() - t0 > VSA_WAIT_LIMIT_CYCLES) {
                    ok = false;
                }
            }
            if (!ok) fail();
            mma_commit(&bars->mma_done);
            wait_noabort(&bars->mma_done, 0);
        }
    } else {
        // softmax warps: P^T = exp2(s * scale_log2 - lse[q]), dS^T = P^T (dP^T - D[q])
        const int r = 16 * warp + (lane & 15), hf = lane >> 4;   // key row, query half of the cube
        const uint32_t lane_base = tbase + ((uint32_t)(32 * warp) << 16);
        bool ok = true;
        for (int t = 0; t < nq; ++t) {
            const int x = t & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[x], (t >> 1) & 1, abort_flag))) { ok = false; break; }
            // lse and D of this query cube landed with its Q / dO cubes
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->x_full[x], (t >> 1) & 1, abort_flag) &&
                                             mbar_wait(&bars->y_full[x], (t >> 1) & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = lane_base + C::S_COL + 64 * x, tP = tS + (16u << 16);
            const float* Ls = sL + 64 * x + 32 * hf;
            const float* Ds = sD + 64 * x + 32 * hf;
            float s[32], dp[32];
            tmem_ld_16x32bx2_x16<32>(tS, *reinterpret_cast<float(*)[16]>(&s[0]));
            tmem_ld_16x32bx2_x16<32>(tS + 16, *reinterpret_cast<float(*)[16]>(&s[16]));
            tmem_ld_16x32bx2_x16<32>(tP, *reinterpret_cast<float(*)[16]>(&dp[0]));
            tmem_ld_16x32bx2_x16<32>(tP + 16, *reinterpret_cast<float(*)[16]>(&dp[16]));
            tmem_wait_ld();
            uint32_t pk[16], dk16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float p0 = ex2(fmaf(s[2 * e], scale_log2, -Ls[2 * e]));
                const float p1 = ex2(fmaf(s[2 * e + 1], scale_log2, -Ls[2 * e + 1]));
                pk[e] = pack_bf16x2(p0, p1);
                dk16[e] = pack_bf16x2(p0 * (dp[2 * e] - Ds[2 * e]), p1 * (dp[2 * e + 1] - Ds[2 * e + 1]));
            }
            tmem_st_16x32bx2_x16u<16>(tS, pk);            // queries 32 hf.. -> columns 16 hf..
            tmem_st_16x32bx2_x16u<16>(tP, dk16);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->ds_full[x]);
        }
        if (ok && !__all_sync(0xffffffffu, mbar_wait(&bars->mma_done, 0, abort_flag))) ok = false;
        if (!ok) fail();
        if (ok) {
            tc_fence_after();
            const TileCoord kc = tile_coord(g, j);
            const int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;
            const bool valid = dt < kc.vt && dh < kc.vh && dw < kc.vw;
            const long long n = ((long long)(kc.t0 + dt) * g.H + (kc.h0 + dh)) * g.W + (kc.w0 + dw);
            const long long base = (((long long)b * g.N + n) * g.heads + head) * D + hf * (D / 2);
            if (nq > 0) {
                store_half_row<D>(lane_base + C::ACC_COL, 1.f, dv + base, valid);
                store_half_row<D>(lane_base + C::ACC_COL + (16u << 16), scale_log2 * 0.6931471805599453f, dk + base, valid);
            } else {                                      // no query cube kept this key cube
                store_zero_half_row(D / 2, dv + base, valid);
                store_zero_half_row(D / 2, dk + base, valid);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tbase, C::TMEM_COLS);
}

// dQ (even CTAs) and dK/dV (odd CTAs) in one launch: the two independent
// halves of the backward share the SMs, and the long tail of the key cubes
// that many query cubes kept overlaps dQ work.
template <int D>
__global__ void __launch_bounds__(224, 2)
bwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
           const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mg, const Grid g,
           const int32_t* __restrict__ block_idx, const int topk, const float scale_log2, const int ragged,
           const int32_t* __restrict__ off, const int32_t* __restrict__ entries,
           const float* __restrict__ lse, const float* __restrict__ delta, __nv_bfloat16* __restrict__ dq,
           __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, int* status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {               // uniform early exit, before any sync
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    const long long row = blockIdx.x >> 1;
    if (blockIdx.x & 1)
        dkdv_body<D>(mq, mk, mv, mg, g, topk, scale_log2, off, entries, lse, delta, dk, dv, status, smem, row);
    else
        dq_body<D>(mq, mk, mv, mg, g, block_idx, topk, scale_log2, ragged, lse, delta, dq, status, smem, row);
}

// ------------------------------------------------------------------ host side

size_t bwd_scratch_bytes(const Grid& g, int topk) {
    const size_t rows = (size_t)g.B * g.heads * g.nt;
    const size_t delta = rows * 64 * sizeof(float);
    const size_t offs = (size_t)g.B * g.heads * (g.nt + 1) * sizeof(int32_t);
    const size_t ents = rows * (size_t)topk * sizeof(int32_t);
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return up(delta) + up(offs) + up(ents);
}

bool bwd_supported(const Grid& g) { return 4ll * ((g.nt + 31) / 32) <= kCsrSmemBytes; }   // nt <= 327680

template <int D>
static cudaError_t launch_bwd_impl(const BwdArgs& a, cudaStream_t stream) {
    using C = BwdCfg<D>;
    const Grid& g = a.g;
    static int configured_device = -1;
    constexpr int SMEM = C::SMEM;
    static_assert(sizeof(BwdBars) <= 256, "barrier block");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const long long rows = (long long)g.B * g.heads * g.nt;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    uint8_t* scratch = static_cast<uint8_t*>(a.scratch);
    float* delta = reinterpret_cast<float*>(scratch);
    int32_t* off = reinterpret_cast<int32_t*>(scratch + up(rows * 64 * sizeof(float)));
    int32_t* ents = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(off) +
                                               up((size_t)g.B * g.heads * (g.nt + 1) * sizeof(int32_t)));
    if (2 * rows > 0x7fffffffll) return cudaErrorInvalidConfiguration;   // a dQ and a dK/dV CTA per cube
    if (!bwd_supported(g)) return cudaErrorInvalidConfiguration;
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    const int ragged = (g.T % g.tt) || (g.H % g.th) || (g.W % g.tw);

    delta_kernel<<<(unsigned)rows, 256, 0, stream>>>(                 // 8 warps x 8 slots per cube
        a.out32, static_cast<const __nv_bfloat16*>(a.dout), g, delta);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // bitmap rows of (nt + 31) / 32 words, in at most kCsrSmemBytes of dynamic
    // shared memory (one row at least: bwd_supported)
    const int words = (g.nt + 31) / 32;
    const int chunk = std::max(1, std::min(std::min(kCsrThreads, g.nt), kCsrSmemBytes / (4 * words)));
    csr_bitmap_kernel<<<(unsigned)(g.B * g.heads), kCsrThreads, (size_t)chunk * words * 4, stream>>>(
        a.block_idx, g, a.topk, chunk, off, ents);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_kernel<D><<<(unsigned)(2 * rows), 224, SMEM, stream>>>(
        *a.mq, *a.mk, *a.mv, *a.mg, g, a.block_idx, a.topk, scale_log2, ragged, off, ents, a.lse, delta,
        static_cast<__nv_bfloat16*>(a.dq), static_cast<__nv_bfloat16*>(a.dk), static_cast<__nv_bfloat16*>(a.dv),
        a.status);
    return cudaGetLastError();
}

cudaError_t launch_fine_bwd(const BwdArgs& a, cudaStream_t stream) {
    return a.g.d == 128 ? launch_bwd_impl<128>(a, stream) : launch_bwd_impl<64>(a, stream);
}

}  // namespace vsa
