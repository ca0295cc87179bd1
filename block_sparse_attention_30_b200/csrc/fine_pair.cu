// fine_pair.cu -- the fine pass of block-sparse video attention, two query
// cubes per CTA in ping-pong, persistent over the grid (sm_100a).
//
// Source of the operation: "FastVideo 稀疏蒸馏技术深度解析" (omica.com.cn),
// section "2. 视频稀疏注意力VSA": only the attention weights of the selected
// key blocks are evaluated, exactly, Flash-Attention style.  A query block is
// one 64-token cube; each kept key block is one cube.
//
// One CTA per SM (persistent).  A work item is two query cubes, A and B (two
// consecutive (b, head, i) rows); the CTA loops over items with a stride of
// gridDim.x.  An M=64 accumulator fills only half of each TMEM sub-partition,
// so cube A lives in lanes 0-15 and cube B in lanes 16-31 of the same columns:
// O in columns [0, d), and two S buffers in [128, 256) and [256, 384)
// (fp32, 128 keys; P overwrites its S buffer as bf16).  With two S buffers
// the tensor core computes S(p+1) while the softmax of step p runs.  Roles:
//   warp 8, lane 0: TMA producer of Q_A, Q_B and the K ring (3 stages of a
//                   key-cube pair at d = 128), load n = 2*step + cube;
//   warp 10, lane 0: TMA producer of the V ring (3 stages), same numbering;
//   warps 9 / 11, lane 0: MMA issuers of cube A / cube B, each in the order
//                   S(0) S(1) | PV(p) S(p+2) | ...  A tcgen05.mma issue holds
//                   its thread for about the MMA's execution time, so the
//                   bookkeeping between MMAs (barrier checks, commits) would
//                   idle the tensor core if one thread issued for both cubes;
//                   with one issuer per cube the other cube's MMAs fill those
//                   gaps.  (S = Q K^T: M=64, N=128, both operands in shared
//                   memory; O += P V: M=64, N=d, P read from TMEM at the same
//                   lanes as O, V MN-major in shared memory.)
// Ring slots are recycled off the MMA-completion barriers the softmax also
// uses (s_full for K, o_ready for V): no separate "empty" commits.  Every
// per-step barrier exists once per S buffer (step parity), so that no waiter
// can find it two phases away from the phase it waits for.
//   warps 0-3 / 4-7: softmax + epilogue of cube A / cube B (one TMEM
//                   sub-partition per warp; each row split over lanes t, t+16).
// Every cube is one 5-D TMA box (d chunk x tw x th x tt) cut from the grid-
// order [B][N][heads][d] tensor, so the cube gather is free and ragged cubes
// arrive zero-filled; the epilogue writes O / l straight to grid order.
//
// Bounded waits everywhere: a timeout records kStatusTimeout, drains the
// CTA's copies and MMAs, frees TMEM and leaves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "fine_attn.h"
#include "sm100.cuh"
#include "softmax_step.cuh"

namespace vsa {
using namespace sm100;

template <int D>
struct PairCfg {
    static constexpr int NCH = D / 64;                 // 64-element (128-byte) d chunks
    static constexpr int Q_BYTES = 64 * D * 2;         // one query cube
    static constexpr int CUBE_BYTES = 64 * D * 2;      // one key cube (K or V)
    static constexpr int PAIR_BYTES = 2 * CUBE_BYTES;  // two key cubes
    static constexpr int CHUNK_STRIDE = 128 * 128;     // bytes between d chunks of a pair
    // Ring depth.  Slots are recycled by waiting on the MMA-completion barrier
    // of the load NK (NV) positions earlier; with loads numbered 2*step + cube
    // that barrier can only be one phase away from the awaited one (so the
    // parity wait is unambiguous) while NK, NV <= 3.
    static constexpr int NK = 3;                       // K ring stages
    static constexpr int NV = 3;                       // V ring stages
    static constexpr int TMEM_COLS = 512;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_BYTES = 2 * Q_BYTES + (NK + NV) * PAIR_BYTES + BAR_BYTES;
    static constexpr int O_COL = 0;                    // fp32 O: d columns
    __host__ __device__ static constexpr int s_col(int buf) { return 128 + 128 * buf; }
    // TMEM lane offset of cube x (A: lanes 0-15, B: lanes 16-31 of a sub-partition)
    __host__ __device__ static constexpr uint32_t lane_off(int x) { return (uint32_t)(16 * x) << 16; }
};
static_assert(PairCfg<128>::NK <= 3 && PairCfg<128>::NV <= 3, "ring depth vs parity waits");
static_assert(PairCfg<128>::SMEM_BYTES <= 232448, "shared memory");
static_assert(PairCfg<64>::SMEM_BYTES <= 232448, "shared memory");

template <int D>
struct PairBars {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[PairCfg<D>::NK];
    uint64_t v_full[PairCfg<D>::NV];
    // Number of the load last issued into each slot (-1: none yet).  The two
    // MMA issuers consume the shared rings independently, so one of them may
    // look at a slot before the producer has refilled it; waiting for the
    // slot's number first makes the following parity wait unambiguous.
    int k_seq[PairCfg<D>::NK];
    int v_seq[PairCfg<D>::NV];
    // [cube][S buffer]: one barrier per buffer, so that neither side can run
    // two phases ahead of the other (parity waits would then be ambiguous)
    uint64_t s_full[2][2], p_full[2][2];
    uint64_t o_ready[2][2];                           // PV(step c) done -> [cube][c % 2]
    uint64_t mma_done[2];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(PairBars<128>) <= PairCfg<128>::BAR_BYTES, "barrier block");
static_assert(sizeof(PairBars<64>) <= PairCfg<64>::BAR_BYTES, "barrier block");

// Wait until load n occupies its slot (the producer has issued it), then
// for the load's completion.  Bounded like every other wait.
__device__ __forceinline__ bool wait_slot(uint64_t* full, const int* seq, long long n, int nst,
                                          const volatile int* abort) {
    const int st = (int)(n % nst);
    const volatile int* sq = seq + st;
    if (*sq != (int)n) {
        const unsigned long long t0 = clock64();
        while (*sq != (int)n) {
            if (*abort) return false;
            if (clock64() - t0 > VSA_WAIT_LIMIT_CYCLES) return false;
        }
    }
    return mbar_wait_spin(full + st, (uint32_t)((n / nst) & 1), abort);
}

struct ItemRows {
    long long row[2];     // (b*heads + head)*nt + i for cube A and B
    bool store[2];        // B may be a duplicate of A when the row count is odd
};

__device__ __forceinline__ ItemRows item_rows(long long item, long long rows) {
    ItemRows r;
    r.row[0] = 2 * item;
    r.row[1] = 2 * item + 1;
    r.store[0] = true;
    r.store[1] = r.row[1] < rows;
    if (!r.store[1]) r.row[1] = r.row[0];
    return r;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
fine_pair_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                 const __grid_constant__ CUtensorMap mv, const Grid g,
                 const int32_t* __restrict__ block_idx, const int topk, const float scale_log2,
                 const int ragged, __nv_bfloat16* __restrict__ out, int* status) {
    using C = PairCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    uint8_t* sQ = smem;                                        // [2][Q_BYTES]
    uint8_t* sK = smem + 2 * C::Q_BYTES;                       // [NK][PAIR_BYTES]
    uint8_t* sV = sK + C::NK * C::PAIR_BYTES;                  // [NV][PAIR_BYTES]
    PairBars<D>* bars = reinterpret_cast<PairBars<D>*>(sV + C::NV * C::PAIR_BYTES);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long rows = (long long)g.B * g.heads * g.nt;
    const long long n_items = (rows + 1) / 2;
    const int n_pairs = (topk + 1) >> 1;

    if (tid == 0) {
        bars->abort = 0;
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->q_full[x], 1);
            mbar_init(&bars->q_empty[x], 1);
            mbar_init(&bars->s_full[x][0], 1);
            mbar_init(&bars->s_full[x][1], 1);
            mbar_init(&bars->p_full[x][0], 128);
            mbar_init(&bars->p_full[x][1], 128);
            mbar_init(&bars->o_ready[x][0], 1);
            mbar_init(&bars->o_ready[x][1], 1);
        }
        for (int s = 0; s < C::NK; ++s) { mbar_init(&bars->k_full[s], 1); bars->k_seq[s] = -1; }
        for (int s = 0; s < C::NV; ++s) { mbar_init(&bars->v_full[s], 1); bars->v_seq[s] = -1; }
        mbar_init(&bars->mma_done[0], 1);
        mbar_init(&bars->mma_done[1], 1);
        fence_barrier_init();
    }
    if (warp == 9) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    if (warp == 8 && lane == 0) { tma_prefetch_desc(&mq); tma_prefetch_desc(&mk); tma_prefetch_desc(&mv); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;

    auto fail = [&]() {
        *abort_flag = 1;
        report(status, kStatusTimeout);
    };
    // kept cube t of pair p of row `row`, range-checked (-1 when out of range)
    auto kept = [&](long long row, int p, int t) -> int {
        int j = __ldg(block_idx + row * topk + 2 * p + t);
        if (j < 0 || j >= g.nt) j = -1;
        return j;
    };
    // the (up to) four kept cubes of pair p for cubes A and B
    auto load_pair_idx = [&](const ItemRows& ir, int p, int (&j)[2][2]) {
        const int ntl = min(2, topk - 2 * p);
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int t = 0; t < 2; ++t) j[x][t] = t < ntl ? kept(ir.row[x], p, t) : 0;
    };

    if (warp == 8) {
        if (lane == 0) {
            // --------------------------------------------- producer: Q and K
            long long n_k = 0;                      // K pair loads issued so far
            int li = 0;
            bool ok = true;
            for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++li) {
                const ItemRows ir = item_rows(item, rows);
                for (int x = 0; x < 2 && ok; ++x) {
                    if (li > 0 && !mbar_wait(&bars->q_empty[x], (li - 1) & 1, abort_flag)) { ok = false; break; }
                    const long long row = ir.row[x];
                    const int i = (int)(row % g.nt), bh = (int)(row / g.nt);
                    const int head = bh % g.heads, b = bh / g.heads;
                    const TileCoord qc = tile_coord(g, i);
                    mbar_arrive_expect_tx(&bars->q_full[x], C::Q_BYTES);
                    for (int c = 0; c < C::NCH; ++c)
                        tma_load_5d(sQ + x * C::Q_BYTES + c * 8192, &mq, &bars->q_full[x],
                                    head * D + 64 * c, qc.w0, qc.h0, qc.t0, b);
                }
                int jn[2][2];                          // kept cubes of the next pair
                load_pair_idx(ir, 0, jn);
                for (int p = 0; ok && p < n_pairs; ++p) {
                    const int ntl = min(2, topk - 2 * p);
                    int jc[2][2] = {{jn[0][0], jn[0][1]}, {jn[1][0], jn[1][1]}};
                    if (p + 1 < n_pairs) load_pair_idx(ir, p + 1, jn);   // in flight during the waits
                    for (int x = 0; x < 2; ++x, ++n_k) {
                        const int st = (int)(n_k % C::NK);
                        if (n_k >= C::NK) {
                            // slot of load m = n_k - NK is free once S_{m&1}(m>>1) completed
                            const long long m = n_k - C::NK, cm = m >> 1;
                            if (!mbar_wait(&bars->s_full[m & 1][cm & 1], (cm >> 1) & 1, abort_flag)) { ok = false; break; }
                        }
                        const long long row = ir.row[x];
                        const int bh = (int)(row / g.nt), head = bh % g.heads, b = bh / g.heads;
                        mbar_arrive_expect_tx(&bars->k_full[st], ntl * C::CUBE_BYTES);
                        *(volatile int*)&bars->k_seq[st] = (int)n_k;
                        for (int t = 0; t < ntl; ++t) {
                            int j = jc[x][t];
                            if (j < 0) { report(status, kStatusBadIndex); j = 0; }
                            const TileCoord kc = tile_coord(g, j);
                            for (int c = 0; c < C::NCH; ++c)
                                tma_load_5d(sK + st * C::PAIR_BYTES + c * C::CHUNK_STRIDE + t * 8192, &mk,
                                            &bars->k_full[st], head * D + 64 * c, kc.w0, kc.h0, kc.t0, b);
                        }
                    }
                }
            }
            if (!ok) fail();
            if (*abort_flag) {
                for (int x = 0; x < 2; ++x) wait_noabort(&bars->q_full[x], (li - 1) & 1);
                for (long long n = max(0ll, n_k - C::NK); n < n_k; ++n)
                    wait_noabort(&bars->k_full[n % C::NK], (n / C::NK) & 1);
            }
        }
    } else if (warp == 10) {
        if (lane == 0) {
            // ---------------------------------------------------- producer: V
            long long n_v = 0;
            bool ok = true;
            for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const ItemRows ir = item_rows(item, rows);
                int jn[2][2];
                load_pair_idx(ir, 0, jn);
                for (int p = 0; ok && p < n_pairs; ++p) {
                    const int ntl = min(2, topk - 2 * p);
                    int jc[2][2] = {{jn[0][0], jn[0][1]}, {jn[1][0], jn[1][1]}};
                    if (p + 1 < n_pairs) load_pair_idx(ir, p + 1, jn);
                    for (int x = 0; x < 2; ++x, ++n_v) {
                        const int st = (int)(n_v % C::NV);
                        if (n_v >= C::NV) {
                            // slot of load m = n_v - NV is free once PV_{m&1}(m>>1) completed
                            const long long m = n_v - C::NV, cm = m >> 1;
                            if (!mbar_wait(&bars->o_ready[m & 1][cm & 1], (cm >> 1) & 1, abort_flag)) { ok = false; break; }
                        }
                        const long long row = ir.row[x];
                        const int bh = (int)(row / g.nt), head = bh % g.heads, b = bh / g.heads;
                        mbar_arrive_expect_tx(&bars->v_full[st], ntl * C::CUBE_BYTES);
                        *(volatile int*)&bars->v_seq[st] = (int)n_v;
                        for (int t = 0; t < ntl; ++t) {
                            const int j = jc[x][t] < 0 ? 0 : jc[x][t];
                            const TileCoord kc = tile_coord(g, j);
                            for (int c = 0; c < C::NCH; ++c)
                                tma_load_5d(sV + st * C::PAIR_BYTES + c * C::CHUNK_STRIDE + t * 8192, &mv,
                                            &bars->v_full[st], head * D + 64 * c, kc.w0, kc.h0, kc.t0, b);
                        }
                    }
                }
            }
            if (!ok) fail();
            if (*abort_flag)
                for (long long n = max(0ll, n_v - C::NV); n < n_v; ++n)
                    wait_noabort(&bars->v_full[n % C::NV], (n / C::NV) & 1);
        }
    } else if (warp == 9 || warp == 11) {
        if (lane == 0) {
            // ------------------------------------------- MMA issuer of cube x
            const int x = warp == 9 ? 0 : 1;
            const uint32_t q_addr = smem_u32(sQ) + x * C::Q_BYTES, k_addr = smem_u32(sK), v_addr = smem_u32(sV);
            const uint32_t id_pv = idesc_bf16_f32(64, D, false, true);
            const uint32_t o_tmem = tbase + C::lane_off(x) + C::O_COL;
            bool ok = true;
            int li = 0;
            // S(step c, pair p of its item) = Q_x K^T into S buffer c % 2; K load 2c + x
            auto issue_s = [&](int p, long long c) -> bool {
                const long long n = 2 * c + x;
                const int st = (int)(n % C::NK);
                if (!wait_slot(bars->k_full, bars->k_seq, n, C::NK, abort_flag)) return false;
                tc_fence_after();
                const int nkeys = min(2, topk - 2 * p) * 64;
                const uint32_t id_s = idesc_bf16_f32(64, nkeys, false, false);
                const uint32_t d_tmem = tbase + C::lane_off(x) + C::s_col((int)(c & 1));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = smem_desc_sw128(q_addr + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(k_addr + st * C::PAIR_BYTES + (kk >> 2) * C::CHUNK_STRIDE + (kk & 3) * 32, 16, 1024);
                    mma_bf16_ss(d_tmem, a, bd, id_s, kk > 0);
                }
                mma_commit(&bars->s_full[x][c & 1]);
                if (p == n_pairs - 1) mma_commit(&bars->q_empty[x]);   // last read of Q_x
                return true;
            };
            for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++li) {
                const long long base = (long long)li * n_pairs;
                if (!mbar_wait_spin(&bars->q_full[x], li & 1, abort_flag)) { ok = false; break; }
                for (int p = 0; ok && p < min(2, n_pairs); ++p) ok = issue_s(p, base + p);
                for (int p = 0; ok && p < n_pairs; ++p) {
                    const long long c = base + p, n = 2 * c + x;
                    const int nkeys = min(2, topk - 2 * p) * 64;
                    if (!mbar_wait_spin(&bars->p_full[x][c & 1], (c >> 1) & 1, abort_flag)) { ok = false; break; }
                    const int st = (int)(n % C::NV);
                    if (!wait_slot(bars->v_full, bars->v_seq, n, C::NV, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t p_tmem = tbase + C::lane_off(x) + C::s_col((int)(c & 1));
                    for (int kk = 0; kk < nkeys / 16; ++kk) {
                        const uint64_t bd = smem_desc_sw128(v_addr + st * C::PAIR_BYTES + kk * 2048, C::CHUNK_STRIDE, 1024);
                        mma_bf16_ts(o_tmem, p_tmem + kk * 8, bd, id_pv, (p > 0 || kk > 0));
                    }
                    mma_commit(&bars->o_ready[x][c & 1]);
                    // S(p+2) reuses this step's S buffer: issued after the PV that reads P
                    if (p + 2 < n_pairs && !issue_s(p + 2, c + 2)) { ok = false; break; }
                }
            }
            if (!ok) fail();
            mma_commit(&bars->mma_done[x]);
            wait_noabort(&bars->mma_done[x], 0);
        }
    } else {
        // ----------------------------------------- softmax + epilogue (x = A/B)
        const int x = warp >> 2, wq = warp & 3;
        const int r = 16 * wq + (lane & 15), hf = lane >> 4;
        const uint32_t lane_base = ((uint32_t)(32 * wq) << 16) + C::lane_off(x);
        const uint32_t tO = tbase + lane_base + C::O_COL;
        bool ok = true;
        int li = 0;
        for (long long item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++li) {
            const ItemRows ir = item_rows(item, rows);
            const long long row = ir.row[x];
            const long long base = (long long)li * n_pairs;
            SoftmaxState sm{-INFINITY, 0.f};
            int j_next = (ragged && hf < min(2, topk)) ? kept(row, 0, hf) : 0;
            for (int p = 0; p < n_pairs; ++p) {
                const long long c = base + p;
                const int ntl = min(2, topk - 2 * p);
                uint64_t vmask = ~0ull;
                if (ragged) {                         // edge cubes: mask padded keys
                    const int j = j_next;
                    if (p + 1 < n_pairs && hf < min(2, topk - 2 * (p + 1))) j_next = kept(row, p + 1, hf);
                    vmask = hf < ntl ? valid_slot_mask(g, tile_coord(g, j < 0 ? 0 : j)) : 0ull;
                } else if (hf >= ntl) {
                    vmask = 0ull;                     // odd tail: this half has no cube
                }
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[x][c & 1], (c >> 1) & 1, abort_flag))) { ok = false; break; }
                tc_fence_after();
                const uint32_t tS = tbase + lane_base + C::s_col((int)(c & 1));
                float s[64];
                tmem_ld_16x32bx2_x16<64>(tS + 0, *reinterpret_cast<float(*)[16]>(&s[0]));
                tmem_ld_16x32bx2_x16<64>(tS + 16, *reinterpret_cast<float(*)[16]>(&s[16]));
                tmem_ld_16x32bx2_x16<64>(tS + 32, *reinterpret_cast<float(*)[16]>(&s[32]));
                tmem_ld_16x32bx2_x16<64>(tS + 48, *reinterpret_cast<float(*)[16]>(&s[48]));
                tmem_wait_ld();
                uint32_t pk[32];
                bool resc;
                const bool masked = __any_sync(0xffffffffu, vmask != ~0ull);
                const float alpha = masked ? softmax_step<true>(s, vmask, scale_log2, sm, resc, pk)
                                           : softmax_step<false>(s, vmask, scale_log2, sm, resc, pk);
                tmem_st_16x32bx2_x32(tS, pk);
                if (p > 0 && __any_sync(0xffffffffu, resc)) {
                    // O holds PV up to pair p-1: wait for it, then rescale in place
                    const long long cp = c - 1;
                    if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_ready[x][cp & 1], (cp >> 1) & 1, abort_flag))) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < D / 2; c0 += 16) {
                        float o[16];
                        tmem_ld_16x32bx2_x16<D / 2>(tO + c0, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] *= alpha;
                        tmem_st_16x32bx2_x16<D / 2>(tO + c0, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[x][c & 1]);
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            // S(p+2) is issued right after PV(p), so when the last softmax step
            // ends the last two PVs may both be pending: wait for them in order
            // (a single parity wait could mistake phase last-1 for phase last).
            {
                const long long c1 = base + n_pairs - 1, c0 = c1 - 1;
                if (n_pairs >= 2 &&
                    !__all_sync(0xffffffffu, mbar_wait(&bars->o_ready[x][c0 & 1], (c0 >> 1) & 1, abort_flag))) { ok = false; break; }
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_ready[x][c1 & 1], (c1 >> 1) & 1, abort_flag))) { ok = false; break; }
            }
            tc_fence_after();
            const float l = sm.l_run + __shfl_xor_sync(0xffffffffu, sm.l_run, 16);
            const float inv = 1.f / l;
            const int i = (int)(row % g.nt), bh = (int)(row / g.nt);
            const int head = bh % g.heads, b = bh / g.heads;
            const TileCoord qc = tile_coord(g, i);
            const int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;
            const bool valid = ir.store[x] && dt < qc.vt && dh < qc.vh && dw < qc.vw;
            const long long n = ((long long)(qc.t0 + dt) * g.H + (qc.h0 + dh)) * g.W + (qc.w0 + dw);
            __nv_bfloat16* orow = out + (((long long)b * g.N + n) * g.heads + head) * D + hf * (D / 2);
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 16) {
                float o[16];
                tmem_ld_16x32bx2_x16<D / 2>(tO + c0, o);
                tmem_wait_ld();
                uint4 w0, w1;
                w0.x = pack_bf16x2(o[0] * inv, o[1] * inv);
                w0.y = pack_bf16x2(o[2] * inv, o[3] * inv);
                w0.z = pack_bf16x2(o[4] * inv, o[5] * inv);
                w0.w = pack_bf16x2(o[6] * inv, o[7] * inv);
                w1.x = pack_bf16x2(o[8] * inv, o[9] * inv);
                w1.y = pack_bf16x2(o[10] * inv, o[11] * inv);
                w1.z = pack_bf16x2(o[12] * inv, o[13] * inv);
                w1.w = pack_bf16x2(o[14] * inv, o[15] * inv);
                if (valid) {
                    reinterpret_cast<uint4*>(orow + c0)[0] = w0;
                    reinterpret_cast<uint4*>(orow + c0)[1] = w1;
                }
            }
            // O_x is read out: the next item's first PV may overwrite it once
            // this warpgroup arrives on p_full again (after these loads).
            tc_fence_before();
        }
        if (!ok) fail();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tbase, C::TMEM_COLS);
}

template <int D>
static cudaError_t launch_pair_impl(const FineArgs& a, cudaStream_t stream) {
    using C = PairCfg<D>;
    static int configured_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(fine_pair_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    int sms = 148;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.g.B * a.g.heads * a.g.nt;
    const long long items = (rows + 1) / 2;
    const unsigned grid = (unsigned)(items < sms ? items : sms);
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    const int ragged = (a.g.T % a.g.tt) || (a.g.H % a.g.th) || (a.g.W % a.g.tw);
    fine_pair_kernel<D><<<grid, 384, C::SMEM_BYTES, stream>>>(
        *a.mq, *a.mk, *a.mv, a.g, a.block_idx, a.topk, scale_log2, ragged,
        reinterpret_cast<__nv_bfloat16*>(a.out), a.status);
    return cudaGetLastError();
}

cudaError_t launch_fine_pair(const FineArgs& a, cudaStream_t stream) {
    if (a.g.d == 128) return launch_pair_impl<128>(a, stream);
    return launch_pair_impl<64>(a, stream);
}

}  // namespace vsa
