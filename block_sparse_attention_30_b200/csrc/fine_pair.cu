// fine_pair.cu -- the fine pass of block-sparse video attention on sm_100a,
// persistent two-cube form (bf16, d = 128, sparse branch).
//
// Source of the operation: "FastVideo 稀疏蒸馏技术深度解析" (omica.com.cn),
// section "2. 视频稀疏注意力VSA": only the attention weights of the selected
// key blocks are evaluated, exactly and Flash-Attention style.  A query block
// is one 64-token cube tile and every kept key block is a cube tile.
//
// Why two cubes per CTA: a 64-query cube gives tcgen05 MMAs of M = 64, whose
// accumulator rows fill TMEM lanes 0-15 of each 32-lane sub-partition.  Here
// one CTA per SM owns a pair of query cubes (A, B) at a time and places cube
// A in lanes 0-15 and cube B in lanes 16-31 of the same columns, so that
//   * each cube has its own MMA-issuing thread: a lone issuer cannot keep up
//     with M = 64 MMAs (about one per 64 cycles) while it also polls
//     barriers and commits, but two issuers fill each other's gaps;
//   * the whole SM's shared memory and TMEM serve both cubes: four ring slots
//     of K (two per cube) and three of V, taken by the two cubes in turn
//     (each slot = two key cubes of one query cube); TMEM holds both cubes'
//     Q (the A operand of Q K^T), two S buffers and one O accumulator;
//   * the CTA walks a list of cube pairs (pair u = cubes 2u, 2u+1 in (batch,
//     head, cube) order; CTA c takes u = c, c + gridDim.x, ...), and its
//     producers load the next pair's Q and key cubes while the current pair
//     finishes, so no CTA set-up or pipeline fill is paid per cube.
// Roles (448 threads):
//   warps 0-7   softmax + epilogue, two warps per TMEM sub-partition: warp w
//               takes rows 16(w%4)..+15 of cube X = w/4, lanes t and t + 16
//               the two key cubes of a step (one shuffle per row maximum);
//   warps 8, 12 K of cubes A and B, warps 10, 13 V of A and B: 5-D TMA
//               boxes cut straight from the [B][N][heads][d] tensors (the
//               cube gather costs no pass; ragged edge cubes arrive
//               zero-filled), four lanes issuing an item's four boxes;
//   warps 9, 11 (one lane each) MMA issuers of cubes A and B; warp 9
//               allocates TMEM.
// Per step (two key cubes = 128 keys of a query cube), for each cube X:
//   S = Q K^T (M = 64, N = 128, A and B from shared memory) into S buffer
//   gs % NS, lanes 16X; softmax writes P as bf16 over S; O += P V (A = P
//   from TMEM, B = V MN-major).  S of step gs + NS is issued right after P V
//   of step gs, so the softmax finds the next S ready.
// Ring items are numbered 2 gs + X in load order; item i uses slot i % R
// (K: R = 4, so cube X owns slots X and X + 2 and each slot serves every
// second step of its cube; V: R = 3, shared by the cubes in turn), signals
// the slot's barrier of cube X (phase gs / 2 for K, gs / 3 for V) and is
// released by its own cube's MMA completion: a K item by the commit of its S
// (s_full[X]), a V item by the commit of its P V (o_ready[X]).  Per-step barriers come in
// NS copies (step gs uses copy gs % NS) and each role observes a barrier's
// phases in order, so every wait is for a phase that is neither overtaken
// nor two phases ahead (a parity wait only tells the last two phases
// apart).  The softmax of step gs, for instance, may run while P V
// of steps gs - 2 and gs - 1 are still pending (S of gs only implies P V of
// gs - 3); with NS copies the copy it waits on has completed step gs - 1 - NS
// already and cannot complete gs - 1 + NS before this softmax step is done.
// Every wait is bounded; on a timeout the CTA records kStatusTimeout in the
// status word, drains its own copies and MMAs, frees TMEM and exits.
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
    static constexpr int NCH = D / 64;                 // 128-byte d chunks
    static constexpr int CUBE = 64 * D * 2;            // one cube of q, k or v (bf16)
    static constexpr int ITEM = 2 * CUBE;              // a ring slot: two key cubes
    static constexpr int CHUNK_STRIDE = 128 * 128;     // bytes between d chunks of a slot
    static constexpr int RK = 4, RV = 3;               // K and V ring slots
    // cube X's items cycle through R / gcd(R, 2) slots: with an even ring
    // each cube keeps its own half of the slots, with an odd one the cubes
    // take every slot in turn
    static constexpr int KCYC = (RK % 2 == 0) ? RK / 2 : RK;
    static constexpr int VCYC = (RV % 2 == 0) ? RV / 2 : RV;
    static constexpr int NS = 2;                       // S buffers in TMEM
    static constexpr int O_COL = 0;                    // fp32 O (D columns)
    static constexpr int S_COL = 128;                  // S buffer x at S_COL + 128 x
    static constexpr int Q_COL = S_COL + 128 * NS;     // bf16 Q, two per column: buffers of D / 2 columns
    static constexpr int TMEM_COLS = 512;
    static constexpr int THREADS = 448;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_BYTES = RK * ITEM + RV * ITEM + BAR_BYTES;
    // producer waits must not be overtaken: an item 2s + X waits for the
    // release of item 2s + X - R (cube X', step s'); the next completion of
    // that barrier copy (step s' + NS of cube X') needs item
    // 2(s' + NS) + X' = 2s + X - R + 2 NS, which is not loaded yet iff 2 NS >= R
    static_assert(2 * NS >= RK && 2 * NS >= RV, "rings deeper than the S buffers allow");
    static_assert(Q_COL + 2 * (D / 2) <= TMEM_COLS && D <= S_COL, "TMEM layout");
    static_assert(D == 128, "the Q row load writes two 64-feature halves");
};

template <int D>
struct PairBars {
    uint64_t q_full[2];                                // Q of cube X in TMEM
    // ring slot s filled for cube X: each issuer waits only on its own cube's
    // barrier of a slot, whose phases it consumes in order
    uint64_t k_full[PairCfg<D>::RK][2], v_full[PairCfg<D>::RV][2];
    uint64_t s_full[2][PairCfg<D>::NS], p_full[2][PairCfg<D>::NS];
    uint64_t o_ready[2][PairCfg<D>::NS];               // P V of step gs done: copy gs % NS
    uint64_t o_free[2], mma_done[2];
    double inv_hw, inv_w;                              // 1/(nh nw), 1/nw for cube coordinates
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(PairBars<128>) <= PairCfg<128>::BAR_BYTES, "barrier block");
static_assert(PairCfg<128>::SMEM_BYTES <= 232448 - 1024, "one CTA per SM");

struct CubeRef {
    int b, head, i;
};

__device__ __forceinline__ CubeRef cube_ref(const Grid& g, long long c) {
    CubeRef r;
    r.i = (int)(c % g.nt);
    const long long bh = c / g.nt;
    r.head = (int)(bh % g.heads);
    r.b = (int)(bh / g.heads);
    return r;
}

// Grid origin of cube j; the cube's coordinates by fp64 reciprocal
// multiplication (inv_hw = 1/(nh nw), inv_w = 1/nw), exact for j < 2^40
// because (j + 1/2) / n stays at least 1/(2n) away from an integer.
__device__ __forceinline__ void cube_origin(const Grid& g, int j, double inv_hw, double inv_w, int& t0, int& h0,
                                            int& w0) {
    const int it = (int)(((double)j + 0.5) * inv_hw);
    const int rem = j - it * (g.nh * g.nw);
    const int ih = (int)(((double)rem + 0.5) * inv_w);
    const int iw = rem - ih * g.nw;
    t0 = it * g.tt; h0 = ih * g.th; w0 = iw * g.tw;
}

// Valid-slot mask of key cube j (all ones for a whole cube).
__device__ __forceinline__ uint64_t cube_valid_mask(const Grid& g, int j, double inv_hw, double inv_w) {
    TileCoord c;
    cube_origin(g, j, inv_hw, inv_w, c.t0, c.h0, c.w0);
    c.vt = min(g.tt, g.T - c.t0);
    c.vh = min(g.th, g.H - c.h0);
    c.vw = min(g.tw, g.W - c.w0);
    return valid_slot_mask(g, c);
}

template <int D>
__global__ void __launch_bounds__(PairCfg<D>::THREADS, 1)
fine_pair_kernel(const __nv_bfloat16* __restrict__ q, const __grid_constant__ CUtensorMap mk,
                 const __grid_constant__ CUtensorMap mv, const Grid g,
                 const int32_t* __restrict__ block_idx, const int topk, const float scale_log2,
                 const int ragged, __nv_bfloat16* __restrict__ out, float* __restrict__ out32,
                 float* __restrict__ lse, int* status) {
    using C = PairCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {               // uniform early exit, before any sync
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    uint8_t* sK = smem;
    uint8_t* sV = sK + C::RK * C::ITEM;
    PairBars<D>* bars = reinterpret_cast<PairBars<D>*>(sV + C::RV * C::ITEM);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long rows = (long long)g.B * g.heads * g.nt;     // query cubes
    const long long n_units = (rows + 1) >> 1;                   // pairs of them
    const int n_steps = (topk + 1) >> 1;                          // key-cube pairs per query cube

    if (tid == 0) {
        bars->abort = 0;
        bars->inv_hw = 1.0 / (double)(g.nh * g.nw);
        bars->inv_w = 1.0 / (double)g.nw;
        for (int X = 0; X < 2; ++X) {
            for (int s = 0; s < C::RK; ++s) mbar_init(&bars->k_full[s][X], 1);
            for (int s = 0; s < C::RV; ++s) mbar_init(&bars->v_full[s][X], 1);
            mbar_init(&bars->q_full[X], 128);
            for (int x = 0; x < C::NS; ++x) {
                mbar_init(&bars->s_full[X][x], 1);
                mbar_init(&bars->p_full[X][x], 128);
                mbar_init(&bars->o_ready[X][x], 1);
            }
            mbar_init(&bars->o_free[X], 128);
            mbar_init(&bars->mma_done[X], 1);
        }
        fence_barrier_init();
    }
    if (warp == 9) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    if (warp == 8 && lane == 0) { tma_prefetch_desc(&mk); tma_prefetch_desc(&mv); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;

    auto fail = [&]() {
        *abort_flag = 1;
        report(status, kStatusTimeout);
    };

    if (warp == 8 || warp == 10 || warp == 12 || warp == 13) {
        // ------------- producers: K of cube A (warp 8), V of A (10), K of B (12), V of B (13)
        // One warp per ring and cube, so that each cube's loads are issued
        // as soon as its slot is free and the two cubes' items stream in
        // parallel.  Lane 0 waits and arms the barriers; the boxes of an item
        // (two key cubes x two d chunks) are issued by lanes 0-3 together.
        const bool is_k = warp == 8 || warp == 12;
        const int X = warp >= 12;
        const int R = is_k ? C::RK : C::RV;
        const int cyc = is_k ? C::KCYC : C::VCYC;
        uint64_t (*full)[2] = is_k ? bars->k_full : bars->v_full;
        uint8_t* ring = is_k ? sK : sV;
        const CUtensorMap* map = is_k ? &mk : &mv;
        long long waited[2] = {-1, -1};        // last step of cube X whose release was seen
        long long issued = 0;                  // steps of this cube loaded so far
        bool ok = true;
        // item 2 gs + X (cube X, step gs) uses slot (2 gs + X) % R and waits
        // for the release of the slot's previous item 2 gs + X - R: a K item
        // by that cube's S completion, a V item by its P V completion; each
        // cube's steps are observed in order
        auto wait_released = [&](int Xp, long long q) -> bool {
            while (waited[Xp] < q) {
                const long long st = ++waited[Xp];
                bool done = true;
                if (lane == 0)
                    done = is_k ? mbar_wait(&bars->s_full[Xp][st % C::NS], (uint32_t)((st / C::NS) & 1), abort_flag)
                                : mbar_wait(&bars->o_ready[Xp][st % C::NS], (uint32_t)((st / C::NS) & 1), abort_flag);
                if (!__shfl_sync(0xffffffffu, done, 0)) return false;
            }
            return true;
        };
        const double inv_hw = 1.0 / (double)(g.nh * g.nw), inv_w = 1.0 / (double)g.nw;
        auto cube_of_unit = [&](long long u) { return X == 0 ? 2 * u : min(2 * u + 1, rows - 1); };
        auto load_idx = [&](long long c, int p, int (&jn)[2]) {
            const int32_t* idx = block_idx + c * topk + 2 * p;
            jn[0] = __ldg(idx);
            jn[1] = 2 * p + 1 < topk ? __ldg(idx + 1) : 0;
        };
        int nj[2] = {0, 0};                    // indices of this producer's next item, fetched ahead
        if (blockIdx.x < n_units) load_idx(cube_of_unit(blockIdx.x), 0, nj);
        long long it = 0;
        for (long long u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++it) {
            const long long gs0 = it * n_steps;
            const long long cube = cube_of_unit(u);
            const CubeRef cr = cube_ref(g, cube);
            for (int p = 0; ok && p < n_steps; ++p) {
                const long long gs = gs0 + p;
                const int ntl = min(2, topk - 2 * p);
                const int j[2] = {nj[0], nj[1]};
                if (p + 1 < n_steps) load_idx(cube, p + 1, nj);
                else if (u + gridDim.x < n_units) load_idx(cube_of_unit(u + gridDim.x), 0, nj);
                const long long item = 2 * gs + X;
                const int slot = (int)(item % R);
                if (item >= R) {
                    const long long prev = item - R;                  // the slot's last item
                    if (!wait_released((int)(prev & 1), prev >> 1)) { ok = false; break; }
                }
                if (lane == 0) mbar_arrive_expect_tx(&full[slot][X], ntl * C::CUBE);
                __syncwarp();
                if (lane < ntl * C::NCH) {                             // box (t, c) from lane t*NCH + c
                    const int t = lane / C::NCH, c = lane % C::NCH;
                    int jj = j[t];
                    if (jj < 0 || jj >= g.nt) {
                        if (is_k && c == 0) report(status, kStatusBadIndex);
                        jj = 0;
                    }
                    int t0, h0, w0;
                    cube_origin(g, jj, inv_hw, inv_w, t0, h0, w0);
                    VSA_DEBUG_CHECK(t0 >= 0 && t0 < g.T && h0 >= 0 && h0 < g.H && w0 >= 0 && w0 < g.W, status,
                                    kStatusBadCoord);
                    tma_load_5d(ring + slot * C::ITEM + c * C::CHUNK_STRIDE + t * 8192, map, &full[slot][X],
                                cr.head * D + 64 * c, w0, h0, t0, cr.b);
                }
                __syncwarp();
                ++issued;
            }
        }
        if (!ok && lane == 0) fail();
        __syncwarp();
        if (lane == 0 && *abort_flag) {
            // drain: the last load this warp issued into each of its slots must
            // land (its items cycle through cyc slots)
            for (long long st = issued > cyc ? issued - cyc : 0; st < issued; ++st)
                wait_noabort(&full[(2 * st + X) % R][X], (uint32_t)((st / cyc) & 1));
        }
    } else if (warp == 9 || warp == 11) {
        // ---------------------------------------------- MMA issuer of cube X
        if (lane == 0) {
            const int X = warp == 11;
            // cube X: TMEM lanes 16X.. of each sub-partition
            const uint32_t tO = tbase + C::O_COL + ((uint32_t)X << 20);
            auto tS = [&](long long gs) { return tbase + C::S_COL + 128u * (uint32_t)(gs % C::NS) + ((uint32_t)X << 20); };
            const uint32_t id_pv = idesc_bf16_f32(64, D, false, true);
            // descriptors of the operands' first 16-element K slices; later
            // slices add their byte offset / 16 to the start-address field
            const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dv = smem_desc_sw128(smem_u32(sV), C::CHUNK_STRIDE, 1024);
            uint32_t tQ = 0;            // Q of the current cube: A operand from TMEM, buffer it & 1
            auto issue_qk = [&](long long gs, int p) -> bool {
                const int nkeys = min(2, topk - 2 * p) * 64;
                const long long item = 2 * gs + X;
                const int slot = (int)(item % C::RK);
                if (!mma_wait(&bars->k_full[slot][X], (uint32_t)((gs / C::KCYC) & 1), abort_flag)) return false;
                tc_fence_after();
                const uint32_t id_s = idesc_bf16_f32(64, nkeys, false, false);
                const uint64_t bk = dk + (uint64_t)((slot * C::ITEM) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t b_off = ((kk >> 2) * C::CHUNK_STRIDE + (kk & 3) * 32) >> 4;
                    mma_bf16_ts(tS(gs), tQ + kk * 8, bk + b_off, id_s, kk > 0);
                }
                mma_commit(&bars->s_full[X][gs % C::NS]);
                return true;
            };
            bool ok = true;
            long long it = 0;
            for (long long u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++it) {
                const long long gs0 = it * n_steps;
                if (!mma_wait(&bars->q_full[X], (uint32_t)(it & 1), abort_flag)) { ok = false; break; }
                tQ = tbase + C::Q_COL + (D / 2) * (uint32_t)(it & 1) + ((uint32_t)X << 20);
                for (int p = 0; ok && p < min(C::NS, n_steps); ++p) ok = issue_qk(gs0 + p, p);
                for (int p = 0; ok && p < n_steps; ++p) {
                    const long long gs = gs0 + p;
                    const int nkeys = min(2, topk - 2 * p) * 64;
                    const long long item = 2 * gs + X;
                    const int slot = (int)(item % C::RV);
                    // the previous pair's epilogue must have read O before it is overwritten
                    if ((p == 0 && it > 0 && !mma_wait(&bars->o_free[X], (uint32_t)((it - 1) & 1), abort_flag)) ||
                        !mma_wait(&bars->p_full[X][gs % C::NS], (uint32_t)((gs / C::NS) & 1), abort_flag) ||
                        !mma_wait(&bars->v_full[slot][X], (uint32_t)((gs / C::VCYC) & 1), abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bv = dv + (uint64_t)((slot * C::ITEM) >> 4);
                    for (int kk = 0; kk < nkeys / 16; ++kk)
                        mma_bf16_ts(tO, tS(gs) + kk * 8, bv + (uint64_t)((kk * 2048) >> 4), id_pv, (p > 0 || kk > 0));
                    mma_commit(&bars->o_ready[X][gs % C::NS]);
                    if (p + C::NS < n_steps) ok = issue_qk(gs + C::NS, p + C::NS);
                }
            }
            if (!ok) fail();
            mma_commit(&bars->mma_done[X]);
            wait_noabort(&bars->mma_done[X], 0);
        }
    } else if (warp < 8) {
        // --------------------------------------------------- softmax / epilogue
        // warps 0-3: rows of cube A (TMEM lanes 0-15 of sub-partition w),
        // warps 4-7: rows of cube B (lanes 16-31).  Lanes t and t + 16 share
        // row r: lane t holds the scores of the step's first key cube, lane
        // t + 16 those of the second, so a row maximum is one shuffle.
        const int sp = warp & 3, X = warp >> 2;
        const int r = 16 * sp + (lane & 15), hf = lane >> 4;
        const uint32_t lane_base = tbase + ((uint32_t)(32 * sp + 16 * X) << 16);
        const uint32_t tO = lane_base + C::O_COL;
        const uint32_t tQ0 = lane_base + C::Q_COL;   // Q buffer b at tQ0 + (D / 2) b
        const int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;   // slot r in its cube
        auto cube_of_unit = [&](long long u) { return X == 0 ? 2 * u : min(2 * u + 1, rows - 1); };
        // address of this thread's half row (D/2 features) of query cube c, or
        // null for a padded slot
        auto q_row = [&](long long c) -> const uint4* {
            const CubeRef qr = cube_ref(g, c);
            const TileCoord qc = tile_coord(g, qr.i);
            if (!(dt < qc.vt && dh < qc.vh && dw < qc.vw)) return nullptr;
            const long long n = ((long long)(qc.t0 + dt) * g.H + (qc.h0 + dh)) * g.W + (qc.w0 + dw);
            return reinterpret_cast<const uint4*>(q + (((long long)qr.b * g.N + n) * g.heads + qr.head) * D + hf * (D / 2));
        };
        // a cube's Q goes to TMEM in four pieces of 16 features (8 columns of
        // each half row); padded slots are zeros.  After the fourth piece one
        // arrival on q_full[X] hands the buffer to the cube's Q K^T.
        auto load_q_piece = [&](const uint4* src, int pc, uint32_t (&w)[8]) {
            const uint4 a = src ? __ldg(src + 2 * pc) : make_uint4(0u, 0u, 0u, 0u);
            const uint4 b = src ? __ldg(src + 2 * pc + 1) : make_uint4(0u, 0u, 0u, 0u);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
            w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
        };
        auto store_q_piece = [&](uint32_t buf, int pc, const uint32_t (&w)[8]) {
            tmem_st_16x32bx2_x8u<32>(tQ0 + (D / 2) * buf + 8 * pc, w);
        };
        auto q_ready = [&]() {
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->q_full[X]);
        };
        bool ok = true;
        long long it = 0;
        if (blockIdx.x < n_units) {                           // the first cube's Q at once, buffer 0
            const uint4* src = q_row(cube_of_unit(blockIdx.x));
#pragma unroll 1
            for (int pc = 0; pc < 4; ++pc) {
                uint32_t w[8];
                load_q_piece(src, pc, w);
                store_q_piece(0, pc, w);
            }
            q_ready();
        }
        for (long long u = blockIdx.x; ok && u < n_units; u += gridDim.x, ++it) {
            const long long gs0 = it * n_steps;
            const long long cube = cube_of_unit(u);
            const long long u_next = u + gridDim.x;
            const bool owner = X == 0 || 2 * u + 1 < rows;     // a repeated last cube writes nothing
            // the next cube's Q streams into the other buffer during this cube's
            // first steps: piece pc is loaded after step pc and written to TMEM
            // after step pc + 1 (the buffer's previous cube is done: its last
            // Q K^T completed before this cube's first S)
            const bool has_next = u_next < n_units;
            const uint4* qsrc = has_next ? q_row(cube_of_unit(u_next)) : nullptr;
            const uint32_t qbuf = (uint32_t)((it + 1) & 1);
            uint32_t qw[8];
            int q_loaded = 0, q_stored = 0;
            const CubeRef cr = cube_ref(g, cube);
            const int32_t* my_idx = block_idx + cube * topk;
            SoftmaxState sm{-INFINITY, 0.f};
            for (int p = 0; p < n_steps; ++p) {
                const long long gs = gs0 + p;
                const int x = (int)(gs % C::NS);
                const uint32_t tS = lane_base + C::S_COL + 128u * (uint32_t)x;
                const int ntl = min(2, topk - 2 * p);
                uint64_t vmask = hf < ntl ? ~0ull : 0ull;            // odd tail: no second cube
                if (ragged && hf < ntl) {                            // edge cubes: mask padded keys
                    int j = __ldg(my_idx + 2 * p + hf);
                    if (j < 0 || j >= g.nt) j = 0;
                    vmask = cube_valid_mask(g, j, bars->inv_hw, bars->inv_w);
                }
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[X][x], (uint32_t)((gs / C::NS) & 1), abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
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
                    // O holds P V up to step gs - 1: rescale it in place once that is done
                    const long long q = gs - 1;
                    if (!__all_sync(0xffffffffu,
                                    mbar_wait(&bars->o_ready[X][q % C::NS], (uint32_t)((q / C::NS) & 1), abort_flag))) {
                        ok = false;
                        break;
                    }
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
                mbar_arrive(&bars->p_full[X][x]);
                if (has_next && q_stored < 4) {
                    if (q_loaded > q_stored) {
                        store_q_piece(qbuf, q_stored, qw);
                        if (++q_stored == 4) q_ready();
                    }
                    if (q_loaded < 4) load_q_piece(qsrc, q_loaded++, qw);
                }
            }
            if (!ok) break;
            if (has_next && q_stored < 4) {                   // a cube of few steps: finish its Q now
                if (q_loaded > q_stored) store_q_piece(qbuf, q_stored++, qw);
#pragma unroll 1
                while (q_stored < 4) {
                    load_q_piece(qsrc, q_stored, qw);
                    store_q_piece(qbuf, q_stored++, qw);
                }
                q_ready();
            }
            // ------------------------------------------------------ epilogue
            const TileCoord qc = tile_coord(g, cr.i);
            const bool valid = owner && dt < qc.vt && dh < qc.vh && dw < qc.vw;
            const long long n = ((long long)(qc.t0 + dt) * g.H + (qc.h0 + dh)) * g.W + (qc.w0 + dw);
            const long long obase = (((long long)cr.b * g.N + n) * g.heads + cr.head) * D + hf * (D / 2);
            const long long gl = gs0 + n_steps - 1;
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&bars->o_ready[X][gl % C::NS], (uint32_t)((gl / C::NS) & 1), abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            float ob[D / 2];                                  // this thread's half row of O
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 16)
                tmem_ld_16x32bx2_x16<D / 2>(tO + c0, *reinterpret_cast<float(*)[16]>(&ob[c0]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars->o_free[X]);                    // O is in registers: the next cube may overwrite it
            const float l = sm.l_run + __shfl_xor_sync(0xffffffffu, sm.l_run, 16);
            const float inv = 1.f / l;
            // log2 of the softmax normaliser of the scaled scores (for the
            // backward pass); +inf marks padded query slots
            if (lse && owner && hf == 0) lse[cube * 64 + r] = valid ? sm.m_run + __log2f(l) : INFINITY;
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 16) {
                float* o = &ob[c0];
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] *= inv;
#ifdef VSA_DEBUG_CHECKS
                if (valid) {
                    bool finite = true;
#pragma unroll
                    for (int e = 0; e < 16; ++e) finite = finite && isfinite(o[e]);
                    VSA_DEBUG_CHECK(finite, status, kStatusNonFinite);
                }
#endif
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(out + obase + c0);
                    dst[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                        pack_bf16x2(o[6], o[7]));
                    dst[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                                        pack_bf16x2(o[14], o[15]));
                    if (out32) {                       // fp32 copy for the backward pass
                        float4* d32 = reinterpret_cast<float4*>(out32 + obase + c0);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            d32[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                    }
                }
            }
        }
        if (!ok) fail();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tbase, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host side

cudaError_t launch_fine_pair(const FineArgs& a, cudaStream_t stream) {
    using C = PairCfg<128>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fine_pair_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.g.B * a.g.heads * a.g.nt;
    const long long units = (rows + 1) / 2;
    const unsigned grid = (unsigned)(units < sms ? units : sms);
    const float scale_log2 = 1.4426950408889634f / sqrtf(128.f);
    const int ragged = (a.g.T % a.g.tt) || (a.g.H % a.g.th) || (a.g.W % a.g.tw);
    fine_pair_kernel<128><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(
        static_cast<const __nv_bfloat16*>(a.q), *a.mk, *a.mv, a.g, a.block_idx, a.topk, scale_log2, ragged,
        reinterpret_cast<__nv_bfloat16*>(a.out), a.out32, a.lse, a.status);
    return cudaGetLastError();
}

}  // namespace vsa
