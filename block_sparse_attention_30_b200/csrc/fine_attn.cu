// fine_attn.cu -- the fine pass of block-sparse video attention on sm_100a.
//
// Source of the operation: "FastVideo 稀疏蒸馏技术深度解析" (omica.com.cn),
// section "2. 视频稀疏注意力VSA": only the attention weights of the selected
// key blocks are evaluated, exactly and Flash-Attention style.  Here a query
// block is one 64-token cube tile and every kept key block is a cube tile.
//
// One CTA owns one query cube (b, head, i) and runs online softmax over its
// top-k key cubes, two cubes (128 keys) per step:
//   * warp 4 (one lane) loads Q once and the K cube pairs, warp 6 (one lane)
//     the V cube pairs, into shared-memory rings with 5-D TMA boxes cut
//     straight from the [B][N][heads][d] tensors (box = d-chunk x tw x th x
//     tt), so the cube gather costs no extra pass and ragged edge cubes arrive
//     zero-filled;
//   * warp 5 (one lane) issues the tensor-core work: S = Q K^T (M=64 queries,
//     N=128 keys, A and B from shared memory) into TMEM, then, once softmax
//     has written P as bf16 over S in TMEM, O += P V (A = P from TMEM,
//     B = V from shared memory, MN-major).  S and O are double-buffered by
//     pair parity without extra TMEM columns: an M=64 accumulator fills only
//     lanes 0-15 of each 32-lane sub-partition, so buffer 1 lives in lanes
//     16-31 of the same columns.  S of pair p+2 is issued right after P V of
//     pair p, so softmax finds the next S ready; the output is
//     O(even pairs) + O(odd pairs);
//   * warps 0-3 (one TMEM sub-partition each; rows 16w..16w+15, each row
//     split in two 64-column halves over lanes t and t+16) do the fp32 online
//     softmax in the exp2 domain (softmax_step.cuh), rescale O in TMEM only
//     when a row maximum grows by more than 2^8, and finally write O / l (+ the
//     linear-branch term) as bf16 in grid order (the cube scatter, fused),
//     skipping padded slots.
// Two CTAs share an SM (256 TMEM columns and ~112 KB of shared memory each),
// so one CTA's softmax overlaps the other's MMAs.
//
// Low-precision variant (Q8): q and k arrive as FP8 E4M3 codes with one scale
// per (b, head, cube) (quant.cu); Q K^T runs as tcgen05 kind::f8f6f4 (K = 32
// per MMA; one row of d bytes per token: 128-byte swizzle at d = 128, 64-byte
// swizzle at d = 64), the softmax multiplies each half row by its query and
// key cube scales, P V stays bf16.  At d = 128 the halved Q and K tiles make
// room for a second V stage.  With the linear
// branch (SageSLA: the sparse + linear attention on quantised products), the
// branch itself stays bf16 hi + lo: phi(q) comes from the bf16 q in global
// memory and goes into the K ring, the (S, z) image into the V ring.
//
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

// Q8: the low-precision variant (q and k as E4M3 codes, one byte each).
template <int D, bool Q8 = false>
struct FineCfg {
    static constexpr int QB = Q8 ? 1 : 2;              // bytes per q / k element
    static constexpr int NCH = D / 64;                 // 128-byte d chunks of V
    static constexpr int QK_ROW = D * QB < 128 ? D * QB : 128;   // bytes of a Q / K box row
    static constexpr int NCH_QK = D * QB / QK_ROW;     // d chunks of Q and K (boxes per cube)
    static constexpr int QK_BOX = 64 * QK_ROW;         // bytes of one cube's box
    static constexpr int Q_BYTES = 64 * D * QB;        // one query cube
    static constexpr int K_CUBE_BYTES = 64 * D * QB;   // one key cube of K
    static constexpr int V_CUBE_BYTES = 64 * D * 2;    // one key cube of V
    static constexpr int K_PAIR_BYTES = 2 * K_CUBE_BYTES;
    static constexpr int V_PAIR_BYTES = 2 * V_CUBE_BYTES;
    static constexpr int CHUNK_STRIDE = 128 * 128;     // bytes between d chunks of a pair
    static constexpr int NK = (D == 128) ? 2 : 3;      // K pair stages
    static_assert(QK_ROW == 128 || (Q8 && D == 64), "64-byte rows only for E4M3 at d = 64");
    // the smaller K and Q of the low-precision variant leave room for a
    // second V stage within two CTAs per SM
    static constexpr int NV = (D == 128) ? (Q8 ? 2 : 1) : 3;   // V pair stages
    static constexpr int TMEM_COLS = 256;
    // A ring slot is free once the MMAs reading it are done.  With two K stages
    // the stage of pair p is the S buffer p & 1, so the K producer can wait on
    // s_full (the completion of Q K^T of pair p-2); with one V stage, on
    // o_ready (P V of pair p-1).  Neither barrier can run two phases ahead of
    // such a waiter, because its next completion needs the very load the
    // producer has not issued yet.  Deeper rings keep their own barriers.
    static constexpr bool K_ON_S = NK == 2;
    static constexpr bool V_ON_O = NV == 1;
    static constexpr int O_COL = 0;                    // fp32 O, D columns
    static constexpr int S_COL = 128;                  // fp32 S (128 cols) / bf16 P (64 cols)
    static constexpr int BAR_BYTES = 256;
    static constexpr int Z_BYTES = D * 4;              // linear branch: z (fp32)
    static constexpr int SMEM_BYTES = Q_BYTES + NK * K_PAIR_BYTES + NV * V_PAIR_BYTES + BAR_BYTES + Z_BYTES;
    // the linear branch's S hi + lo image must fit the K ring, phi(Q) lo the V
    // ring (bf16); low precision: phi(Q) hi + lo the K ring, the image the V ring
    static_assert(Q8 ? (2 * 64 * D * 2 <= NK * K_PAIR_BYTES && 4 * D * D <= NV * V_PAIR_BYTES)
                     : (4 * D * D <= NK * K_PAIR_BYTES && Q_BYTES <= NV * V_PAIR_BYTES), "linear operands");
};

template <int D, bool Q8 = false>
struct FineBars {
    uint64_t q_full;
    uint64_t k_full[FineCfg<D, Q8>::NK], k_empty[FineCfg<D, Q8>::NK];
    uint64_t v_full[FineCfg<D, Q8>::NV], v_empty[FineCfg<D, Q8>::NV];
    uint64_t s_full[2], p_full[2], o_ready[2];   // per S / O buffer (pair parity)
    uint64_t vc_full[2], v_half;                 // one V stage: per-cube halves (see the V producer)
    uint64_t mma_done, lin_full, lin_ready, lin_done;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(FineBars<128>) <= FineCfg<128>::BAR_BYTES, "barrier block");
static_assert(sizeof(FineBars<64>) <= FineCfg<64>::BAR_BYTES, "barrier block");
static_assert(sizeof(FineBars<128, true>) <= FineCfg<128, true>::BAR_BYTES, "barrier block");
static_assert(FineCfg<128, true>::SMEM_BYTES <= 232448 / 2 - 1024, "two CTAs per SM");
static_assert(sizeof(FineBars<64, true>) <= FineCfg<64, true>::BAR_BYTES, "barrier block");
static_assert(FineCfg<64, true>::SMEM_BYTES <= 232448 / 2 - 1024, "two CTAs per SM");

template <int D, bool LIN, bool Q8>
__global__ void __launch_bounds__(224, 2)
fine_attn_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                 const __grid_constant__ CUtensorMap mv, const Grid g,
                 const int32_t* __restrict__ block_idx, const int topk, const float scale_log2,
                 const int ragged, const uint8_t* __restrict__ lin_image,
                 __nv_bfloat16* __restrict__ out, float* __restrict__ out32, float* __restrict__ lse,
                 const float* __restrict__ q_scale, const float* __restrict__ k_scale,
                 const __nv_bfloat16* __restrict__ q_bf16, int* status) {
    using C = FineCfg<D, Q8>;

    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023) {               // uniform early exit, before any sync
        if (threadIdx.x == 0) report(status, kStatusMisaligned);
        return;
    }
    uint8_t* sQ = smem;
    uint8_t* sK = smem + C::Q_BYTES;
    uint8_t* sV = sK + C::NK * C::K_PAIR_BYTES;
    FineBars<D, Q8>* bars = reinterpret_cast<FineBars<D, Q8>*>(sV + C::NV * C::V_PAIR_BYTES);
    volatile int* abort_flag = &bars->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long row_id = blockIdx.x;                 // (b*heads + head)*nt + i
    const int i = (int)(row_id % g.nt);
    const int bh = (int)(row_id / g.nt);
    const int head = bh % g.heads, b = bh / g.heads;
    const int32_t* my_idx = block_idx + row_id * topk;
    const int n_pairs = (topk + 1) >> 1;
    constexpr bool lin = LIN;
    // Linear-branch operands reuse the buffers of the sparse pass:
    //   S hi / lo (B, MN-major) + z: one bulk copy of the (b, head) image into
    //     the K ring once the last Q K^T is done (bf16 q, k) or into the V
    //     ring once the last P V is done (E4M3 q, k), z into its own 512 bytes;
    //   phi(Q) hi / lo (A, K-major like a bf16 Q): bf16 q, k: hi over Q in
    //     place, lo in the V ring, once the last P V is done; E4M3 q, k: both
    //     in the K ring, from the bf16 q in global memory.
    uint8_t* sPhiHi = Q8 ? sK : sQ;
    uint8_t* sPhiLo = Q8 ? sK + 64 * D * 2 : sV;
    uint8_t* sSHi = Q8 ? sV : sK;
    uint8_t* sSLo = sSHi + D * D * 2;
    float* sZ = reinterpret_cast<float*>(sV + C::NV * C::V_PAIR_BYTES + C::BAR_BYTES);

    if (tid == 0) {
        bars->abort = 0;
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < C::NK; ++s) { mbar_init(&bars->k_full[s], 1); mbar_init(&bars->k_empty[s], 1); }
        for (int s = 0; s < C::NV; ++s) { mbar_init(&bars->v_full[s], 1); mbar_init(&bars->v_empty[s], 1); }
        mbar_init(&bars->vc_full[0], 1); mbar_init(&bars->vc_full[1], 1); mbar_init(&bars->v_half, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->p_full[x], 128);
            mbar_init(&bars->o_ready[x], 1);
        }
        mbar_init(&bars->mma_done, 1);
        mbar_init(&bars->lin_full, 1);
        mbar_init(&bars->lin_ready, 128);
        mbar_init(&bars->lin_done, 1);
        fence_barrier_init();
    }
    if (warp == 5) { tmem_alloc(&bars->tmem_base, C::TMEM_COLS); tmem_relinquish(); }
    if (warp == 4 && lane == 0) { tma_prefetch_desc(&mq); tma_prefetch_desc(&mk); tma_prefetch_desc(&mv); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = bars->tmem_base;

    auto fail = [&]() {
        *abort_flag = 1;
        report(status, kStatusTimeout);
    };

    if (warp == 4 || warp == 6) {
        // --------------------------------------- producers: Q + K (warp 4), V (warp 6)
        // Two warps, so that a wait for a free V slot never delays a K load.
        if (lane == 0) {
            const bool is_k = warp == 4;
            int issued = 0;
            if (is_k) {
                const TileCoord qc = tile_coord(g, i);
                VSA_DEBUG_CHECK(qc.t0 < g.T && qc.h0 < g.H && qc.w0 < g.W, status, kStatusBadCoord);
                mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
                for (int c = 0; c < C::NCH_QK; ++c)
                    tma_load_5d(sQ + c * C::QK_BOX, &mq, &bars->q_full, head * D + (C::QK_ROW / C::QB) * c, qc.w0,
                                qc.h0, qc.t0, b);
            }
            const int nst = is_k ? C::NK : C::NV;
            uint64_t* full = is_k ? bars->k_full : bars->v_full;
            uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
            uint8_t* ring = is_k ? sK : sV;
            const CUtensorMap* map = is_k ? &mk : &mv;
            // With one V stage the two cubes of a pair have a barrier each
            // (vc_full): cube 0 of pair p is loaded as soon as P V of pair
            // p - 1 has read its cube 0 (v_half), cube 1 once all of that
            // P V is done (o_ready), so the stage refills in two halves.
            const bool vsplit = C::V_ON_O && !is_k;
            int last_half[2] = {-1, -1};                // pair of the last load into each half
            int jn[2] = {__ldg(my_idx), topk > 1 ? __ldg(my_idx + 1) : 0};
            for (int p = 0; p < n_pairs; ++p) {
                const int ntl = min(2, topk - 2 * p);
                int jt[2] = {jn[0], jn[1]};
                if (p + 1 < n_pairs) {                      // next pair's cubes, in flight meanwhile
                    jn[0] = __ldg(my_idx + 2 * p + 2);
                    jn[1] = 2 * p + 3 < topk ? __ldg(my_idx + 2 * p + 3) : 0;
                }
                for (int t = 0; t < ntl; ++t)
                    if (jt[t] < 0 || jt[t] >= g.nt) { if (is_k) report(status, kStatusBadIndex); jt[t] = 0; }
                if (vsplit) {
                    bool ok_v = true;
                    for (int t = 0; t < ntl && ok_v; ++t) {
                        if (p >= 1) {
                            ok_v = t == 0 ? mbar_wait(&bars->v_half, (p - 1) & 1, abort_flag)
                                          : mbar_wait(&bars->o_ready[(p - 1) & 1], ((p - 1) >> 1) & 1, abort_flag);
                            if (!ok_v) break;
                        }
                        const TileCoord kc = tile_coord(g, jt[t]);
                        VSA_DEBUG_CHECK(kc.t0 < g.T && kc.h0 < g.H && kc.w0 < g.W, status, kStatusBadCoord);
                        mbar_arrive_expect_tx(&bars->vc_full[t], C::V_CUBE_BYTES);
                        for (int c = 0; c < C::NCH; ++c)
                            tma_load_5d(ring + c * C::CHUNK_STRIDE + t * 8192, map, &bars->vc_full[t],
                                        head * D + 64 * c, kc.w0, kc.h0, kc.t0, b);
                        last_half[t] = p;
                    }
                    if (!ok_v) { fail(); break; }
                    ++issued;
                    continue;
                }
                const int st = p % nst;
                if (p >= nst) {
                    uint64_t* bar = &empty[st];
                    uint32_t par = ((p / nst) - 1) & 1;
                    if (is_k && C::K_ON_S) { bar = &bars->s_full[p & 1]; par = ((p >> 1) - 1) & 1; }
                    if (!is_k && C::V_ON_O) { bar = &bars->o_ready[(p - 1) & 1]; par = ((p - 1) >> 1) & 1; }
                    if (!mbar_wait(bar, par, abort_flag)) { fail(); break; }
                }
                // K: NCH_QK chunks of QK_ROW / QB elements; V: NCH chunks of 64
                const int nch = is_k ? C::NCH_QK : C::NCH;
                const int cw = is_k ? C::QK_ROW / C::QB : 64;
                const int cube_box = is_k ? C::QK_BOX : 8192;
                const int pair_bytes = is_k ? C::K_PAIR_BYTES : C::V_PAIR_BYTES;
                mbar_arrive_expect_tx(&full[st], ntl * (is_k ? C::K_CUBE_BYTES : C::V_CUBE_BYTES));
                for (int t = 0; t < ntl; ++t) {
                    const TileCoord kc = tile_coord(g, jt[t]);
                    VSA_DEBUG_CHECK(kc.t0 < g.T && kc.h0 < g.H && kc.w0 < g.W, status, kStatusBadCoord);
                    for (int c = 0; c < nch; ++c)
                        tma_load_5d(ring + st * pair_bytes + c * C::CHUNK_STRIDE + t * cube_box, map,
                                    &full[st], head * D + cw * c, kc.w0, kc.h0, kc.t0, b);
                }
                ++issued;
            }
            bool lin_issued = false;
            if (lin && is_k != Q8 && issued == n_pairs && !*abort_flag) {
                // the (S, z) image goes into the K ring (bf16) or the V ring
                // (E4M3) once the last MMAs reading each of its stages are done
                bool free = true;
                for (int p = max(0, n_pairs - nst); p < n_pairs && free; ++p) {
                    if (is_k && C::K_ON_S) free = mbar_wait(&bars->s_full[p & 1], (p >> 1) & 1, abort_flag);
                    else if (!is_k && C::V_ON_O) free = mbar_wait(&bars->o_ready[p & 1], (p >> 1) & 1, abort_flag);
                    else free = mbar_wait(&empty[p % nst], (p / nst) & 1, abort_flag);
                }
                if (free) {
                    const uint8_t* img = lin_image + (long long)bh * (4 * D * D + 4 * D);
                    mbar_arrive_expect_tx(&bars->lin_full, 4 * D * D + 4 * D);
                    for (int off = 0; off < 4 * D * D; off += 16384)
                        bulk_load(sSHi + off, img + off, min(16384, 4 * D * D - off), &bars->lin_full);
                    bulk_load(sZ, img + 4 * D * D, 4 * D, &bars->lin_full);
                    lin_issued = true;
                } else {
                    fail();
                }
            }
            if (*abort_flag) {
                // drain: the last load issued into each stage must land before exit
                if (is_k) wait_noabort(&bars->q_full, 0);
                if (vsplit) {
                    for (int t = 0; t < 2; ++t)
                        if (last_half[t] >= 0) wait_noabort(&bars->vc_full[t], last_half[t] & 1);
                } else {
                    for (int n = max(0, issued - nst); n < issued; ++n)
                        wait_noabort(&full[n % nst], (n / nst) & 1);
                }
                if (lin_issued) wait_noabort(&bars->lin_full, 0);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
            // pair p uses S buffer p & 1 and O buffer p & 1: the M = 64
            // accumulators sit in TMEM lanes 0-15 (buffer 0) or 16-31 (buffer 1)
            // of the same columns
            auto tS = [&](int x) { return tbase + C::S_COL + ((uint32_t)x << 20); };   // lane 16 x
            auto tO = [&](int x) { return tbase + C::O_COL + ((uint32_t)x << 20); };
            const uint32_t id_pv = idesc_bf16_f32(64, D, false, true);
            auto issue_qk = [&](int p) -> bool {
                const int nkeys = min(2, topk - 2 * p) * 64;
                const int sk = p % C::NK;
                if (!mbar_wait(&bars->k_full[sk], (p / C::NK) & 1, abort_flag)) return false;
                tc_fence_after();
                if constexpr (Q8) {
                    // E4M3 codes: K = 32 per MMA, one row of D bytes per token
                    // (8-row groups of 1024 bytes at d = 128, 512 at d = 64)
                    const uint32_t id_s = idesc_e4m3_f32(64, nkeys, false, false);
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk) {
                        const uint32_t qa = q_addr + kk * 32, ka = k_addr + sk * C::K_PAIR_BYTES + kk * 32;
                        const uint64_t a = D == 128 ? smem_desc_sw128(qa, 16, 1024) : smem_desc_sw64(qa, 16, 512);
                        const uint64_t bd = D == 128 ? smem_desc_sw128(ka, 16, 1024) : smem_desc_sw64(ka, 16, 512);
                        mma_e4m3_ss(tS(p & 1), a, bd, id_s, kk > 0);
                    }
                } else {
                    const uint32_t id_s = idesc_bf16_f32(64, nkeys, false, false);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = smem_desc_sw128(q_addr + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(k_addr + sk * C::K_PAIR_BYTES + (kk >> 2) * C::CHUNK_STRIDE + (kk & 3) * 32, 16, 1024);
                        mma_bf16_ss(tS(p & 1), a, bd, id_s, kk > 0);
                    }
                }
                mma_commit(&bars->s_full[p & 1]);
                if (!C::K_ON_S) mma_commit(&bars->k_empty[sk]);
                return true;
            };
            // S of pair p + 2 is computed while softmax works on pair p + 1
            bool ok = mbar_wait(&bars->q_full, 0, abort_flag) && issue_qk(0) && (n_pairs < 2 || issue_qk(1));
            for (int p = 0; ok && p < n_pairs; ++p) {
                const int nkeys = min(2, topk - 2 * p) * 64;
                const int sv = p % C::NV, x = p & 1;
                if (!mbar_wait(&bars->p_full[x], (p >> 1) & 1, abort_flag)) { ok = false; break; }
                if constexpr (C::V_ON_O) {
                    // one V stage in two cube halves: the first 64 keys as soon
                    // as cube 0 landed, then release that half (v_half)
                    for (int t = 0; t < nkeys / 64; ++t) {
                        if (!mbar_wait(&bars->vc_full[t], p & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        for (int kk = 4 * t; kk < 4 * t + 4; ++kk) {
                            const uint64_t bd = smem_desc_sw128(v_addr + kk * 2048, C::CHUNK_STRIDE, 1024);
                            mma_bf16_ts(tO(x), tS(x) + kk * 8, bd, id_pv, (p >= 2 || kk > 0));
                        }
                        if (t == 0) mma_commit(&bars->v_half);
                    }
                    if (!ok) break;
                } else {
                    if (!mbar_wait(&bars->v_full[sv], (p / C::NV) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    for (int kk = 0; kk < nkeys / 16; ++kk) {
                        const uint64_t bd = smem_desc_sw128(v_addr + sv * C::V_PAIR_BYTES + kk * 2048, C::CHUNK_STRIDE, 1024);
                        mma_bf16_ts(tO(x), tS(x) + kk * 8, bd, id_pv, (p >= 2 || kk > 0));
                    }
                }
                mma_commit(&bars->o_ready[x]);
                if (!C::V_ON_O) mma_commit(&bars->v_empty[sv]);
                if (p + 2 < n_pairs && !issue_qk(p + 2)) { ok = false; break; }
            }
            if (ok && lin) {
                // Lin = phi(Q) S with S and phi(Q) split into bf16 hi + lo parts:
                // hi*hi + hi*lo + lo*hi, fp32 accumulation in the S columns.
                if (mbar_wait(&bars->lin_full, 0, abort_flag) && mbar_wait(&bars->lin_ready, 0, abort_flag)) {
                    tc_fence_after();
                    const uint32_t id_lin = idesc_bf16_f32(64, D, false, true);
                    const uint32_t a_hi = smem_u32(sPhiHi), a_lo = smem_u32(sPhiLo);
                    const uint32_t b_hi = smem_u32(sSHi), b_lo = smem_u32(sSLo);
                    for (int pass = 0; pass < 3; ++pass) {
                        const uint32_t aa = pass == 2 ? a_lo : a_hi;
                        const uint32_t bb = pass == 1 ? b_lo : b_hi;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t a = smem_desc_sw128(aa + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(bb + kk * 2048, D * 128, 1024);
                            mma_bf16_ss(tS(0), a, bd, id_lin, (pass > 0 || kk > 0));
                        }
                    }
                    mma_commit(&bars->lin_done);
                } else {
                    ok = false;
                }
            }
            if (!ok) fail();
            mma_commit(&bars->mma_done);
            wait_noabort(&bars->mma_done, 0);
        }
    } else {
        // --------------------------------------------------- softmax / epilogue
        const int r = 16 * warp + (lane & 15), hf = lane >> 4;
        // buffer x of this warp's rows: TMEM lanes 32*warp + 16*x .. + 15
        const uint32_t lane_base = tbase + ((uint32_t)(32 * warp) << 16);
        auto tS = [&](int x) { return lane_base + C::S_COL + ((uint32_t)x << 20); };
        auto tO = [&](int x) { return lane_base + C::O_COL + ((uint32_t)x << 20); };
        SoftmaxState sm{-INFINITY, 0.f};
        bool ok = true;
        // low-precision variant: raw scores are in units of the query cube's
        // scale times the key cube's scale
        const float sq_row = Q8 ? __ldg(q_scale + row_id) : 1.f;
        for (int p = 0; p < n_pairs; ++p) {
            const int ntl = min(2, topk - 2 * p);
            uint64_t vmask = hf < ntl ? ~0ull : 0ull;   // odd tail: this half has no cube
            float sc = scale_log2;
            if ((ragged || Q8) && hf < ntl) {
                int j = __ldg(my_idx + 2 * p + hf);
                if (j < 0 || j >= g.nt) j = 0;
                if (ragged) vmask = valid_slot_mask(g, tile_coord(g, j));   // edge cubes: mask padded keys
                if (Q8) sc = scale_log2 * sq_row * __ldg(k_scale + (long long)bh * g.nt + j);
            }
            const int x = p & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[x], (p >> 1) & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            float s[64];
            tmem_ld_16x32bx2_x16<64>(tS(x) + 0, *reinterpret_cast<float(*)[16]>(&s[0]));
            tmem_ld_16x32bx2_x16<64>(tS(x) + 16, *reinterpret_cast<float(*)[16]>(&s[16]));
            tmem_ld_16x32bx2_x16<64>(tS(x) + 32, *reinterpret_cast<float(*)[16]>(&s[32]));
            tmem_ld_16x32bx2_x16<64>(tS(x) + 48, *reinterpret_cast<float(*)[16]>(&s[48]));
            tmem_wait_ld();
            uint32_t pk[32];
            bool resc;
            const bool masked = __any_sync(0xffffffffu, vmask != ~0ull);
            const float alpha = masked ? softmax_step<true>(s, vmask, sc, sm, resc, pk)
                                       : softmax_step<false>(s, vmask, sc, sm, resc, pk);
            tmem_st_16x32bx2_x32(tS(x), pk);
            if (p > 0 && __any_sync(0xffffffffu, resc)) {
                // the two O buffers hold PV up to pair p-1 (the completion of
                // PV(p-1) implies that of every earlier MMA): rescale in place
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_ready[(p - 1) & 1], ((p - 1) >> 1) & 1, abort_flag))) { ok = false; break; }
                tc_fence_after();
                for (int ob = 0; ob < min(p, 2); ++ob) {
#pragma unroll
                    for (int c0 = 0; c0 < D / 2; c0 += 16) {
                        float o[16];
                        tmem_ld_16x32bx2_x16<D / 2>(tO(ob) + c0, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] *= alpha;
                        tmem_st_16x32bx2_x16<D / 2>(tO(ob) + c0, o);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[x]);
        }
        if (ok && !__all_sync(0xffffffffu, mbar_wait(&bars->o_ready[(n_pairs - 1) & 1], ((n_pairs - 1) >> 1) & 1, abort_flag))) ok = false;
        // this thread's query slot: token n of the grid, if the slot is valid
        const TileCoord qc = tile_coord(g, i);
        const int dt = r / (g.th * g.tw), dh = (r / g.tw) % g.th, dw = r % g.tw;
        const bool valid = dt < qc.vt && dh < qc.vh && dw < qc.vw;
        const long long n = ((long long)(qc.t0 + dt) * g.H + (qc.h0 + dh)) * g.W + (qc.w0 + dw);
        // ------------------------------------------------------- linear branch
        // phi(q) = elu(q) + 1 (SparkDiffusion RoLA / TurboDiffusion SLA linear
        // branch).  Each thread owns half a query row: D/2 features.
        float den = 1.f;
        if (ok && lin && !__all_sync(0xffffffffu, mbar_wait(&bars->lin_full, 0, abort_flag))) ok = false;
        if (ok && lin) {
            tc_fence_after();
            const float* zb = sZ + hf * (D / 2);
            float dpart = 0.f;
            // phi(Q) hi/lo: this thread's D/2 features sit in chunk (hf*(D/2))/64
            // of a bf16 Q cube, 16-byte units u0 .. u0 + D/16 - 1 of row r.
            // bf16 q, k: q is read from the Q tile, hi replaces it in place and
            // lo goes to the same offset in the V ring.  E4M3 q, k: q is read
            // from global memory (0 for padded slots), hi and lo go to the two
            // halves of the K ring, which the last Q K^T no longer needs.
            const int chunk = (hf * (D / 2)) / 64, u0 = ((hf * (D / 2)) % 64) / 8;
            const uint4* qrow = reinterpret_cast<const uint4*>(
                q_bf16 + (((long long)b * g.N + n) * g.heads + head) * D + hf * (D / 2));
#pragma unroll
            for (int u = 0; u < D / 16; ++u) {
                const int uu = u0 + u;
                const uint32_t off = chunk * 8192 + r * 128 + (((uu) ^ (r & 7)) << 4);
                uint4 raw;
                if constexpr (Q8) raw = valid ? __ldg(qrow + u) : make_uint4(0u, 0u, 0u, 0u);
                else raw = *reinterpret_cast<const uint4*>(sQ + off);
                const float4 z0 = reinterpret_cast<const float4*>(zb + u * 8)[0];
                const float4 z1 = reinterpret_cast<const float4*>(zb + u * 8)[1];
                const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float q0 = __uint_as_float(w[e] << 16), q1 = __uint_as_float(w[e] & 0xffff0000u);
                    const float f0 = q0 > 0.f ? q0 + 1.f : __expf(q0);
                    const float f1 = q1 > 0.f ? q1 + 1.f : __expf(q1);
                    dpart += f0 * zz[2 * e] + f1 * zz[2 * e + 1];
                    hi[e] = pack_bf16x2(f0, f1);
                    lo[e] = pack_bf16x2(f0 - __uint_as_float(hi[e] << 16), f1 - __uint_as_float(hi[e] & 0xffff0000u));
                }
                *reinterpret_cast<uint4*>(sPhiHi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(sPhiLo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            den = dpart + __shfl_xor_sync(0xffffffffu, dpart, 16);
            fence_proxy_async_smem();
            mbar_arrive(&bars->lin_ready);
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->lin_done, 0, abort_flag))) ok = false;
        }
        if (!ok) fail();
        // ------------------------------------------------------------ epilogue
        if (ok) {
            tc_fence_after();
            const float l = sm.l_run + __shfl_xor_sync(0xffffffffu, sm.l_run, 16);
            const float inv = 1.f / l;
            const float inv_den = 1.f / den;
            __nv_bfloat16* orow = out + (((long long)b * g.N + n) * g.heads + head) * D + hf * (D / 2);
            // log2 of the softmax normaliser of the scaled scores (for the
            // backward pass); +inf marks padded query slots (zero weight there)
            if (lse && hf == 0) lse[row_id * 64 + r] = valid ? sm.m_run + __log2f(l) : INFINITY;
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 16) {
                float o[16];
                tmem_ld_16x32bx2_x16<D / 2>(tO(0) + c0, o);
                if (n_pairs > 1) {                     // O = O(even pairs) + O(odd pairs)
                    float o1[16];
                    tmem_ld_16x32bx2_x16<D / 2>(tO(1) + c0, o1);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] += o1[e];
                }
                if (lin) {
                    float li[16];
                    tmem_ld_16x32bx2_x16<D / 2>(tS(0) + c0, li);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = o[e] * inv + li[e] * inv_den;
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] *= inv;
                }
#ifdef VSA_DEBUG_CHECKS
                if (valid) {
                    bool finite = true;
#pragma unroll
                    for (int e = 0; e < 16; ++e) finite = finite && isfinite(o[e]);
                    VSA_DEBUG_CHECK(finite, status, kStatusNonFinite);
                }
#endif
                uint4 w0, w1;
                w0.x = pack_bf16x2(o[0], o[1]);
                w0.y = pack_bf16x2(o[2], o[3]);
                w0.z = pack_bf16x2(o[4], o[5]);
                w0.w = pack_bf16x2(o[6], o[7]);
                w1.x = pack_bf16x2(o[8], o[9]);
                w1.y = pack_bf16x2(o[10], o[11]);
                w1.z = pack_bf16x2(o[12], o[13]);
                w1.w = pack_bf16x2(o[14], o[15]);
                if (valid) {
                    reinterpret_cast<uint4*>(orow + c0)[0] = w0;
                    reinterpret_cast<uint4*>(orow + c0)[1] = w1;
                    if (out32) {                       // fp32 copy for the backward pass
                        float4* o4 = reinterpret_cast<float4*>(
                            out32 + (((long long)b * g.N + n) * g.heads + head) * D + hf * (D / 2) + c0);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            o4[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tbase, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host side

template <int D, bool LIN, bool Q8 = false>
static cudaError_t launch_fine_impl(const FineArgs& a, cudaStream_t stream) {
    using C = FineCfg<D, Q8>;
    static int configured_device = -1;   // per process: attribute set once per device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(fine_attn_kernel<D, LIN, Q8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const long long rows = (long long)a.g.B * a.g.heads * a.g.nt;
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    const int ragged = (a.g.T % a.g.tt) || (a.g.H % a.g.th) || (a.g.W % a.g.tw);
    fine_attn_kernel<D, LIN, Q8><<<(unsigned)rows, 224, C::SMEM_BYTES, stream>>>(
        *a.mq, *a.mk, *a.mv, a.g, a.block_idx, a.topk, scale_log2, ragged,
        static_cast<const uint8_t*>(a.lin_image), reinterpret_cast<__nv_bfloat16*>(a.out), a.out32, a.lse,
        a.q_scale, a.k_scale, static_cast<const __nv_bfloat16*>(a.q), a.status);
    return cudaGetLastError();
}

cudaError_t launch_fine_single(const FineArgs& a, cudaStream_t stream) {
    const bool lin = a.lin_image != nullptr;
    if (a.q_scale && a.g.d == 128)                                      // E4M3 q, k
        return lin ? launch_fine_impl<128, true, true>(a, stream) : launch_fine_impl<128, false, true>(a, stream);
    if (a.q_scale) return lin ? launch_fine_impl<64, true, true>(a, stream) : launch_fine_impl<64, false, true>(a, stream);
    if (a.g.d == 128) return lin ? launch_fine_impl<128, true>(a, stream) : launch_fine_impl<128, false>(a, stream);
    return lin ? launch_fine_impl<64, true>(a, stream) : launch_fine_impl<64, false>(a, stream);
}

// Kernel choice for the bf16, d = 128 sparse branch.  Short rows (few kept
// cubes per query cube) go to the persistent two-cube kernel (fine_pair.cu),
// which pays a CTA's set-up and pipeline fill once per SM instead of once
// per query cube; long rows amortise that set-up and run faster here, with
// one CTA per query cube and two CTAs per SM (measured on B200 at the 97 %
// shape, k = 11: 0.196 vs 0.212 ms; at 14B-480P, k = 46: 2.63 vs 2.42 ms).
constexpr int kPairMaxTopk = 24;

cudaError_t launch_fine(const FineArgs& a, cudaStream_t stream) {
    if (!a.q_scale && !a.lin_image && a.g.d == 128 && a.topk <= kPairMaxTopk) return launch_fine_pair(a, stream);
    return launch_fine_single(a, stream);
}

int fine_smem_bytes(int d) { return d == 128 ? FineCfg<128>::SMEM_BYTES : FineCfg<64>::SMEM_BYTES; }

}  // namespace vsa
