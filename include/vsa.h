/*
 * vsa.h -- C ABI of a B200-native (sm_100a) block-sparse video attention
 * library: VSA-style trainable block-sparse attention with an optional
 * SLA/RoLA-style linear branch.
 *
 * What the method computes (sources, by page title and section):
 *  - "FastVideo 稀疏蒸馏技术深度解析" (omica.com.cn), section "2. 视频稀疏注意力VSA":
 *    video sparse attention picks, per block of queries, the key blocks that
 *    matter and evaluates only 10-20 % of the attention weights (sparsity
 *    0.8-0.9), staying compatible with exact Flash-Attention-style softmax.
 *  - SparkDiffusion news item (bazainvestora.ru), paragraphs 2-3: at 97 %
 *    sparsity 3 % of the blocks remain; RoLA adds a low-rank linear branch
 *    that keeps global context next to the block-sparse branch.
 *  - TurboDiffusion article (dolphinsci.com), section "稀疏、蒸馏与全链路量化":
 *    SLA = trainable sparse attention plus a linear-attention branch.
 * The pages leave the mechanics open; this library reads them as:
 *  tokens of a T x H x W latent grid are grouped into tt x th x tw cube tiles
 *  of 64 tokens (ceiling division; slots outside the grid are padding); each
 *  cube is mean-pooled over its valid tokens; a query cube i scores every key
 *  cube j with Qp[i].Kp[j]/sqrt(d) and keeps the top-k (ties -> lower j);
 *  the fine pass is exact softmax attention (scale 1/sqrt(d)) of each query
 *  over the valid tokens of its kept cubes; the optional linear branch adds
 *  phi(q) S / (phi(q).z) with phi = elu + 1, S = sum_n phi(k_n)^T v_n and
 *  z = sum_n phi(k_n) over all tokens.
 *
 * Conventions shared by every entry point
 *  - Shape arguments: B (batch), heads, head_dim d (64 or 128), grid T, H, W
 *    (token n = (t*H + h)*W + w, N = T*H*W), tile tt, th, tw with
 *    tt*th*tw == 64.  Cube j = (it*nh + ih)*nw + iw with nT = ceil(T/tt),
 *    nh = ceil(H/th), nw = ceil(W/tw), nt = nT*nh*nw; inside a cube, slot
 *    s = (dt*th + dh)*tw + dw.
 *  - q, k, v, out: bf16 (raw bit patterns, vsa_bf16), contiguous
 *    [B][N][heads][d] in device memory.
 *  - block_idx: int32 [B][heads][nt][topk] in device memory; each row is
 *    strictly ascending with values in [0, nt).
 *  - Every device pointer must be 16-byte aligned (TMA requirement).
 *  - The caller owns every buffer and the stream.  The library never
 *    allocates device memory, never frees it and never synchronises, except
 *    vsa_device_status.  It keeps no global state besides a cached driver
 *    entry point, per-device kernel attributes and the fixed device array of
 *    vsa_select_blocks_noalloc (end of this header).  It is re-entrant, except
 *    vsa_select_blocks_noalloc, whose calls share that array and must be
 *    ordered on one stream.
 *  - Faults recorded on the device: a bounded wait that gave up
 *    (VSA_ERR_TIMEOUT), a block index out of range or a misaligned shared
 *    memory window (VSA_ERR_DEVICE_CHECK); the debug-check build
 *    (libvsa_debug.so, compiled with -DVSA_DEBUG_CHECKS) also records a NaN
 *    or Inf reaching an output and a TMA box outside the grid
 *    (VSA_ERR_DEVICE_CHECK).  Nothing traps.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream).  Argument errors are reported before any launch;
 *    launch failures return VSA_ERR_CUDA.  Faults detected on the device
 *    (a bounded wait that gave up, a block index out of range) are recorded
 *    in the workspace's status word and reported by vsa_device_status.
 */
#ifndef VSA_H
#define VSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t vsa_bf16;                 /* raw bfloat16 bits            */
typedef struct CUstream_st* vsa_stream_t;  /* == cudaStream_t              */

typedef enum {
    VSA_OK = 0,
    VSA_ERR_INVALID_ARGUMENT = 1,  /* bad shape, null/misaligned pointer, bad topk */
    VSA_ERR_UNSUPPORTED = 2,       /* head_dim not in {64,128}, tile volume != 64,
                                      2^30 or more cubes in all (B*heads*nt)   */
    VSA_ERR_WORKSPACE = 3,         /* workspace missing or smaller than required   */
    VSA_ERR_CUDA = 4,              /* a CUDA runtime/driver call or launch failed  */
    VSA_ERR_TIMEOUT = 5,           /* a device-side bounded wait gave up           */
    VSA_ERR_DEVICE_CHECK = 6       /* a device-side range check failed             */
} vsa_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* vsa_status_string(vsa_status status);

/* Number of cube tiles nt of a T x H x W grid cut into tt x th x tw tiles
 * (ceiling division); 0 if any argument is < 1. */
int vsa_num_tiles(int T, int H, int W, int tt, int th, int tw);

/* Bytes of device workspace vsa_select_blocks and vsa_sparse_attn_fwd need
 * for these shapes: a 256-byte status block followed by a scratch area that
 * holds either the selection's intermediates (256 bytes of counters, the cube
 * means of q and k as fp32 hi + lo pairs [2][2][B][heads][nt][d], a
 * feature-major copy of the k means [B][heads][d][ntp] (ntp = nt rounded up
 * to a multiple of 4) and one fallback row of nt 64-bit keys for each of at
 * most 1024 CTAs: 256 + 16*B*heads*nt*d + 4*B*heads*d*ntp + 8192*nt bytes;
 * no nt x nt term), or the linear
 * branch's operand image (B*heads*(4*d*d + 4*d) bytes), whichever is larger (the backward passes' scratch fits it too: the
 * sparse branch's row terms and block-index transpose, the linear branch's
 * two operand images and fp32 gradient sums).  Returns 0 for invalid shapes.  The
 * same workspace may be passed to every call of one forward pass; calls that
 * share a workspace must be ordered on one stream. */
size_t vsa_workspace_bytes(int B, int heads, int head_dim, int T, int H, int W,
                           int tt, int th, int tw, int topk);

/* Clear the workspace's status word (enqueued on `stream`).  Call once after
 * allocating a workspace, before its first use. */
vsa_status vsa_workspace_init(void* workspace, size_t workspace_bytes, vsa_stream_t stream);

/* Tile gather: grid order x[B][N][heads][d] -> cube-major
 * x_tiles[B][heads][nt][64][d] (slot order above); padded slots are written
 * as zeros.  A bit-exact copy (the tiling step of the pages' block selection,
 * "2. 视频稀疏注意力VSA"). */
vsa_status vsa_gather_tiles(const vsa_bf16* x, vsa_bf16* x_tiles, int B, int heads,
                            int head_dim, int T, int H, int W, int tt, int th, int tw,
                            vsa_stream_t stream);

/* Tile scatter: cube-major x_tiles -> grid order x; only valid slots are
 * written (padded slots of x_tiles are ignored).  Bit-exact. */
vsa_status vsa_scatter_tiles(const vsa_bf16* x_tiles, vsa_bf16* x, int B, int heads,
                             int head_dim, int T, int H, int W, int tt, int th, int tw,
                             vsa_stream_t stream);

/* Block selection ("2. 视频稀疏注意力VSA": pick the key blocks each query block
 * attends to).  Mean-pools q and k per cube over valid tokens (fp64 sums),
 * scores C[i][j] = Qp[i].Kp[j]/sqrt(d) and writes, per (b, head, i), the
 * topk key cubes with the largest C (ties -> lower j) in ascending order to
 * block_idx.  The kept set is the one fp64 scores give: the scores are formed
 * in fp32 with a bound on their error, and every score the bound leaves
 * undecided is recomputed in fp64.  1 <= topk <= nt; nt up to about 3200
 * cubes (the 16 score rows of a work item live in shared memory: 64*nt +
 * 64*d + 14464 bytes must fit 227 KB, VSA_ERR_UNSUPPORTED beyond).  Needs
 * vsa_workspace_bytes() of workspace.  One kernel (after a memset of its
 * work counters, at most 256 bytes): the cube means go through the
 * workspace, the nt x nt scores only through shared memory. */
vsa_status vsa_select_blocks(const vsa_bf16* q, const vsa_bf16* k, int B, int heads,
                             int head_dim, int T, int H, int W, int tt, int th, int tw,
                             int topk, int32_t* block_idx, void* workspace,
                             size_t workspace_bytes, vsa_stream_t stream);

/* Linear-branch state (SparkDiffusion RoLA, paragraph 3; TurboDiffusion SLA,
 * "稀疏、蒸馏与全链路量化"): lin_S[B][heads][d][d] = sum_n phi(k_n)^T v_n and
 * lin_z[B][heads][d] = sum_n phi(k_n) over all N tokens, phi = elu + 1,
 * fp32 accumulation (phi split into bf16 hi + lo parts on the tensor cores).
 * Both outputs are fully overwritten.  The workspace (vsa_workspace_bytes()
 * of any tile shape, only its status word is used) receives device faults. */
vsa_status vsa_linear_branch_fwd(const vsa_bf16* k, const vsa_bf16* v, float* lin_S,
                                 float* lin_z, int B, int heads, int head_dim, int T, int H,
                                 int W, void* workspace, size_t workspace_bytes,
                                 vsa_stream_t stream);

/* Fine pass ("2. 视频稀疏注意力VSA": evaluate only the weights of the kept
 * blocks, exactly, Flash-Attention style).  For every valid query token of
 * cube i: softmax over the valid tokens of cubes block_idx[b][head][i][:] of
 * q.k/sqrt(d) (fp32 online softmax, bf16 tensor-core products), times v,
 * written as bf16 to out in grid order.  Padded slots take no part.  When
 * lin_S and lin_z are both non-NULL (from vsa_linear_branch_fwd) the linear
 * branch phi(q) S / (phi(q).z) is added in fp32 before rounding; pass both
 * NULL for the sparse branch alone.  Without the linear branch only the
 * workspace's status word is used; with it the call also writes a bf16 hi/lo
 * copy of (lin_S, lin_z) into the workspace scratch (B*heads*(4*d*d + 4*d)
 * bytes, within vsa_workspace_bytes()), so the scratch of an earlier
 * vsa_select_blocks on the same workspace is overwritten (block_idx is not).
 * Returns VSA_ERR_WORKSPACE when the workspace is smaller than that. */
vsa_status vsa_sparse_attn_fwd(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                               const int32_t* block_idx, const float* lin_S,
                               const float* lin_z, vsa_bf16* out, int B, int heads,
                               int head_dim, int T, int H, int W, int tt, int th, int tw,
                               int topk, void* workspace, size_t workspace_bytes,
                               vsa_stream_t stream);

/* Training forward: vsa_sparse_attn_fwd for the sparse branch alone that
 * also writes, for the backward pass, out_f32 (the same output in fp32,
 * [B][N][heads][d], padded slots not written) and lse[B][heads][nt][64]
 * (fp32, one value per cube slot): log2 of the softmax normaliser of the
 * row's scaled scores, i.e. m + log2(sum_m 2^(s_m*log2(e)/sqrt(d) - m));
 * +inf for padded slots.  Needs vsa_workspace_bytes() of workspace (status
 * word only). */
vsa_status vsa_sparse_attn_fwd_train(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                                     const int32_t* block_idx, vsa_bf16* out, float* out_f32,
                                     float* lse, int B, int heads, int head_dim, int T, int H, int W,
                                     int tt, int th, int tw, int topk, void* workspace,
                                     size_t workspace_bytes, vsa_stream_t stream);

/* Backward of the fine pass (the sparse branch is trainable: "FastVideo
 * 稀疏蒸馏技术深度解析", section "2. 视频稀疏注意力VSA"; TurboDiffusion article,
 * section "稀疏、蒸馏与全链路量化"), with block_idx held fixed: given q, k, v
 * and the output gradient `dout` (bf16 [B][N][heads][d]) and out_f32 and lse
 * from vsa_sparse_attn_fwd_train, writes bf16 dq, dk, dv (same layout,
 * fully overwritten; keys no query cube kept get 0):
 *     dv = P^T dout, dS = P o (dout v^T - rowsum(dout o out_f32)),
 *     dq = dS k / sqrt(d), dk = dS^T q / sqrt(d),
 * P recomputed from lse, products on the tensor cores with fp32
 * accumulation.  Uses the workspace scratch (vsa_workspace_bytes()) for the
 * row terms and the transpose of block_idx, so it overwrites an earlier
 * selection's scratch on the same workspace (not block_idx).  The transpose
 * keeps one bitmap row of nt bits in shared memory: nt <= 327680, else
 * VSA_ERR_UNSUPPORTED before any launch. */
vsa_status vsa_sparse_attn_bwd(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                               const float* out_f32, const vsa_bf16* dout, const int32_t* block_idx,
                               const float* lse, vsa_bf16* dq, vsa_bf16* dk, vsa_bf16* dv, int B,
                               int heads, int head_dim, int T, int H, int W, int tt, int th, int tw,
                               int topk, void* workspace, size_t workspace_bytes,
                               vsa_stream_t stream);

/* Backward of the linear branch (SparkDiffusion RoLA, paragraph 3;
 * TurboDiffusion SLA, "稀疏、蒸馏与全链路量化": the linear branch is trained
 * with the sparse one).  For lin_n = phi(q_n) S / (phi(q_n).z), phi = elu + 1,
 * with lin_S and lin_z from vsa_linear_branch_fwd over the same k and v, and
 * the output gradient dout (bf16 [B][N][heads][d]), writes the bf16
 * gradients of the branch to dq, dk, dv (same layout):
 *     u_n = S dout_n, e_n = -phi(q_n).u_n / (phi(q_n).z)^2,
 *     dq_n = (u_n / (phi(q_n).z) + e_n z) o phi'(q_n),
 *     dS = sum_n phi(q_n)^T dout_n / (phi(q_n).z),  dz = sum_n e_n phi(q_n),
 *     dk_m = (dS v_m + dz) o phi'(k_m),  dv_m = phi(k_m) dS,
 * products on the tensor cores with bf16 hi + lo operands (fp32-level) and
 * fp32 accumulation, dS and dz summed with fp32 atomics (run-to-run
 * differences at the fp32 rounding level).  accumulate == 0 overwrites dq,
 * dk, dv; accumulate != 0 adds the branch's gradients to the bf16 values
 * already there (e.g. from vsa_sparse_attn_bwd), rounding the sum once.
 * Uses B*heads*3*(4*d*d + 4*d) bytes (each third rounded up to 256) of the
 * workspace scratch, within vsa_workspace_bytes(); returns VSA_ERR_WORKSPACE
 * when the workspace is smaller. */
vsa_status vsa_linear_branch_bwd(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                                 const vsa_bf16* dout, const float* lin_S, const float* lin_z,
                                 vsa_bf16* dq, vsa_bf16* dk, vsa_bf16* dv, int accumulate, int B,
                                 int heads, int head_dim, int T, int H, int W, void* workspace,
                                 size_t workspace_bytes, vsa_stream_t stream);

/* Low-precision fine pass (sparse attention is orthogonal to low-bit tensor
 * cores: TurboDiffusion article, section "稀疏、蒸馏与全链路量化", SageSLA).
 * Step 1, vsa_quantize_qk_e4m3: per (b, head, cube) scale = amax / 448 (fp32,
 * over the cube's valid tokens and all d features; 1 for an all-zero cube)
 * and codes = FP8 E4M3 of x * (1 / scale) (reciprocal and product rounded to
 * nearest fp32; conversion nearest-even, saturating at 448), for q and k.  q8, k8: [B][N][heads][d] codes, one byte each (only
 * valid tokens are written); q_scale, k_scale: fp32 [B][heads][nt].  All
 * device pointers 16-byte aligned; no workspace. */
vsa_status vsa_quantize_qk_e4m3(const vsa_bf16* q, const vsa_bf16* k, uint8_t* q8, uint8_t* k8,
                                float* q_scale, float* k_scale, int B, int heads, int head_dim,
                                int T, int H, int W, int tt, int th, int tw, vsa_stream_t stream);

/* Step 2, vsa_sparse_attn_fwd_e4m3: the fine pass of vsa_sparse_attn_fwd with
 * Q K^T on the tensor cores in E4M3 (fp32 accumulation), scores rescaled by
 * q_scale[query cube] * k_scale[key cube], softmax and P V as in the bf16
 * pass (bf16 P and v), output bf16 in grid order.  head_dim 64 or 128; the
 * linear branch is added by
 * vsa_sparse_linear_attn_fwd_e4m3 below.  Needs
 * vsa_workspace_bytes() of workspace (status word only). */
vsa_status vsa_sparse_attn_fwd_e4m3(const uint8_t* q8, const uint8_t* k8, const float* q_scale,
                                    const float* k_scale, const vsa_bf16* v,
                                    const int32_t* block_idx, vsa_bf16* out, int B, int heads,
                                    int head_dim, int T, int H, int W, int tt, int th, int tw,
                                    int topk, void* workspace, size_t workspace_bytes,
                                    vsa_stream_t stream);

/* Low-precision sparse + linear attention (SageSLA: SLA built on SageAttention's
 * quantised products, TurboDiffusion article, section "稀疏、蒸馏与全链路量化"):
 * vsa_sparse_attn_fwd_e4m3 plus the linear branch of vsa_sparse_attn_fwd,
 *     out = softmax-pass(E4M3 Q K^T, bf16 P V) + phi(q) S / (phi(q) . z),
 * with lin_S, lin_z from vsa_linear_branch_fwd (fp32) and phi(q) computed
 * from the bf16 q (the quantisation covers the sparse branch's Q K^T only;
 * the branch's products run as bf16 hi + lo pairs, fp32-level, as in
 * vsa_sparse_attn_fwd).  q8, k8, q_scale, k_scale from vsa_quantize_qk_e4m3;
 * q, v bf16 [B][N][heads][d].  head_dim 64 or 128.  All pointers 16-byte
 * aligned (VSA_ERR_INVALID_ARGUMENT).
 * Needs vsa_workspace_bytes() of workspace: the status word plus the
 * operand image of (S, z) (VSA_ERR_WORKSPACE when smaller). */
vsa_status vsa_sparse_linear_attn_fwd_e4m3(const uint8_t* q8, const uint8_t* k8, const float* q_scale,
                                           const float* k_scale, const vsa_bf16* q, const vsa_bf16* v,
                                           const int32_t* block_idx, const float* lin_S,
                                           const float* lin_z, vsa_bf16* out, int B, int heads,
                                           int head_dim, int T, int H, int W, int tt, int th, int tw,
                                           int topk, void* workspace, size_t workspace_bytes,
                                           vsa_stream_t stream);

/* Self-test of the device failure path (no counterpart on the pages): a
 * one-warp kernel waits on a barrier nobody arrives at, gives up after
 * `limit_cycles` SM clock cycles exactly as the library's kernels do, and
 * records VSA_ERR_TIMEOUT in the workspace status word, which
 * vsa_device_status then returns.  No fault, trap or hang is involved; the
 * context stays usable.  limit_cycles > 0. */
vsa_status vsa_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                     unsigned int limit_cycles, vsa_stream_t stream);

/* Synchronise `stream`, then report and clear the device status word the
 * kernels of this workspace wrote: VSA_OK, VSA_ERR_TIMEOUT or
 * VSA_ERR_DEVICE_CHECK (VSA_ERR_CUDA if the stream itself failed). */
vsa_status vsa_device_status(void* workspace, vsa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Allocation-free block selection.
 *
 * No counterpart on the pages: this entry point exists for callers that cannot
 * allocate device memory (no cudaMalloc: a callback or runtime that forbids
 * allocation, a fixed memory budget, an embedding without an allocator) and
 * so cannot provide vsa_select_blocks' workspace.  It computes exactly what
 * vsa_select_blocks computes, with the same kernel, but keeps the
 * selection's intermediates (work counters, cube means, fallback rows) in one
 * file-scope device array of VSA_NOALLOC_SELECT_SCRATCH_BYTES, reserved on
 * every GPU that loads the library until the process exits.  It allocates and
 * frees nothing.
 *
 *  - The caller still passes q, k (device, bf16 [B][N][heads][d]) and
 *    block_idx (device, int32 [B][heads][nt][topk]), 16-byte aligned.
 *  - Shapes whose intermediates exceed the array
 *    (256 + 16*B*heads*nt*d + 4*B*heads*d*ntp + 8192*nt bytes, ntp = nt
 *    rounded up to 4, > the maximum) are rejected
 *    with VSA_ERR_WORKSPACE before anything is enqueued; argument errors as
 *    for vsa_select_blocks.
 *  - All calls share the array, which keeps the last call's contents; every
 *    call clears its work counters (a memset it enqueues) and rewrites what
 *    it reads.  Calls that overlap on the GPU (other streams, unordered host
 *    threads) race on it: order them on one stream.
 *  - There is no status word: a wait that gives up (the kernel's bounded
 *    wait for its own pooling, about 2 s) leaves rows of block_idx unwritten
 *    without a report.  vsa_select_blocks reports it as VSA_ERR_TIMEOUT.
 *  - The first call on each device (and the first after the device's
 *    primary context was reset) looks up the array's device address with that
 *    device current; make that first call before any stream capture.
 */
#define VSA_NOALLOC_SELECT_SCRATCH_BYTES (32u * 1024u * 1024u)

vsa_status vsa_select_blocks_noalloc(const vsa_bf16* q, const vsa_bf16* k, int B, int heads,
                                     int head_dim, int T, int H, int W, int tt, int th, int tw,
                                     int topk, int32_t* block_idx, vsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H */
