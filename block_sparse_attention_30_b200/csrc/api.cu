// api.cu -- the C ABI declared in include/vsa.h: argument validation,
// workspace layout, TMA descriptor encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/vsa.h"
#include "common.cuh"
#include "fine_attn.h"
#include "linear.h"
#include "quant.h"
#include "select.h"
#include "tiles.h"
#include "fine_bwd.h"

namespace {

constexpr size_t kStatusBytes = 256;     // status block at the start of the workspace

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

vsa_status check_shape(int B, int heads, int d, int T, int H, int W, int tt, int th, int tw) {
    switch (vsa::shape_error(B, heads, d, T, H, W, tt, th, tw)) {
        case 0: break;
        case 2: return VSA_ERR_UNSUPPORTED;
        default: return VSA_ERR_INVALID_ARGUMENT;
    }
    // the fine pass and its backward launch one or two CTAs per (b, head,
    // query cube): at most 2^30 cubes in all
    const long long nt = (long long)vsa::ceil_div_i(T, tt) * vsa::ceil_div_i(H, th) * vsa::ceil_div_i(W, tw);
    if ((long long)B * heads * nt >= (1ll << 30)) return VSA_ERR_UNSUPPORTED;
    return VSA_OK;
}

vsa::Grid grid_of(int B, int heads, int d, int T, int H, int W, int tt, int th, int tw) {
    return vsa::make_grid(B, heads, d, T, H, W, tt, th, tw);
}

// Workspace scratch the linear-branch apply needs: one operand image per (b, head).
size_t lin_image_bytes(const vsa::Grid& g) {
    return (size_t)g.B * g.heads * (size_t)vsa::linear_image_bytes(g.d);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 5-D view of a [B][N][heads][d] bf16 tensor as (heads*d, W, H, T, B) with a
// box of one 64-element d chunk x one cube (tw x th x tt) of one batch; the
// box lands in shared memory as 64 rows of 128 bytes in cube-slot order with
// the 128-byte swizzle, and out-of-grid slots are zero-filled.
bool encode_grid_map(CUtensorMap* m, const void* base, const vsa::Grid& g) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t row = (cuuint64_t)g.heads * g.d;
    cuuint64_t dims[5] = {row, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T, (cuuint64_t)g.B};
    cuuint64_t strides[4] = {row * 2, row * 2 * g.W, row * 2 * g.W * g.H, row * 2 * g.W * g.H * g.T};
    cuuint32_t box[5] = {64, (cuuint32_t)g.tw, (cuuint32_t)g.th, (cuuint32_t)g.tt, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same 5-D view over E4M3 codes (one byte per element): box {d codes
// (the whole d of a head: 128 bytes with the 128-byte swizzle at d = 128,
// 64 bytes with the 64-byte swizzle at d = 64), tw, th, tt, 1}.
bool encode_grid_map_u8(CUtensorMap* m, const void* base, const vsa::Grid& g) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t row = (cuuint64_t)g.heads * g.d;
    cuuint64_t dims[5] = {row, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T, (cuuint64_t)g.B};
    cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.H, row * g.W * g.H * g.T};
    cuuint32_t box[5] = {(cuuint32_t)g.d, (cuuint32_t)g.tw, (cuuint32_t)g.th, (cuuint32_t)g.tt, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, g.d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

vsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA; }

}  // namespace

extern "C" {
#pragma GCC visibility push(default)

const char* vsa_status_string(vsa_status s) {
    switch (s) {
        case VSA_OK: return "VSA_OK";
        case VSA_ERR_INVALID_ARGUMENT: return "VSA_ERR_INVALID_ARGUMENT";
        case VSA_ERR_UNSUPPORTED: return "VSA_ERR_UNSUPPORTED";
        case VSA_ERR_WORKSPACE: return "VSA_ERR_WORKSPACE";
        case VSA_ERR_CUDA: return "VSA_ERR_CUDA";
        case VSA_ERR_TIMEOUT: return "VSA_ERR_TIMEOUT";
        case VSA_ERR_DEVICE_CHECK: return "VSA_ERR_DEVICE_CHECK";
    }
    return "VSA_ERR_UNKNOWN";
}

int vsa_num_tiles(int T, int H, int W, int tt, int th, int tw) {
    if (T < 1 || H < 1 || W < 1 || tt < 1 || th < 1 || tw < 1) return 0;
    return vsa::ceil_div_i(T, tt) * vsa::ceil_div_i(H, th) * vsa::ceil_div_i(W, tw);
}

size_t vsa_workspace_bytes(int B, int heads, int head_dim, int T, int H, int W, int tt, int th,
                           int tw, int topk) {
    if (check_shape(B, heads, head_dim, T, H, W, tt, th, tw) != VSA_OK) return 0;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return 0;
    size_t scratch = vsa::select_scratch_bytes(g);
    const size_t image = lin_image_bytes(g);
    const size_t bwd = vsa::bwd_scratch_bytes(g, topk);
    const size_t lin_bwd = (size_t)vsa::linear_bwd_scratch_bytes(g);
    if (image > scratch) scratch = image;
    if (bwd > scratch) scratch = bwd;
    if (lin_bwd > scratch) scratch = lin_bwd;
    return kStatusBytes + scratch;
}

vsa_status vsa_workspace_init(void* workspace, size_t workspace_bytes, vsa_stream_t stream) {
    if (!aligned16(workspace)) return VSA_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < kStatusBytes) return VSA_ERR_WORKSPACE;
    return from_cuda(cudaMemsetAsync(workspace, 0, kStatusBytes, (cudaStream_t)stream));
}

vsa_status vsa_gather_tiles(const vsa_bf16* x, vsa_bf16* x_tiles, int B, int heads, int head_dim,
                            int T, int H, int W, int tt, int th, int tw, vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    if (!aligned16(x) || !aligned16(x_tiles)) return VSA_ERR_INVALID_ARGUMENT;
    return from_cuda(vsa::launch_gather(grid_of(B, heads, head_dim, T, H, W, tt, th, tw), x, x_tiles,
                                        (cudaStream_t)stream));
}

vsa_status vsa_scatter_tiles(const vsa_bf16* x_tiles, vsa_bf16* x, int B, int heads, int head_dim,
                             int T, int H, int W, int tt, int th, int tw, vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    if (!aligned16(x) || !aligned16(x_tiles)) return VSA_ERR_INVALID_ARGUMENT;
    return from_cuda(vsa::launch_scatter(grid_of(B, heads, head_dim, T, H, W, tt, th, tw), x_tiles,
                                         x, (cudaStream_t)stream));
}

vsa_status vsa_select_blocks(const vsa_bf16* q, const vsa_bf16* k, int B, int heads, int head_dim,
                             int T, int H, int W, int tt, int th, int tw, int topk,
                             int32_t* block_idx, void* workspace, size_t workspace_bytes,
                             vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(block_idx)) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    if (!vsa::select_supported(g)) return VSA_ERR_UNSUPPORTED;
    if (workspace_bytes < kStatusBytes + vsa::select_scratch_bytes(g)) return VSA_ERR_WORKSPACE;
    vsa::SelectArgs a;
    a.g = g;
    a.q = q;
    a.k = k;
    a.topk = topk;
    a.block_idx = block_idx;
    a.scratch = static_cast<uint8_t*>(workspace) + kStatusBytes;
    a.status = static_cast<int*>(workspace);
    return from_cuda(vsa::launch_select(a, (cudaStream_t)stream));
}

vsa_status vsa_linear_branch_fwd(const vsa_bf16* k, const vsa_bf16* v, float* lin_S, float* lin_z,
                                 int B, int heads, int head_dim, int T, int H, int W,
                                 void* workspace, size_t workspace_bytes, vsa_stream_t stream) {
    // the tile shape does not enter the linear branch; any valid one will do
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, 4, 4, 4);
    if (s != VSA_OK) return s;
    if (!aligned16(k) || !aligned16(v) || !aligned16(lin_S) || !aligned16(lin_z))
        return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    if (workspace_bytes < kStatusBytes) return VSA_ERR_WORKSPACE;
    auto fn = encode_fn();
    if (!fn) return VSA_ERR_CUDA;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, 4, 4, 4);
    return from_cuda(vsa::launch_linear_state(g, k, v, lin_S, lin_z, static_cast<int*>(workspace),
                                              (cudaStream_t)stream, fn));
}

vsa_status vsa_sparse_attn_fwd(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                               const int32_t* block_idx, const float* lin_S, const float* lin_z,
                               vsa_bf16* out, int B, int heads, int head_dim, int T, int H, int W,
                               int tt, int th, int tw, int topk, void* workspace,
                               size_t workspace_bytes, vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(block_idx) || !aligned16(out))
        return VSA_ERR_INVALID_ARGUMENT;
    if ((lin_S == nullptr) != (lin_z == nullptr)) return VSA_ERR_INVALID_ARGUMENT;
    if (lin_S && (!aligned16(lin_S) || !aligned16(lin_z))) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    if (workspace_bytes < kStatusBytes + (lin_S ? lin_image_bytes(g) : 0)) return VSA_ERR_WORKSPACE;
    CUtensorMap mq, mk, mv;
    if (!encode_grid_map(&mq, q, g) || !encode_grid_map(&mk, k, g) || !encode_grid_map(&mv, v, g))
        return VSA_ERR_CUDA;
    vsa::FineArgs a;
    a.g = g;
    a.q = q;
    a.mq = &mq;
    a.mk = &mk;
    a.mv = &mv;
    a.block_idx = block_idx;
    a.topk = topk;
    a.lin_image = nullptr;
    a.out = out;
    a.out32 = nullptr;
    a.lse = nullptr;
    a.q_scale = a.k_scale = nullptr;
    a.status = static_cast<int*>(workspace);
    if (lin_S) {
        // the bf16 hi/lo operand image of (S, z) goes into the workspace scratch
        a.lin_image = static_cast<uint8_t*>(workspace) + kStatusBytes;
        cudaError_t e = vsa::launch_linear_pack(g, lin_S, lin_z, const_cast<void*>(a.lin_image),
                                                (cudaStream_t)stream);
        if (e != cudaSuccess) return from_cuda(e);
    }
    return from_cuda(vsa::launch_fine(a, (cudaStream_t)stream));
}

vsa_status vsa_sparse_attn_fwd_train(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                                     const int32_t* block_idx, vsa_bf16* out, float* out_f32,
                                     float* lse, int B, int heads, int head_dim, int T, int H, int W,
                                     int tt, int th, int tw, int topk, void* workspace,
                                     size_t workspace_bytes, vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(block_idx) || !aligned16(out) ||
        !aligned16(out_f32) || !aligned16(lse))
        return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    if (workspace_bytes < kStatusBytes) return VSA_ERR_WORKSPACE;
    CUtensorMap mq, mk, mv;
    if (!encode_grid_map(&mq, q, g) || !encode_grid_map(&mk, k, g) || !encode_grid_map(&mv, v, g))
        return VSA_ERR_CUDA;
    vsa::FineArgs a;
    a.g = g;
    a.q = q;
    a.mq = &mq;
    a.mk = &mk;
    a.mv = &mv;
    a.block_idx = block_idx;
    a.topk = topk;
    a.lin_image = nullptr;
    a.out = out;
    a.out32 = out_f32;
    a.lse = lse;
    a.q_scale = a.k_scale = nullptr;
    a.status = static_cast<int*>(workspace);
    return from_cuda(vsa::launch_fine(a, (cudaStream_t)stream));
}

vsa_status vsa_sparse_attn_bwd(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                               const float* out_f32, const vsa_bf16* dout, const int32_t* block_idx,
                               const float* lse, vsa_bf16* dq, vsa_bf16* dk, vsa_bf16* dv, int B,
                               int heads, int head_dim, int T, int H, int W, int tt, int th, int tw,
                               int topk, void* workspace, size_t workspace_bytes,
                               vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return VSA_ERR_INVALID_ARGUMENT;
    if (!vsa::bwd_supported(g)) return VSA_ERR_UNSUPPORTED;
    for (const void* p : {(const void*)q, (const void*)k, (const void*)v, (const void*)out_f32,
                          (const void*)dout, (const void*)block_idx, (const void*)lse, (const void*)dq,
                          (const void*)dk, (const void*)dv})
        if (!aligned16(p)) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    if (workspace_bytes < kStatusBytes + vsa::bwd_scratch_bytes(g, topk)) return VSA_ERR_WORKSPACE;
    CUtensorMap mq, mk, mv, mg;
    if (!encode_grid_map(&mq, q, g) || !encode_grid_map(&mk, k, g) || !encode_grid_map(&mv, v, g) ||
        !encode_grid_map(&mg, dout, g))
        return VSA_ERR_CUDA;
    vsa::BwdArgs a;
    a.g = g;
    a.mq = &mq;
    a.mk = &mk;
    a.mv = &mv;
    a.mg = &mg;
    a.block_idx = block_idx;
    a.topk = topk;
    a.out32 = out_f32;
    a.dout = dout;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.scratch = static_cast<uint8_t*>(workspace) + kStatusBytes;
    a.status = static_cast<int*>(workspace);
    return from_cuda(vsa::launch_fine_bwd(a, (cudaStream_t)stream));
}

vsa_status vsa_linear_branch_bwd(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                                 const vsa_bf16* dout, const float* lin_S, const float* lin_z,
                                 vsa_bf16* dq, vsa_bf16* dk, vsa_bf16* dv, int accumulate, int B,
                                 int heads, int head_dim, int T, int H, int W, void* workspace,
                                 size_t workspace_bytes, vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, 4, 4, 4);
    if (s != VSA_OK) return s;
    for (const void* p : {(const void*)q, (const void*)k, (const void*)v, (const void*)dout,
                          (const void*)lin_S, (const void*)lin_z, (const void*)dq, (const void*)dk,
                          (const void*)dv})
        if (!aligned16(p)) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, 4, 4, 4);
    if (workspace_bytes < kStatusBytes + (size_t)vsa::linear_bwd_scratch_bytes(g)) return VSA_ERR_WORKSPACE;
    auto fn = encode_fn();
    if (!fn) return VSA_ERR_CUDA;
    return from_cuda(vsa::launch_linear_bwd(g, q, k, v, dout, lin_S, lin_z, dq, dk, dv, accumulate,
                                            static_cast<uint8_t*>(workspace) + kStatusBytes,
                                            static_cast<int*>(workspace), (cudaStream_t)stream, fn));
}

vsa_status vsa_quantize_qk_e4m3(const vsa_bf16* q, const vsa_bf16* k, uint8_t* q8, uint8_t* k8,
                                float* q_scale, float* k_scale, int B, int heads, int head_dim,
                                int T, int H, int W, int tt, int th, int tw, vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    for (const void* p : {(const void*)q, (const void*)k, (const void*)q8, (const void*)k8,
                          (const void*)q_scale, (const void*)k_scale})
        if (!aligned16(p)) return VSA_ERR_INVALID_ARGUMENT;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    return from_cuda(vsa::launch_quant_e4m3(g, q, k, q8, k8, q_scale, k_scale, (cudaStream_t)stream));
}

vsa_status vsa_sparse_attn_fwd_e4m3(const uint8_t* q8, const uint8_t* k8, const float* q_scale,
                                    const float* k_scale, const vsa_bf16* v,
                                    const int32_t* block_idx, vsa_bf16* out, int B, int heads,
                                    int head_dim, int T, int H, int W, int tt, int th, int tw,
                                    int topk, void* workspace, size_t workspace_bytes,
                                    vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return VSA_ERR_INVALID_ARGUMENT;
    for (const void* p : {(const void*)q8, (const void*)k8, (const void*)q_scale, (const void*)k_scale,
                          (const void*)v, (const void*)block_idx, (const void*)out})
        if (!aligned16(p)) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    if (workspace_bytes < kStatusBytes) return VSA_ERR_WORKSPACE;
    CUtensorMap mq, mk, mv;
    if (!encode_grid_map_u8(&mq, q8, g) || !encode_grid_map_u8(&mk, k8, g) || !encode_grid_map(&mv, v, g))
        return VSA_ERR_CUDA;
    vsa::FineArgs a;
    a.g = g;
    a.q = nullptr;             // no linear branch: no bf16 q needed
    a.mq = &mq;
    a.mk = &mk;
    a.mv = &mv;
    a.block_idx = block_idx;
    a.topk = topk;
    a.lin_image = nullptr;
    a.out = out;
    a.out32 = nullptr;
    a.lse = nullptr;
    a.q_scale = q_scale;
    a.k_scale = k_scale;
    a.status = static_cast<int*>(workspace);
    return from_cuda(vsa::launch_fine(a, (cudaStream_t)stream));
}

vsa_status vsa_sparse_linear_attn_fwd_e4m3(const uint8_t* q8, const uint8_t* k8, const float* q_scale,
                                           const float* k_scale, const vsa_bf16* q, const vsa_bf16* v,
                                           const int32_t* block_idx, const float* lin_S,
                                           const float* lin_z, vsa_bf16* out, int B, int heads,
                                           int head_dim, int T, int H, int W, int tt, int th, int tw,
                                           int topk, void* workspace, size_t workspace_bytes,
                                           vsa_stream_t stream) {
    vsa_status s = check_shape(B, heads, head_dim, T, H, W, tt, th, tw);
    if (s != VSA_OK) return s;
    const vsa::Grid g = grid_of(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return VSA_ERR_INVALID_ARGUMENT;
    for (const void* p : {(const void*)q8, (const void*)k8, (const void*)q_scale, (const void*)k_scale,
                          (const void*)q, (const void*)v, (const void*)block_idx, (const void*)lin_S,
                          (const void*)lin_z, (const void*)out})
        if (!aligned16(p)) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(workspace)) return VSA_ERR_WORKSPACE;
    if (workspace_bytes < kStatusBytes + lin_image_bytes(g)) return VSA_ERR_WORKSPACE;
    CUtensorMap mq, mk, mv;
    if (!encode_grid_map_u8(&mq, q8, g) || !encode_grid_map_u8(&mk, k8, g) || !encode_grid_map(&mv, v, g))
        return VSA_ERR_CUDA;
    vsa::FineArgs a;
    a.g = g;
    a.q = q;                   // bf16 q: the linear branch's phi(q)
    a.mq = &mq;
    a.mk = &mk;
    a.mv = &mv;
    a.block_idx = block_idx;
    a.topk = topk;
    a.out = out;
    a.out32 = nullptr;
    a.lse = nullptr;
    a.q_scale = q_scale;
    a.k_scale = k_scale;
    a.status = static_cast<int*>(workspace);
    // the bf16 hi/lo operand image of (S, z) goes into the workspace scratch
    a.lin_image = static_cast<uint8_t*>(workspace) + kStatusBytes;
    cudaError_t e = vsa::launch_linear_pack(g, lin_S, lin_z, const_cast<void*>(a.lin_image),
                                            (cudaStream_t)stream);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(vsa::launch_fine(a, (cudaStream_t)stream));
}

vsa_status vsa_device_status(void* workspace, vsa_stream_t stream) {
    if (!aligned16(workspace)) return VSA_ERR_INVALID_ARGUMENT;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return VSA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return VSA_ERR_CUDA;
    if (word != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return VSA_ERR_CUDA;
    if (word & vsa::kStatusTimeout) return VSA_ERR_TIMEOUT;
    if (word & (vsa::kStatusBadIndex | vsa::kStatusMisaligned | vsa::kStatusNonFinite | vsa::kStatusBadCoord))
        return VSA_ERR_DEVICE_CHECK;
    return VSA_OK;
}

#pragma GCC visibility pop
}  // extern "C"
