// noalloc.cu -- block selection for callers that cannot allocate device memory.
//
// vsa_select_blocks needs a caller-allocated workspace for its intermediate
// work counters and cube means.  Some callers cannot obtain one: code that
// runs where cudaMalloc is not permitted or not wanted (inside a framework
// callback that forbids allocation, behind a fixed memory budget, or in an
// embedding that has no allocator of its own).  For them this file keeps the
// intermediates in one fixed, file-scope device array and offers
// vsa_select_blocks_noalloc, which allocates nothing.
//
// Properties a caller must know:
//  * The array (VSA_NOALLOC_SELECT_SCRATCH_BYTES) is reserved on every GPU
//    that loads this library, until the process exits.
//  * Shapes whose intermediates do not fit are rejected with
//    VSA_ERR_WORKSPACE before anything is enqueued.
//  * Every call shares the array and it keeps the last call's contents; each
//    call clears the selection kernel's work counters (a memset it enqueues)
//    and writes all the other bytes it later reads.
//    Calls whose work overlaps on the GPU (different streams, or different
//    host threads without ordering) race on the array and may produce wrong
//    indices: order them on one stream.
//  * The first call on a device looks up the array's device address (once per
//    device, with that device current); make that first call before any
//    stream capture begins.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/vsa.h"
#include "common.cuh"
#include "select.h"

namespace {

static __device__ __align__(256) unsigned char g_select_scratch[VSA_NOALLOC_SELECT_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, found through the runtime (no link-time
// dependency on the driver library).
PFN_cuCtxGetCurrent_v4000 ctx_get_fn() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    });
    return fn;
}

// Device address of g_select_scratch on the current device, looked up once
// per device and context.  In host code the symbol itself is only a
// host-side stand-in, never a device address, so the kernels must be given
// this pointer instead.  The context is remembered beside the address: after
// a reset of the device's primary context (cudaDeviceReset) the module is
// loaded again and the array may sit elsewhere, so the lookup is repeated
// (also when this thread has no current context yet: the lookup binds the
// device's primary context to it).
cudaError_t scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_get_fn();
    if (!get_ctx) return cudaErrorInitializationError;
    std::lock_guard<std::mutex> lock(g_mutex);
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
    if (g_scratch_ptr[dev] == nullptr || ctx == nullptr || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess) return e;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorInitializationError;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {
#pragma GCC visibility push(default)

vsa_status vsa_select_blocks_noalloc(const vsa_bf16* q, const vsa_bf16* k, int B, int heads,
                                     int head_dim, int T, int H, int W, int tt, int th, int tw,
                                     int topk, int32_t* block_idx, vsa_stream_t stream) {
    // the same shape rules as every other entry point (common.cuh)
    switch (vsa::shape_error(B, heads, head_dim, T, H, W, tt, th, tw)) {
        case 0: break;
        case 2: return VSA_ERR_UNSUPPORTED;
        default: return VSA_ERR_INVALID_ARGUMENT;
    }
    const vsa::Grid g = vsa::make_grid(B, heads, head_dim, T, H, W, tt, th, tw);
    if (topk < 1 || topk > g.nt) return VSA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(block_idx)) return VSA_ERR_INVALID_ARGUMENT;
    if (!vsa::select_supported(g)) return VSA_ERR_UNSUPPORTED;
    if (vsa::select_scratch_bytes(g) > (size_t)VSA_NOALLOC_SELECT_SCRATCH_BYTES)
        return VSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return VSA_ERR_CUDA;
    vsa::SelectArgs a;
    a.g = g;
    a.q = q;
    a.k = k;
    a.topk = topk;
    a.block_idx = block_idx;
    a.scratch = scratch;
    a.status = nullptr;        // no caller-visible status word (see the header)
    return vsa::launch_select(a, (cudaStream_t)stream) == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

#pragma GCC visibility pop
}  // extern "C"
