// common.cuh -- shared definitions of the CUDA library: tile geometry,
// device status word, small math helpers.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace vsa {

// Bits of the device status word (first int of the workspace).
enum : int {
    kStatusTimeout = 1,      // a bounded wait gave up
    kStatusBadIndex = 2,     // a block index outside [0, nt)
    kStatusMisaligned = 4,   // shared memory not aligned as the kernel needs
    kStatusNonFinite = 8,    // debug-check build: a NaN or Inf reached an output
    kStatusBadCoord = 16,    // debug-check build: a TMA box outside the grid
};

// Checks compiled in only with -DVSA_DEBUG_CHECKS (the library's debug-check
// build, libvsa_debug.so): they record a status bit and let the kernel run on,
// never trap.
#ifdef VSA_DEBUG_CHECKS
#define VSA_DEBUG_CHECK(cond, status, bit) \
    do {                                   \
        if (!(cond)) report(status, bit);  \
    } while (0)
#else
#define VSA_DEBUG_CHECK(cond, status, bit) \
    do {                                   \
    } while (0)
#endif

// Geometry of the cube tiling of a T x H x W token grid.
struct Grid {
    int B, heads, d;
    int T, H, W;
    int tt, th, tw;
    int nT, nh, nw, nt;
    long long N;
};

__host__ __device__ inline int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

// Shape rules every entry point shares (0 = valid): 1 an invalid argument,
// 2 an unsupported head_dim or tile volume.  Index arithmetic is 64-bit, but
// grid and tile counts must fit int32.
inline int shape_error(int B, int heads, int d, int T, int H, int W, int tt, int th, int tw) {
    if (B < 1 || heads < 1 || d < 1 || T < 1 || H < 1 || W < 1 || tt < 1 || th < 1 || tw < 1) return 1;
    if (d != 64 && d != 128) return 2;
    if (tt * th * tw != 64) return 2;
    if ((long long)T * H * W > (1ll << 31) || (long long)B * heads > (1ll << 24)) return 1;
    return 0;
}

inline Grid make_grid(int B, int heads, int d, int T, int H, int W, int tt, int th, int tw) {
    Grid g;
    g.B = B; g.heads = heads; g.d = d;
    g.T = T; g.H = H; g.W = W;
    g.tt = tt; g.th = th; g.tw = tw;
    g.nT = ceil_div_i(T, tt); g.nh = ceil_div_i(H, th); g.nw = ceil_div_i(W, tw);
    g.nt = g.nT * g.nh * g.nw;
    g.N = (long long)T * H * W;
    return g;
}

// Cube j -> its first (t, h, w) coordinates and its valid extents.
struct TileCoord {
    int t0, h0, w0;      // origin in the grid
    int vt, vh, vw;      // number of valid layers along each axis
};

__device__ __forceinline__ TileCoord tile_coord(const Grid& g, int j) {
    TileCoord c;
    const int it = j / (g.nh * g.nw);
    const int ih = (j / g.nw) % g.nh;
    const int iw = j % g.nw;
    c.t0 = it * g.tt; c.h0 = ih * g.th; c.w0 = iw * g.tw;
    c.vt = min(g.tt, g.T - c.t0);
    c.vh = min(g.th, g.H - c.h0);
    c.vw = min(g.tw, g.W - c.w0);
    return c;
}

// 64-bit mask of the valid slots of a cube (slot s = (dt*th + dh)*tw + dw):
// a row of vw bits, repeated for the vh valid rows, repeated for the vt
// valid layers.
__device__ __forceinline__ uint64_t valid_slot_mask(const Grid& g, const TileCoord& c) {
    if (c.vt == g.tt && c.vh == g.th && c.vw == g.tw) return ~0ull;
    const uint64_t row = (1ull << c.vw) - 1ull;
    uint64_t layer = 0;
    for (int dh = 0; dh < c.vh; ++dh) layer |= row << (dh * g.tw);
    uint64_t m = 0;
    const int layer_bits = g.th * g.tw;
    for (int dt = 0; dt < c.vt; ++dt) m |= layer << (dt * layer_bits);
    return m;
}

__device__ __forceinline__ void report(int* status, int bits) {
    if (status) atomicOr(status, bits);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Packed fp32x2 helpers (one 64-bit register holds two floats; sm_100a has
// two-wide fp32 add and fma).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void unf32x2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Fire-and-forget vector add of four floats into global memory (16-byte aligned).
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// 2^x on the MUFU unit (hardware approximation, ~2 ulp).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace vsa
