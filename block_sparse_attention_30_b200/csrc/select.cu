// select.cu -- block selection for block-sparse video attention on sm_100a.
//
// Source of the operation: "FastVideo 稀疏蒸馏技术深度解析" (omica.com.cn),
// section "2. 视频稀疏注意力VSA": attention blocks are chosen dynamically per
// query block, keeping 10-20 % of them.  The selection rule (mean-pooled cube
// scores Qp[i].Kp[j]/sqrt(d), top-k per query cube, ties to the lower cube id,
// indices emitted ascending) is this library's reading of that outline.
//
// Three HBM-friendly kernels, all in fp64 so the chosen cubes match an exact
// evaluation except for genuine ties:
//   pool_kernel    one CTA per (cube, batch, q|k): 16-byte vector loads of the
//                  cube's valid token rows (all heads at once), fp64 sums,
//                  divide by the valid count -> pooled [2][B][heads][nt][d].
//   coarse_kernel  per (b, head) a 64x64 tile of C = Qp Kp^T / sqrt(d) with an
//                  8x4 register tile per thread -> scores [B][heads][nt][nt].
//   topk_kernel    one warp per score row: 8-pass MSD radix select on
//                  order-preserving 64-bit keys finds the k-th largest score,
//                  then a ballot sweep in ascending j emits the kept cubes
//                  (equal keys taken lowest j first).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "select.h"

namespace vsa {

// ------------------------------------------------------------------ pooling

__device__ __forceinline__ void add_bf16x8(double (&acc)[8], const uint4 raw) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] += (double)__uint_as_float(w[e] << 16);
        acc[2 * e + 1] += (double)__uint_as_float(w[e] & 0xffff0000u);
    }
}

__global__ void __launch_bounds__(320)
pool_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const Grid g,
            double* __restrict__ pooled) {
    const int j = blockIdx.x, b = blockIdx.y, which = blockIdx.z;
    const uint16_t* x = which ? k : q;
    const int it = j / (g.nh * g.nw), ih = (j / g.nw) % g.nh, iw = j % g.nw;
    const int t0 = it * g.tt, h0 = ih * g.th, w0 = iw * g.tw;
    const int vt = min(g.tt, g.T - t0), vh = min(g.th, g.H - h0), vw = min(g.tw, g.W - w0);
    const double count = (double)(vt * vh * vw);
    const int row_elems = g.heads * g.d;              // one token: all heads
    const int nvec = row_elems / 8;
    const bool full444 = vt == 4 && vh == 4 && vw == 4 && g.tt == 4 && g.th == 4 && g.tw == 4;
    double* out = pooled + ((long long)which * g.B + b) * g.heads * (long long)g.nt * g.d;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        double acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0;
        if (full444) {
            // all 64 tokens valid: 16 loads in flight per layer
            for (int dt = 0; dt < 4; ++dt) {
                uint4 raw[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const long long n = ((long long)(t0 + dt) * g.H + (h0 + (r >> 2))) * g.W + w0 + (r & 3);
                    raw[r] = __ldg(reinterpret_cast<const uint4*>(x + ((long long)b * g.N + n) * row_elems) + v);
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) add_bf16x8(acc, raw[r]);
            }
        } else {
            for (int dt = 0; dt < vt; ++dt)
                for (int dh = 0; dh < vh; ++dh) {
                    const long long n0 = ((long long)(t0 + dt) * g.H + (h0 + dh)) * g.W + w0;
                    const uint4* src = reinterpret_cast<const uint4*>(x + ((long long)b * g.N + n0) * row_elems) + v;
                    for (int dw = 0; dw < vw; ++dw) add_bf16x8(acc, __ldg(src + (long long)dw * nvec));
                }
        }
        const int e0 = v * 8, head = e0 / g.d, c0 = e0 % g.d;
        double* dst = out + ((long long)head * g.nt + j) * g.d + c0;
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[e] = acc[e] / count;
    }
}

// ------------------------------------------------------------ coarse scores
// C[i][j] = (sum_c Qp[i][c] Kp[j][c]) / sqrt(d), per (b, head); 64x64 tiles,
// 128 threads, 8 (rows) x 4 (cols) fp64 outputs per thread, operands staged
// 16 features at a time, read back with 16-byte shared loads.  The features
// are summed in increasing order, as in the exact definition.
__global__ void __launch_bounds__(128)
coarse_kernel(const double* __restrict__ qp, const double* __restrict__ kp, const Grid g,
              const double inv_sqrt_d, double* __restrict__ scores) {
    __shared__ __align__(16) double As[16][64 + 2];
    __shared__ __align__(16) double Bs[16][64 + 2];
    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
    const int nt = g.nt, d = g.d;
    const double* Q = qp + (long long)bh * nt * d;
    const double* K = kp + (long long)bh * nt * d;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;     // 16 column groups x 8 row groups
    double acc[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = 0.0;
    for (int e0 = 0; e0 < d; e0 += 16) {
        for (int l = threadIdx.x; l < 64 * 16; l += 128) {
            const int rr = l / 16, ee = l % 16;
            As[ee][rr] = (i0 + rr < nt) ? Q[(long long)(i0 + rr) * d + e0 + ee] : 0.0;
            Bs[ee][rr] = (j0 + rr < nt) ? K[(long long)(j0 + rr) * d + e0 + ee] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int ee = 0; ee < 16; ++ee) {
            double a[8], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const double2 t2 = *reinterpret_cast<const double2*>(&As[ee][8 * ty + 2 * u]);
                a[2 * u] = t2.x; a[2 * u + 1] = t2.y;
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const double2 t2 = *reinterpret_cast<const double2*>(&Bs[ee][4 * tx + 2 * u]);
                bv[2 * u] = t2.x; bv[2 * u + 1] = t2.y;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc[u][w] = fma(a[u], bv[w], acc[u][w]);
        }
        __syncthreads();
    }
    double* S = scores + (long long)bh * nt * nt;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int ii = i0 + 8 * ty + u;
        if (ii >= nt) continue;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int jj = j0 + 4 * tx + w;
            if (jj < nt) S[(long long)ii * nt + jj] = acc[u][w] * inv_sqrt_d;
        }
    }
}

// -------------------------------------------------------------------- top-k

__device__ __forceinline__ unsigned long long ordered_key(double x) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// One warp per (b, head, i) row; rows_per_cta warps per CTA.
__global__ void __launch_bounds__(256)
topk_kernel(const double* __restrict__ scores, const int nt, const int k, const long long rows,
            int32_t* __restrict__ idx) {
    extern __shared__ unsigned long long tk_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const long long row = (long long)blockIdx.x * nwarps + warp;
    unsigned long long* keys = tk_smem + (long long)warp * nt;
    unsigned int* hist = reinterpret_cast<unsigned int*>(tk_smem + (long long)nwarps * nt) + warp * 256;
    if (row >= rows) return;                          // whole warp leaves together
    const double* src = scores + row * nt;
    for (int j = lane; j < nt; j += 32) keys[j] = ordered_key(src[j]);
    __syncwarp();

    unsigned long long prefix = 0, mask = 0;
    int remaining = k;                                 // how many still to place at/below prefix
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int h = lane; h < 256; h += 32) hist[h] = 0;
        __syncwarp();
        for (int j = lane; j < nt; j += 32) {
            const unsigned long long u = keys[j];
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255], 1u);
        }
        __syncwarp();
        // lane l owns digits 255-8l .. 248-8l (descending); inclusive scan from the top
        int cnt[8], lsum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { cnt[e] = (int)hist[255 - 8 * lane - e]; lsum += cnt[e]; }
        int incl = lsum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const int excl = incl - lsum;
        // the digit holding the remaining-th largest key lies in the first lane
        // whose inclusive count reaches `remaining`
        const unsigned ball = __ballot_sync(0xffffffffu, incl >= remaining);
        const int owner = __ffs(ball) - 1;
        int digit = 0, above = 0;
        if (lane == owner) {
            int run = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (run + cnt[e] >= remaining) { digit = 255 - 8 * lane - e; above = run; break; }
                run += cnt[e];
            }
        }
        digit = __shfl_sync(0xffffffffu, digit, owner);
        above = __shfl_sync(0xffffffffu, above, owner);
        remaining -= above;
        prefix |= (unsigned long long)digit << shift;
        mask |= 255ull << shift;
        __syncwarp();
    }
    // prefix is the k-th largest key; take every larger key and the first
    // `remaining` keys equal to it, sweeping j upward (ascending output).
    int32_t* out = idx + row * k;
    int base = 0, eq_seen = 0;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int j0 = 0; j0 < nt; j0 += 32) {
        const int j = j0 + lane;
        const bool in = j < nt;
        const unsigned long long u = in ? keys[j] : 0ull;
        const bool gt = in && u > prefix;
        const bool eq = in && u == prefix;
        const unsigned eqb = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = eq_seen + __popc(eqb & lt_mask);
        const bool take = gt || (eq && eq_rank < remaining);
        const unsigned tb = __ballot_sync(0xffffffffu, take);
        if (take) out[base + __popc(tb & lt_mask)] = j;
        base += __popc(tb);
        eq_seen += __popc(eqb);
    }
}

// ------------------------------------------------------------------ launchers

size_t select_scratch_bytes(const Grid& g) {
    const size_t pooled = 2ull * g.B * g.heads * g.nt * g.d * sizeof(double);
    const size_t scores = (size_t)g.B * g.heads * g.nt * g.nt * sizeof(double);
    return pooled + scores;
}

static int topk_warps_per_cta(int nt) {
    // shared memory per warp: nt keys (8 B) + 256 histogram bins (4 B)
    const size_t per_warp = (size_t)nt * 8 + 1024;
    int w = 8;
    while (w > 1 && per_warp * w > 96 * 1024) w >>= 1;
    return w;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
    const Grid& g = a.g;
    double* pooled = reinterpret_cast<double*>(a.scratch);
    double* scores = pooled + 2ull * g.B * g.heads * g.nt * g.d;
    pool_kernel<<<dim3(g.nt, g.B, 2), 320, 0, stream>>>(a.q, a.k, g, pooled);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const double* qp = pooled;
    const double* kp = pooled + (size_t)g.B * g.heads * g.nt * g.d;
    const int tiles = ceil_div_i(g.nt, 64);
    coarse_kernel<<<dim3(tiles, tiles, g.B * g.heads), 128, 0, stream>>>(qp, kp, g, 1.0 / sqrt((double)g.d), scores);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int wpc = topk_warps_per_cta(g.nt);
    const size_t smem = (size_t)wpc * ((size_t)g.nt * 8 + 1024);
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const long long rows = (long long)g.B * g.heads * g.nt;
    const unsigned blocks = (unsigned)((rows + wpc - 1) / wpc);
    topk_kernel<<<blocks, 32 * wpc, smem, stream>>>(scores, g.nt, a.topk, rows, a.block_idx);
    return cudaGetLastError();
}

}  // namespace vsa
