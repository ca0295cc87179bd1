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
//   coarse_kernel  per (b, head) a 64x64 tile of C = Qp Kp^T / sqrt(d) on the
//                  fp64 tensor cores -> scores [B][heads][nt][nt].
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
// C[i][j] = (sum_c Qp[i][c] Kp[j][c]) / sqrt(d), per (b, head), in fp64 on
// the fp64 tensor cores (mma.sync m8n8k4, exact products, fp64 accumulation;
// tcgen05 has no fp64 kind).  64x64 tiles of C per CTA, 4 warps of 32x32
// (4x4 MMA tiles), operands staged 32 features at a time in shared memory.
// The summation order differs from a sequential dot product only at the fp64
// rounding level, far inside the near-tie tolerance of the selection.
__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

constexpr int kCoarseChunk = 32;                 // features staged per step
constexpr int kCoarseStride = kCoarseChunk + 4;  // doubles per smem row: 8-byte loads of a
                                                 // half-warp (4 rows x 4 features) hit distinct banks

__global__ void __launch_bounds__(128)
coarse_kernel(const double* __restrict__ qp, const double* __restrict__ kp, const Grid g,
              const double inv_sqrt_d, double* __restrict__ scores) {
    __shared__ __align__(16) double As[64 * kCoarseStride];
    __shared__ __align__(16) double Bs[64 * kCoarseStride];
    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
    const int nt = g.nt, d = g.d;
    const double* Q = qp + (long long)bh * nt * d;
    const double* K = kp + (long long)bh * nt * d;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wm = warp >> 1, wn = warp & 1;         // warp tile: rows 32*wm.., cols 32*wn..
    const int gr = lane >> 2, tq = lane & 3;         // MMA fragment coordinates
    double acc[4][4][2];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c][0] = acc[a][c][1] = 0.0;
    for (int e0 = 0; e0 < d; e0 += kCoarseChunk) {
        // 64 rows x 32 features of each operand, 16-byte loads, zero rows past nt
        for (int l = threadIdx.x; l < 64 * kCoarseChunk / 2; l += 128) {
            const int rr = l / (kCoarseChunk / 2), cc = 2 * (l % (kCoarseChunk / 2));
            const double2 qa = i0 + rr < nt ? *reinterpret_cast<const double2*>(Q + (long long)(i0 + rr) * d + e0 + cc)
                                            : make_double2(0.0, 0.0);
            const double2 kb = j0 + rr < nt ? *reinterpret_cast<const double2*>(K + (long long)(j0 + rr) * d + e0 + cc)
                                            : make_double2(0.0, 0.0);
            *reinterpret_cast<double2*>(&As[rr * kCoarseStride + cc]) = qa;
            *reinterpret_cast<double2*>(&Bs[rr * kCoarseStride + cc]) = kb;
        }
        __syncthreads();
#pragma unroll
        for (int ks = 0; ks < kCoarseChunk / 4; ++ks) {
            double a[4], b[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                a[t] = As[(32 * wm + 8 * t + gr) * kCoarseStride + 4 * ks + tq];   // A[row][k]
                b[t] = Bs[(32 * wn + 8 * t + gr) * kCoarseStride + 4 * ks + tq];   // B[k][col] = Kp[col][k]
            }
#pragma unroll
            for (int rt = 0; rt < 4; ++rt)
#pragma unroll
                for (int ct = 0; ct < 4; ++ct) dmma_8x8x4(acc[rt][ct][0], acc[rt][ct][1], a[rt], b[ct]);
        }
        __syncthreads();
    }
    double* S = scores + (long long)bh * nt * nt;
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
        const int ii = i0 + 32 * wm + 8 * rt + gr;
        if (ii >= nt) continue;
#pragma unroll
        for (int ct = 0; ct < 4; ++ct) {
            const int jj = j0 + 32 * wn + 8 * ct + 2 * tq;
            if (jj < nt) S[(long long)ii * nt + jj] = acc[rt][ct][0] * inv_sqrt_d;
            if (jj + 1 < nt) S[(long long)ii * nt + jj + 1] = acc[rt][ct][1] * inv_sqrt_d;
        }
    }
}

// -------------------------------------------------------------------- top-k

__device__ __forceinline__ unsigned long long ordered_key(double x) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Top-k of one row of nt order-preserving keys in shared memory, by one warp
// (hist: 256 bins of this warp's own): MSD radix select of the k-th largest
// key, then the kept indices in ascending order (equal keys lowest j first)
// written to out[0..k).
__device__ void warp_topk(const unsigned long long* __restrict__ keys, const int nt, const int k,
                          unsigned int* __restrict__ hist, int32_t* __restrict__ out, const int lane) {
    // Skip the leading bytes every key shares (for scores of one magnitude
    // the sign and exponent byte): start at the highest byte where the
    // smallest and largest keys differ.
    unsigned long long kmin = ~0ull, kmax = 0ull;
    for (int j = lane; j < nt; j += 32) { kmin = min(kmin, keys[j]); kmax = max(kmax, keys[j]); }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
    }
    const unsigned long long diff = kmin ^ kmax;
    const int top_shift = diff ? ((63 - __clzll(diff)) / 8) * 8 : -8;
    unsigned long long mask = top_shift >= 56 ? 0ull : (~0ull << (top_shift + 8));
    unsigned long long prefix = kmin & mask;        // the common leading bytes
    int remaining = k;                                 // how many still to place at/below prefix
    for (int shift = top_shift; shift >= 0; shift -= 8) {
        for (int h = lane; h < 256; h += 32) hist[h] = 0;
        __syncwarp();
        for (int j0 = 0; j0 < nt; j0 += 32) {
            const int j = j0 + lane;
            const unsigned long long u = j < nt ? keys[j] : 0ull;
            const int bin = (j < nt && (u & mask) == prefix) ? (int)((u >> shift) & 255) : 256;
            // one atomic per distinct bin of the warp (keys cluster in few bins)
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (bin < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (unsigned)__popc(peers));
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
        int digit = 0, above = 0, bucket = 0;
        if (lane == owner) {
            int run = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (run + cnt[e] >= remaining) { digit = 255 - 8 * lane - e; above = run; bucket = cnt[e]; break; }
                run += cnt[e];
            }
        }
        digit = __shfl_sync(0xffffffffu, digit, owner);
        above = __shfl_sync(0xffffffffu, above, owner);
        bucket = __shfl_sync(0xffffffffu, bucket, owner);
        remaining -= above;
        prefix |= (unsigned long long)digit << shift;
        mask |= 255ull << shift;
        __syncwarp();
        if (bucket == remaining) break;                // the whole bucket is kept: done
    }
    // Every key whose masked value exceeds prefix is kept, and of the keys
    // equal to it under the mask the first `remaining` in ascending j (all of
    // them when the loop stopped early; equal full keys go lowest j first).
    int base = 0, eq_seen = 0;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int j0 = 0; j0 < nt; j0 += 32) {
        const int j = j0 + lane;
        const bool in = j < nt;
        const unsigned long long u = in ? (keys[j] & mask) : 0ull;
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

// One warp per (b, head, i) row of the score matrix in global memory;
// rows_per_cta warps per CTA.
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
    warp_topk(keys, nt, k, hist, idx + row * k, lane);
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
