// select.cu -- block selection for block-sparse video attention on sm_100a.
//
// Source of the operation: "FastVideo 稀疏蒸馏技术深度解析" (omica.com.cn),
// section "2. 视频稀疏注意力VSA": attention blocks are chosen dynamically per
// query block, keeping 10-20 % of them.  The selection rule (mean-pooled cube
// scores Qp[i].Kp[j]/sqrt(d), top-k per query cube, ties to the lower cube id,
// indices emitted ascending) is this library's reading of that outline.
//
// One persistent kernel, select_kernel, does the whole selection.  Its CTAs
// claim work items from an atomic counter, per group of 8 heads (more per
// group beyond 504 heads, so that at most 63 groups need counters):
//   pool items   one per (cubes j0 .. j0 + cpi - 1, batch, q|k) of the group:
//                16-byte vector loads of the cubes' valid token rows (the
//                group's heads, contiguous within a token row), fp64 sums,
//                divide by the valid count; the mean is stored as an fp32
//                pair hi + lo (hi = RN(mean), lo = RN(mean - hi), together
//                within 2^-48 of the fp64 mean) -> pooled [2][2][B][heads][nt][d].
//   score items  one per (b, head, block of 16 query cubes): the coarse
//                scores of the 16 rows against all nt key cubes,
//                C = Qp Kp^T / sqrt(d), in fp32 (packed fp32x2 FMA, the 16
//                rows' Qp in shared memory, four key cubes per lane read
//                from a feature-major copy of Kp, the features split over
//                two warps) into shared memory -- the nt x nt
//                score matrix never reaches HBM -- then per row (one warp)
//                the exact top-k:
//                  1. a bracket [lo, hi] around the k-th largest fp32 score
//                     (two levels of 256 value bins, about 1/65536 of the
//                     row's range wide);
//                  2. every score above hi + 2 eps is kept, every score
//                     below lo - 2 eps dropped, where eps bounds the fp32
//                     error of a score (forward error of a d-term fp32 dot
//                     product: (d + 8) 2^-24 |Qp_i| max_j |Kp_j| / sqrt(d),
//                     doubled);
//                  3. the few scores in between are recomputed in fp64 from
//                     hi + lo and ranked (larger first, then lower cube id)
//                     for the remaining places (more than 64 of them, e.g.
//                     exact ties: fp64 keys for the whole row and a 64-bit
//                     radix select);
//                  4. a ballot sweep in ascending j writes the kept cubes.
//                Since every fp32 score is within eps of its fp64 value, the
//                kept set is the one the fp64 scores give, up to the rounding
//                of the fp64 dot products themselves.
// Claim order P_0, P_1, S_0, P_2, S_1, ... (pool and score items of head
// group g): the pooling of the next group (HBM bound) runs while the current
// group is scored (compute bound).  A score item waits for its group's pool
// items with a bounded spin on the group's counter; items are claimed in
// order, so every pool item it needs is held by a running CTA that never
// waits, and the wait ends without any assumption about which CTAs are
// resident.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "select.h"
#include "sm100.cuh"

namespace vsa {

constexpr int kSelThreads = 256;                 // 8 warps
constexpr int kSelRows = 16;                     // query cubes per score item
constexpr int kSelMaxCand = 64;                  // fp64-refined candidates per row (fast path)
constexpr int kSelMaxCtas = 1024;                // grid bound (fallback scratch rows)

// ------------------------------------------------------------------ pooling

__device__ __forceinline__ void add_bf16x8(double (&acc)[8], const uint4 raw) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] += (double)__uint_as_float(w[e] << 16);
        acc[2 * e + 1] += (double)__uint_as_float(w[e] & 0xffff0000u);
    }
}

// Means of cubes j0 .. j0 + cpi - 1 (those < nt) of batch b of q (which = 0)
// or k (which = 1), heads h0 .. h0 + nh - 1, written as fp32 hi + lo into
// pooled[which][0|1][b][head][j][d], and for k the hi part once more
// feature-major into kt[b][head][d][ntp] (the coarse scores' loads).  Thread t takes (cube, 16-byte vector)
// pairs t, t + 256, ...
__device__ void pool_item(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const Grid& g,
                          const int j0, const int cpi, const int b, const int which, const int h0, const int nh,
                          float* __restrict__ pooled, float* __restrict__ kt, const int ntp) {
    const uint16_t* x = which ? k : q;
    const int row_elems = g.heads * g.d;              // one token: all heads
    const int nvec = nh * g.d / 8;                    // per cube: heads h0 .. h0 + nh - 1
    const uint16_t* xg = x + (long long)h0 * g.d;
    const long long plane = (long long)g.B * g.heads * g.nt * g.d;
    float* hi = pooled + (2ll * which) * plane + (long long)b * g.heads * g.nt * g.d;
    float* lo = hi + plane;
    for (int u = threadIdx.x; u < cpi * nvec; u += blockDim.x) {
        const int j = j0 + u / nvec, v = u % nvec;
        if (j >= g.nt) break;
        const int it = j / (g.nh * g.nw), ih = (j / g.nw) % g.nh, iw = j % g.nw;
        const int t0 = it * g.tt, h0c = ih * g.th, w0 = iw * g.tw;
        const int vt = min(g.tt, g.T - t0), vh = min(g.th, g.H - h0c), vw = min(g.tw, g.W - w0);
        const double count = (double)(vt * vh * vw);
        const bool full444 = vt == 4 && vh == 4 && vw == 4 && g.tt == 4 && g.th == 4 && g.tw == 4;
        double acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0;
        if (full444) {
            // all 64 tokens valid: 16 loads in flight per layer
            for (int dt = 0; dt < 4; ++dt) {
                uint4 raw[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const long long n = ((long long)(t0 + dt) * g.H + (h0c + (r >> 2))) * g.W + w0 + (r & 3);
                    raw[r] = __ldg(reinterpret_cast<const uint4*>(xg + ((long long)b * g.N + n) * row_elems) + v);
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) add_bf16x8(acc, raw[r]);
            }
        } else {
            for (int dt = 0; dt < vt; ++dt)
                for (int dh = 0; dh < vh; ++dh) {
                    const long long n0 = ((long long)(t0 + dt) * g.H + (h0c + dh)) * g.W + w0;
                    const uint4* src = reinterpret_cast<const uint4*>(xg + ((long long)b * g.N + n0) * row_elems) + v;
                    for (int dw = 0; dw < vw; ++dw) add_bf16x8(acc, __ldg(src + (long long)dw * (row_elems / 8)));
                }
        }
        const int e0 = v * 8, head = h0 + e0 / g.d, c0 = e0 % g.d;
        const long long off = ((long long)head * g.nt + j) * g.d + c0;
        float h8[8], l8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double m = acc[e] / count;
            h8[e] = (float)m;
            l8[e] = (float)(m - (double)h8[e]);
        }
        reinterpret_cast<float4*>(hi + off)[0] = make_float4(h8[0], h8[1], h8[2], h8[3]);
        reinterpret_cast<float4*>(hi + off)[1] = make_float4(h8[4], h8[5], h8[6], h8[7]);
        reinterpret_cast<float4*>(lo + off)[0] = make_float4(l8[0], l8[1], l8[2], l8[3]);
        reinterpret_cast<float4*>(lo + off)[1] = make_float4(l8[4], l8[5], l8[6], l8[7]);
        if (which) {                                  // k hi once more, feature-major
            float* t = kt + (((long long)b * g.heads + head) * g.d + c0) * ntp + j;
#pragma unroll
            for (int e = 0; e < 8; ++e) t[(long long)e * ntp] = h8[e];
        }
    }
}

// -------------------------------------------------------------------- top-k

__device__ __forceinline__ unsigned long long ordered_key(double x) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Top-k of one row of nt order-preserving 64-bit keys, by one warp (hist:
// 256 shared-memory bins of this warp's own): MSD radix select of the k-th
// largest key, then the kept indices in ascending order (equal keys lowest j
// first) written to out[0..k).
__device__ __noinline__ void warp_topk(const unsigned long long* __restrict__ keys, const int nt, const int k,
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


// In a warp's 256-bin histogram (counts in descending bin order = descending
// values), the bin holding the remaining-th largest value: its index and the
// count of all higher bins.
__device__ __forceinline__ void warp_hist_pick(const unsigned int* __restrict__ hist, const int remaining,
                                               const int lane, int& bin, int& above) {
    int cnt[8], lsum = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) { cnt[e] = (int)hist[255 - 8 * lane - e]; lsum += cnt[e]; }
    int incl = lsum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const unsigned ball = __ballot_sync(0xffffffffu, incl >= remaining);
    const int owner = ball ? __ffs(ball) - 1 : 31;
    int b = 0, a = 0;
    if (lane == owner) {
        int run = incl - lsum;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (run + cnt[e] >= remaining) { b = 255 - 8 * lane - e; a = run; break; }
            run += cnt[e];
        }
    }
    bin = __shfl_sync(0xffffffffu, b, owner);
    above = __shfl_sync(0xffffffffu, a, owner);
}

// Bin index 0..255 of x in [0, 256]: x rounded to an integer by the fp32
// adder (add 1.5 * 2^23 and read the low mantissa bits), non-decreasing in x,
// on the FMA/ALU pipes rather than a float-to-int conversion.
__device__ __forceinline__ int bin256(float x) {
    const int n = __float_as_int((x - 0.5f) + 12582912.f) - 0x4B400000;
    return min(255, max(0, n));
}

// A bracket [lo, hi] that holds the k-th largest of the nt fp32 values
// row[0..nt) (shared memory), by one warp: two levels of 256 equal-width
// value bins over [min, max] (x = (s - min) * 256 / (max - min), bin
// round(x - 1/2) clamped to 0..255, level 2 the same on 256 (x - t1) within
// bin t1; both non-decreasing in s, so the k-th largest value lies in the
// chosen bins), so the bracket is about (max - min) / 65536 wide: bin t1, t2
// holds x in [t1 + t2 / 256, t1 + (t2 + 1) / 256] up to the rounding of x
// (3.1 ulp relative, at most 3.2 * 2^-24 * (max - min) in s); the bracket is
// widened by 8 * 2^-24 * (|min| + |max| + max - min).
__device__ __noinline__ void warp_bracket(const float* __restrict__ row, const int nt, const int k,
                             unsigned int* __restrict__ hist, const int lane, double& lo, double& hi) {
    float mn = INFINITY, mx = -INFINITY;
    for (int j0 = 0; j0 < nt; j0 += 128) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + 32 * u + lane;
            if (j < nt) { const float v = row[j]; mn = fminf(mn, v); mx = fmaxf(mx, v); }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if (!(mx - mn > 1e-30f)) { lo = mn; hi = mx; return; }      // (nearly) one value
    const float sc1 = 256.f / (mx - mn);
    // level 1
    for (int h = lane; h < 256; h += 32) hist[h] = 0;
    __syncwarp();
    for (int j0 = 0; j0 < nt; j0 += 128) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + 32 * u + lane;
            if (j < nt) atomicAdd(&hist[bin256((row[j] - mn) * sc1)], 1u);
        }
    }
    __syncwarp();
    int t1, above1;
    warp_hist_pick(hist, k, lane, t1, above1);
    __syncwarp();
    // level 2: the values in bin t1
    for (int h = lane; h < 256; h += 32) hist[h] = 0;
    __syncwarp();
    for (int j0 = 0; j0 < nt; j0 += 128) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + 32 * u + lane;
            if (j < nt) {
                const float x = (row[j] - mn) * sc1;
                if (bin256(x) == t1) atomicAdd(&hist[bin256((x - (float)t1) * 256.f)], 1u);
            }
        }
    }
    __syncwarp();
    int t2, above2;
    warp_hist_pick(hist, k - above1, lane, t2, above2);
    __syncwarp();
    const double w1 = ((double)mx - (double)mn) / 256.0;
    const double margin = 8.0 * 0x1p-24 * (fabs((double)mn) + fabs((double)mx) + ((double)mx - (double)mn));
    lo = (double)mn + ((double)t1 + t2 / 256.0) * w1 - margin;
    hi = (double)mn + ((double)t1 + (t2 + 1) / 256.0) * w1 + margin;
}

// fp64 coarse scores against one query cube row, by one warp: lane l holds
// features fpl*l .. fpl*l + fpl - 1 (fpl = d / 32) of the row as fp64
// (hi + lo); score(j) sums its lane's products in feature order and the 32
// lane partials in a butterfly; the same value on every lane.
struct RowF64 {
    double q[4];
    int fpl;
    __device__ void load(const float* __restrict__ qh, const float* __restrict__ ql, int d, int lane) {
        fpl = d / 32;
        const int c = lane * fpl;
        if (fpl == 4) {
            const float4 h = __ldcg(reinterpret_cast<const float4*>(qh + c)), l = __ldcg(reinterpret_cast<const float4*>(ql + c));
            q[0] = (double)h.x + l.x; q[1] = (double)h.y + l.y; q[2] = (double)h.z + l.z; q[3] = (double)h.w + l.w;
        } else {
            const float2 h = __ldcg(reinterpret_cast<const float2*>(qh + c)), l = __ldcg(reinterpret_cast<const float2*>(ql + c));
            q[0] = (double)h.x + l.x; q[1] = (double)h.y + l.y; q[2] = q[3] = 0.0;
        }
    }
    // this lane's partial of key cube row (kh, kl)
    __device__ double partial(const float* __restrict__ kh, const float* __restrict__ kl, int lane) const {
        const int c = lane * fpl;
        if (fpl == 4) {
            const float4 h = __ldcg(reinterpret_cast<const float4*>(kh + c)), l = __ldcg(reinterpret_cast<const float4*>(kl + c));
            double s = q[0] * ((double)h.x + l.x);
            s = fma(q[1], (double)h.y + l.y, s);
            s = fma(q[2], (double)h.z + l.z, s);
            return fma(q[3], (double)h.w + l.w, s);
        }
        const float2 h = __ldcg(reinterpret_cast<const float2*>(kh + c)), l = __ldcg(reinterpret_cast<const float2*>(kl + c));
        return fma(q[1], (double)h.y + l.y, q[0] * ((double)h.x + l.x));
    }
};

__device__ __forceinline__ double warp_sum_f64(double s) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

__device__ __forceinline__ unsigned long long f64_key(double x) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(x);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

struct SelShared {
    int item;
    int ready;                  // the current item's pooling is done (1) or timed out (-1)
    int lock;                   // fallback scratch row of this CTA
    float kmax2[2];             // max_j of |Kp_j|^2 over each half of the features
};

// Dynamic shared memory of a score item: SelShared, Qp^T [d][16] fp32, the
// scores [16][ntp] fp32, per warp 256 histogram bins and kSelMaxCand
// candidates (cube id + fp64 score).
__host__ __device__ inline int sel_ntp(int nt) { return (nt + 3) & ~3; }
__host__ __device__ inline size_t sel_smem_bytes(int nt, int d) {
    return 128 + (size_t)d * kSelRows * 4 + (size_t)kSelRows * sel_ntp(nt) * 4 +
           (kSelThreads / 32) * (256 * 4 + kSelMaxCand * 12);
}

__device__ void score_item(const Grid& g, const int topk, const int item, const float* __restrict__ pooled,
                           const float* __restrict__ kt,
                           unsigned long long* __restrict__ fallback, int32_t* __restrict__ idx,
                           uint8_t* smem, int* status) {
    SelShared* sh = reinterpret_cast<SelShared*>(smem);
    const int d = g.d, nt = g.nt, ntp = sel_ntp(nt);
    float* sQ = reinterpret_cast<float*>(smem + 128);                   // [d][16]
    float* sc = sQ + d * kSelRows;                                       // [16][ntp]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kWarps = kSelThreads / 32;
    unsigned int* hist_all = reinterpret_cast<unsigned int*>(sc + kSelRows * ntp);   // [8][256]
    double* cs_all = reinterpret_cast<double*>(hist_all + kWarps * 256);            // [8][64]
    int* ci_all = reinterpret_cast<int*>(cs_all + kWarps * kSelMaxCand);            // [8][64]
    unsigned int* hist = hist_all + warp * 256;
    double* cs = cs_all + warp * kSelMaxCand;
    int* ci = ci_all + warp * kSelMaxCand;
    const int rblocks = ceil_div_i(nt, kSelRows);
    const int bh = item / rblocks, i0 = (item % rblocks) * kSelRows;
    const long long plane = (long long)g.B * g.heads * nt * d;
    const float* Qh = pooled + (long long)bh * nt * d;                   // q hi
    const float* Ql = Qh + plane;                                        // q lo
    const float* Kh = pooled + 2 * plane + (long long)bh * nt * d;       // k hi
    const float* Kl = Kh + plane;                                        // k lo
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    const float inv_sqrt_d_f = (float)inv_sqrt_d;

    // Qp hi of the 16 rows, transposed (rows past nt are zero)
    for (int e = tid; e < kSelRows * d; e += kSelThreads) {
        const int r = e / d, c = e % d;
        sQ[c * kSelRows + r] = i0 + r < nt ? __ldcg(Qh + (long long)(i0 + r) * d + c) : 0.f;
    }
    if (tid == 0) sh->kmax2[0] = sh->kmax2[1] = 0.f;
    __syncthreads();

    // ---- coarse scores, fp32: each lane four consecutive key cubes and all
    // 16 rows (acc[b][p] holds rows 2p, 2p+1 of key b; one packed fp32x2 FMA
    // per row pair); warps w and w + 4 take the two halves of the features of
    // the same 128 keys, each half summed in feature order, and the two
    // partial sums meet in shared memory (C = (half 0 + half 1) / sqrt(d)).
    // The keys come from the feature-major copy kt: one 16-byte load per lane
    // and feature, 512 contiguous bytes per warp, PF features in flight.
    const int half = warp >> 2, kw = warp & 3, dh = d / 2, c0 = half * dh;
    const int passes = ceil_div_i(nt, 512);
    const float* Kt = kt + (long long)bh * d * ntp;
    float kmax2 = 0.f;                                    // max_j of this half's |Kp_j|^2
    for (int ps = 0; ps < passes; ++ps) {
        const int j0 = ps * 512 + kw * 128 + 4 * lane;
        const bool live = j0 < ntp;                       // ntp and j0 multiples of 4
        const float* kp = Kt + (long long)c0 * ntp + (live ? j0 : 0);
        uint64_t acc[4][kSelRows / 2];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int p = 0; p < kSelRows / 2; ++p) acc[b][p] = 0ull;
        float nrm[4] = {0.f, 0.f, 0.f, 0.f};
        constexpr int PF = 2;
        float4 ring[PF];
#pragma unroll
        for (int e = 0; e < PF; ++e)
            ring[e] = live ? __ldcg(reinterpret_cast<const float4*>(kp + (long long)e * ntp)) : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = 0; c < dh; c += PF) {
#pragma unroll
            for (int e = 0; e < PF; ++e) {
                const float4 kv4 = ring[e];
                const int cn = c + e + PF;
                ring[e] = live && cn < dh ? __ldcg(reinterpret_cast<const float4*>(kp + (long long)cn * ntp))
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                const float kv[4] = {kv4.x, kv4.y, kv4.z, kv4.w};
                uint64_t kd[4];
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    nrm[b] = fmaf(kv[b], kv[b], nrm[b]);
                    kd[b] = f32x2(kv[b], kv[b]);
                }
                const float4* qq = reinterpret_cast<const float4*>(sQ + (c0 + c + e) * kSelRows);
#pragma unroll
                for (int p4 = 0; p4 < kSelRows / 4; ++p4) {
                    const float4 q4 = qq[p4];
                    const uint64_t qlo = f32x2(q4.x, q4.y), qhi = f32x2(q4.z, q4.w);
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        acc[b][2 * p4] = fma_f32x2(qlo, kd[b], acc[b][2 * p4]);
                        acc[b][2 * p4 + 1] = fma_f32x2(qhi, kd[b], acc[b][2 * p4 + 1]);
                    }
                }
            }
        }
#pragma unroll
        for (int b = 0; b < 4; ++b)
            if (j0 + b < nt) kmax2 = fmaxf(kmax2, nrm[b]);
        if (half == 0) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                if (j0 + b >= nt) continue;
#pragma unroll
                for (int p = 0; p < kSelRows / 2; ++p) {
                    float r0, r1;
                    unf32x2(acc[b][p], r0, r1);
                    sc[(2 * p) * ntp + j0 + b] = r0;
                    sc[(2 * p + 1) * ntp + j0 + b] = r1;
                }
            }
        }
        __syncthreads();
        if (half == 1) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                if (j0 + b >= nt) continue;
#pragma unroll
                for (int p = 0; p < kSelRows / 2; ++p) {
                    float r0, r1;
                    unf32x2(acc[b][p], r0, r1);
                    float* c0p = sc + (2 * p) * ntp + j0 + b;
                    float* c1p = sc + (2 * p + 1) * ntp + j0 + b;
                    *c0p = (*c0p + r0) * inv_sqrt_d_f;
                    *c1p = (*c1p + r1) * inv_sqrt_d_f;
                }
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kmax2 = fmaxf(kmax2, __shfl_xor_sync(0xffffffffu, kmax2, off));
    if (lane == 0) atomicMax(reinterpret_cast<int*>(&sh->kmax2[half]), __float_as_int(kmax2));   // >= 0: int order
    __syncthreads();

    // ---- per row (one warp each): exact top-k
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int r = warp; r < kSelRows; r += kSelThreads / 32) {
        const int i = i0 + r;
        if (i >= nt) break;
        float* row = sc + r * ntp;
        int32_t* out = idx + ((long long)bh * nt + i) * topk;
        if (topk == nt) {                                   // every cube kept
            for (int j = lane; j < nt; j += 32) out[j] = j;
            continue;
        }
        float qn2 = 0.f;
        for (int c = lane; c < d; c += 32) qn2 = fmaf(sQ[c * kSelRows + r], sQ[c * kSelRows + r], qn2);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) qn2 += __shfl_xor_sync(0xffffffffu, qn2, off);
        // bound on |fp32 score - fp64 score|, doubled, plus an absolute term
        // for products in the subnormal range
        // (max_j |Kp_j|^2 <= the sum of the two halves' maxima)
        const double eps = 2.0 * (d + 8) * 0x1p-24 *
                           sqrt((double)qn2 * ((double)sh->kmax2[0] + (double)sh->kmax2[1])) * 1.0001 * inv_sqrt_d + 1e-30;
        double blo, bhi;
        warp_bracket(row, nt, topk, hist, lane, blo, bhi);
        // every score above hi is kept, every score below lo dropped: fp32
        // thresholds rounded outward from the bracket widened by 2 eps
        const float hi = __double2float_ru(bhi + 2.0 * eps), lo = __double2float_rd(blo - 2.0 * eps);
        int above = 0, nc = 0;
        for (int j0 = 0; j0 < nt; j0 += 32) {
            const int j = j0 + lane;
            const float v = j < nt ? row[j] : -INFINITY;
            const bool gt = v > hi, band = j < nt && !gt && v >= lo;
            above += __popc(__ballot_sync(0xffffffffu, gt));
            const unsigned bb = __ballot_sync(0xffffffffu, band);
            const int pos = nc + __popc(bb & lt_mask);
            if (band && pos < kSelMaxCand) ci[pos] = j;
            nc += __popc(bb);
        }
        const int need = topk - above;                      // 1 <= need <= nc
        RowF64 qrow;
        qrow.load(Qh + (long long)i * d, Ql + (long long)i * d, d, lane);
        if (nc <= kSelMaxCand) {
            __syncwarp();
            for (int c = 0; c < nc; c += 2) {               // two candidates' loads in flight
                const int ja = ci[c], jb = c + 1 < nc ? ci[c + 1] : ja;
                const double pa = qrow.partial(Kh + (long long)ja * d, Kl + (long long)ja * d, lane);
                const double pb = qrow.partial(Kh + (long long)jb * d, Kl + (long long)jb * d, lane);
                const double sa = warp_sum_f64(pa) * inv_sqrt_d, sb = warp_sum_f64(pb) * inv_sqrt_d;
                if (lane == 0) { cs[c] = sa; if (c + 1 < nc) cs[c + 1] = sb; }
            }
            __syncwarp();
            for (int c = lane; c < nc; c += 32) {
                const double s = cs[c];
                const int j = ci[c];
                int rank = 0;
                for (int o = 0; o < nc; ++o) rank += (cs[o] > s || (cs[o] == s && ci[o] < j)) ? 1 : 0;
                row[j] = rank < need ? INFINITY : -INFINITY;
            }
            __syncwarp();
            int base = 0;
            for (int j0 = 0; j0 < nt; j0 += 32) {
                const int j = j0 + lane;
                const bool take = j < nt && row[j] > hi;
                const unsigned tb = __ballot_sync(0xffffffffu, take);
                const int pos = base + __popc(tb & lt_mask);
                if (take && pos < topk) out[pos] = j;       // exactly topk are taken for finite scores
                base += __popc(tb);
            }
        } else {
            // Many scores within the error band (ties, or many nearly equal
            // cubes): fp64 keys for the whole row in this CTA's global
            // scratch row, then the 64-bit radix select.  One warp of the
            // CTA at a time owns the scratch row; the owner waits on nothing.
            bool got = false;
            const unsigned long long t0 = clock64();
            while (true) {
                int v = 0;
                if (lane == 0) v = atomicCAS(&sh->lock, 0, 1) == 0;
                got = __shfl_sync(0xffffffffu, v, 0);
                if (got || clock64() - t0 > VSA_WAIT_LIMIT_CYCLES) break;
                __nanosleep(256);
            }
            if (!got) { if (lane == 0) report(status, kStatusTimeout); continue; }
            unsigned long long* keys = fallback + (long long)blockIdx.x * nt;
            // the query row in fp64 in this warp's histogram bins (d <= 128
            // doubles = 1 KB; the radix select below reuses them afterwards),
            // then each lane the fp64 score of its own band cube, 32 at a time
            double* qs = reinterpret_cast<double*>(hist);
            const float* qh = Qh + (long long)i * d;
            const float* ql = Ql + (long long)i * d;
            for (int c = lane; c < d; c += 32) qs[c] = (double)__ldcg(qh + c) + (double)__ldcg(ql + c);
            __syncwarp();
            for (int j0 = 0; j0 < nt; j0 += 32) {
                const int j = j0 + lane;
                const float v = j < nt ? row[j] : -INFINITY;
                const bool gt = v > hi, band = j < nt && !gt && v >= lo;
                unsigned long long key = gt ? ~0ull : 0ull;
                if (band) {
                    const float4* kh4 = reinterpret_cast<const float4*>(Kh + (long long)j * d);
                    const float4* kl4 = reinterpret_cast<const float4*>(Kl + (long long)j * d);
                    double sacc = 0.0;
                    for (int c4 = 0; c4 < d / 4; ++c4) {
                        const float4 h = __ldcg(kh4 + c4), l = __ldcg(kl4 + c4);
                        sacc = fma(qs[4 * c4], (double)h.x + l.x, sacc);
                        sacc = fma(qs[4 * c4 + 1], (double)h.y + l.y, sacc);
                        sacc = fma(qs[4 * c4 + 2], (double)h.z + l.z, sacc);
                        sacc = fma(qs[4 * c4 + 3], (double)h.w + l.w, sacc);
                    }
                    key = f64_key(sacc * inv_sqrt_d);
                }
                if (j < nt) keys[j] = key;
            }
            __syncwarp();
            warp_topk(keys, nt, topk, hist, out, lane);
            __syncwarp();
            __threadfence_block();
            if (lane == 0) atomicExch(&sh->lock, 0);
        }
    }
}

// Work items in claim order, for G head groups of hg heads (the last group
// may be smaller): P_0, P_1, S_0, P_2, S_1, ..., P_{G-1}, S_{G-2}, S_{G-1},
// where P_g are the 2 * B * ceil(nt / cpi) pool items of group g (cpi cubes,
// batch, q|k) and
// S_g its score items (b, head, block of 16 query cubes).  The pooling of
// group g + 1 (HBM bound) is under way while group g is scored (compute
// bound); a score item of group g needs exactly the pool items of P_g, all
// of which come earlier in the order.
struct SelItem {
    int kind;                   // 0 pool, 1 score, -1 none
    int group, local;
};

__device__ __forceinline__ SelItem decode_item(int item, const Grid& g, const int hg, const int ngroups,
                                               const int n_pool) {
    const int rb = ceil_div_i(g.nt, kSelRows);
    if (item < n_pool) return {0, 0, item};
    item -= n_pool;
    for (int grp = 0; grp < ngroups; ++grp) {
        if (grp + 1 < ngroups) {
            if (item < n_pool) return {0, grp + 1, item};
            item -= n_pool;
        }
        const int nh = min(hg, g.heads - grp * hg);
        const int n_score = g.B * nh * rb;
        if (item < n_score) return {1, grp, item};
        item -= n_score;
    }
    return {-1, 0, 0};
}

__global__ void __launch_bounds__(kSelThreads, 2)
select_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const Grid g, const int topk,
              const int hg, const int ngroups, const int cpi, float* __restrict__ pooled, float* __restrict__ kt,
              unsigned long long* __restrict__ fallback, unsigned int* __restrict__ ctr,
              int32_t* __restrict__ idx, int* status) {
    extern __shared__ __align__(16) uint8_t sel_smem[];
    SelShared* sh = reinterpret_cast<SelShared*>(sel_smem);
    const int cubes_per_b = ceil_div_i(g.nt, cpi);
    const unsigned n_pool = 2u * g.B * cubes_per_b;     // pool items per group
    const int rb = ceil_div_i(g.nt, kSelRows);
    if (threadIdx.x == 0) sh->lock = 0;
    for (;;) {
        __syncthreads();                                   // the previous item is done with smem
        if (threadIdx.x == 0) sh->item = (int)atomicAdd(&ctr[0], 1u);
        __syncthreads();
        const SelItem it = decode_item(sh->item, g, hg, ngroups, (int)n_pool);
        if (it.kind < 0) break;
        const int h0 = it.group * hg, nh = min(hg, g.heads - h0);
        if (it.kind == 0) {
            const int jb = it.local % cubes_per_b, b = (it.local / cubes_per_b) % g.B;
            const int which = it.local / (cubes_per_b * g.B);
            pool_item(q, k, g, jb * cpi, cpi, b, which, h0, nh, pooled, kt, sel_ntp(g.nt));
            __syncthreads();
            if (threadIdx.x == 0) {
                __threadfence();                           // the item's means, then the count
                atomicAdd(&ctr[1 + it.group], 1u);
            }
            continue;
        }
        if (threadIdx.x == 0) {                            // the group's pooling, bounded wait
            const unsigned long long t0 = clock64();
            unsigned int done = 0;
            while (true) {
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(done) : "l"(ctr + 1 + it.group) : "memory");
                if (done >= n_pool || clock64() - t0 > VSA_WAIT_LIMIT_CYCLES) break;
                __nanosleep(200);
            }
            __threadfence();
            sh->ready = done >= n_pool ? 1 : -1;
            if (sh->ready < 0) report(status, kStatusTimeout);
        }
        __syncthreads();
        if (sh->ready < 0) break;
        // local = (b * nh + head in group) * rb + row block
        const int bl = it.local / rb, rbi = it.local % rb;
        const int b = bl / nh, head = h0 + bl % nh;
        score_item(g, topk, (b * g.heads + head) * rb + rbi, pooled, kt, fallback, idx, sel_smem, status);
    }
}

// ------------------------------------------------------------------ launchers

// Scratch: 256 bytes of counters, the pooled means as fp32 hi + lo
// (2 * 2 * B * heads * nt * d * 4 bytes), the feature-major copy of the k hi
// means (B * heads * d * ntp * 4 bytes, ntp = nt rounded up to 4) and one
// fallback row of nt 64-bit keys per CTA.
// The 16 score rows of a work item must fit one CTA's shared memory, and the
// work items (claimed through a 32-bit counter) must number fewer than 2^30.
bool select_supported(const Grid& g) {
    const long long items = 2ll * g.B * g.nt * ceil_div_i(g.heads, 8) + (long long)g.B * g.heads * ceil_div_i(g.nt, kSelRows);
    return sel_smem_bytes(g.nt, g.d) <= 232448 && items < (1ll << 30);
}

size_t select_scratch_bytes(const Grid& g) {
    const size_t pooled = 4ull * g.B * g.heads * g.nt * g.d * sizeof(float);
    const size_t kt = (size_t)g.B * g.heads * g.d * sel_ntp(g.nt) * sizeof(float);
    const size_t fallback = (size_t)kSelMaxCtas * g.nt * sizeof(unsigned long long);
    return 256 + pooled + kt + fallback;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
    const Grid& g = a.g;
    unsigned int* ctr = reinterpret_cast<unsigned int*>(a.scratch);
    float* pooled = reinterpret_cast<float*>(static_cast<uint8_t*>(a.scratch) + 256);
    float* kt = pooled + 4ull * g.B * g.heads * g.nt * g.d;
    unsigned long long* fallback = reinterpret_cast<unsigned long long*>(kt + (size_t)g.B * g.heads * g.d * sel_ntp(g.nt));
    const size_t smem = sel_smem_bytes(g.nt, g.d);
    if (!select_supported(g)) return cudaErrorInvalidValue;   // refused earlier by the entry points
    static int configured_device = -1, sms = 0;         // per process: once per device
    int dev = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_kernel, kSelThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // head groups of hg heads: at most 63, so that their counters and the
    // claim counter fit the 256-byte counter block
    const int hg = std::max(8, ceil_div_i(g.heads, 63));
    const int ngroups = ceil_div_i(g.heads, hg);
    const int cpi = std::max(1, kSelThreads / (hg * g.d / 8));   // cubes per pool item: ~one vector per thread
    const long long items = 2ll * g.B * ceil_div_i(g.nt, cpi) * ngroups +
                            (long long)g.B * g.heads * ceil_div_i(g.nt, kSelRows);
    const int grid = (int)std::min<long long>(items, std::min(kSelMaxCtas, sms * per_sm));
    e = cudaMemsetAsync(ctr, 0, (1 + ngroups) * sizeof(unsigned int), stream);
    if (e != cudaSuccess) return e;
    select_kernel<<<grid, kSelThreads, smem, stream>>>(a.q, a.k, g, a.topk, hg, ngroups, cpi, pooled, kt, fallback, ctr,
                                                       a.block_idx, a.status);
    return cudaGetLastError();
}

}  // namespace vsa
