// softmax_step.cuh -- one online-softmax step of the fine pass on half a row
// of scores (64 keys), written for instruction economy on sm_100a:
//   3-input max, packed fp32x2 FMA for the exp2 argument, MUFU ex2, bf16x2
//   packing, packed fp32x2 accumulation of the row sum.
//
// The row maximum lives in the exp2 domain (scores times log2(e)/sqrt(d)).
// It is raised only when a new maximum exceeds it by more than 2^8
// ("lazy rescale"); the weights then stay below 256, exact enough in bf16 and
// far from fp32 overflow.  The row sum adds the bf16-ROUNDED weights -- the
// values the tensor core multiplies with V -- so that O / l is an exactly
// normalised average of V rows even when the reference maximum is stale.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace vsa {

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}

struct SoftmaxState {
    float m_run;    // running maximum, exp2 domain (shared by both row halves)
    float l_run;    // this half's running sum of weights
};

// s: this thread's 64 raw scores (q.k); scale_log2: this thread's factor from
// a raw score to the exp2 domain; vmask: valid keys (bit e = key e),
// consulted only when `masked`.  Writes the 32 packed bf16x2 weights to pk
// and returns the factor by which O must be rescaled (1 if unchanged) and
// whether any rescale happened for this row.
template <bool MASKED>
__device__ __forceinline__ float softmax_step(float (&s)[64], uint64_t vmask, float scale_log2,
                                              SoftmaxState& st, bool& rescaled,
                                              uint32_t (&pk)[32]) {
    if (MASKED) {
#pragma unroll
        for (int e = 0; e < 64; ++e)
            if (!((vmask >> e) & 1ull)) s[e] = -INFINITY;
    }
    float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
    for (int e = 4; e + 8 <= 60; e += 8) {       // s[4] .. s[59]
        m0 = max3f(m0, s[e], s[e + 1]);
        m1 = max3f(m1, s[e + 2], s[e + 3]);
        m2 = max3f(m2, s[e + 4], s[e + 5]);
        m3 = max3f(m3, s[e + 6], s[e + 7]);
    }
    m0 = max3f(m0, s[60], s[61]);
    m1 = max3f(m1, s[62], s[63]);
    // each half scales its own maximum (the two halves may hold key cubes
    // with different scales); for a common positive scale this equals scaling
    // the maximum of both, as rounding is monotonic
    float mx = fmaxf(max3f(m0, m1, m2), m3) * scale_log2;
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    rescaled = mx > st.m_run + 8.f;
    const float m_new = rescaled ? mx : st.m_run;
    const float alpha = rescaled ? ex2(st.m_run - m_new) : 1.f;
    st.m_run = m_new;
    const uint64_t sc2 = f32x2(scale_log2, scale_log2);
    const uint64_t nm2 = f32x2(-m_new, -m_new);
    uint64_t acc0 = 0, acc1 = 0;            // two independent packed sums
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        float t0, t1;
        unf32x2(fma_f32x2(f32x2(s[2 * e], s[2 * e + 1]), sc2, nm2), t0, t1);
        const uint32_t w = pack_bf16x2(ex2(t0), ex2(t1));
        pk[e] = w;
        const uint64_t r = f32x2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
        if (e & 1) acc1 = add_f32x2(acc1, r);
        else acc0 = add_f32x2(acc0, r);
    }
    float a0, a1, b0, b1;
    unf32x2(acc0, a0, a1);
    unf32x2(acc1, b0, b1);
    st.l_run = st.l_run * alpha + ((a0 + a1) + (b0 + b1));
    return alpha;
}

}  // namespace vsa
