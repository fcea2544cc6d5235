// e4m3_quotient.cuh -- the float32 value whose e4m3 conversion (round to
// nearest, ties to even) is the real quotient x / s rounded once to e4m3.
//
// Fast path: the product q1 = x * inv with inv = RN(1 / s) is within two
// float32 steps of x / s (two roundings of relative size 2^-24 each), so when
// q1 lies more than 8 steps from every e4m3 rounding boundary, x / s lies on
// the same side and e4m3(q1) is the answer.  e4m3 midpoints in the normal
// range (|q| >= 2^-6) have four significant bits with the fourth one set, so
// the distance in float32 steps is the low 20 mantissa bits' distance from
// 0x80000.  Values below 2^-6 (the subnormal range, rare for block-scaled
// data) and values near a midpoint take the exact path.
//
// Exact path: the float32 quotient q = RN(x / s) rounds to the same e4m3
// value as x / s unless q itself lies exactly halfway between two e4m3 values
// while x / s does not (double rounding).  Only then the residual
// r = x - q s, which one fused multiply-add computes exactly for a correctly
// rounded quotient (the exact-remainder property of IEEE division), says on
// which side of that midpoint x / s lies, and q moves one float32 step
// towards it.  Below 2^-6 the midpoints are the odd multiples of 2^-10.
// Requires s > 0.
//
// Self-contained (no CUDA headers) so that the host test can build it.
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

namespace fa {

// Out of line: the kernel reaches it rarely, and one copy keeps the unrolled
// quantiser loop small.
#ifdef __CUDA_ARCH__
__device__ __noinline__
#else
inline
#endif
float e4m3_quotient_exact(float x, float s) {
#ifdef __CUDA_ARCH__
    float q = __fdiv_rn(x, s);
#else
    float q = x / s;
#endif
    const float a = fabsf(q);
    bool mid;
    if (a >= 0.015625f) {
        uint32_t bits;
        memcpy(&bits, &a, 4);
        mid = (bits & 0x7FFFFu) == 0u && (bits & 0x80000u) != 0u;
    } else {
        const float t = a * 1024.f;          // exact: a power-of-two scaling, t < 16
        mid = t == floorf(t) && (static_cast<int>(t) & 1) == 1;
    }
    if (mid) {
#ifdef __CUDA_ARCH__
        const float r = __fmaf_rn(-q, s, x);
#else
        const float r = fmaf(-q, s, x);
#endif
        if (r != 0.f) {
            // one float32 step towards x / s: up when r > 0 (s > 0)
            uint32_t qb;
            memcpy(&qb, &q, 4);
            const bool up = r > 0.f;
            const bool neg = (qb >> 31) != 0u;
            qb = (up != neg) ? qb + 1u : qb - 1u;   // the magnitude grows iff moving away from 0
            memcpy(&q, &qb, 4);
        }
    }
    return q;
}

// The fast path's test: q1 at least 2^-6 in magnitude and more than 8
// float32 steps from every e4m3 midpoint.
__host__ __device__ __forceinline__ bool e4m3_product_safe(float q1) {
    uint32_t bits;
    memcpy(&bits, &q1, 4);
    bits &= 0x7FFFFFFFu;
    const int dist = static_cast<int>(bits & 0xFFFFFu) - 0x80000;
    return bits >= 0x3C800000u /* 2^-6 */ && (dist > 8 || dist < -8);
}

// inv must be RN(1 / s).
__host__ __device__ __forceinline__ float e4m3_quotient(float x, float s, float inv) {
#ifdef __CUDA_ARCH__
    const float q1 = __fmul_rn(x, inv);
#else
    const float q1 = x * inv;
#endif
    return e4m3_product_safe(q1) ? q1 : e4m3_quotient_exact(x, s);
}

// Four at once: the products first, and the exact path only when one of them
// needs it (one rarely taken branch per four values).
__host__ __device__ __forceinline__ void e4m3_quotient4(const float (&x)[4], float s, float inv,
                                                       float (&q)[4]) {
    bool all_safe = true;
#ifdef __CUDA_ARCH__
#pragma unroll
#endif
    for (int e = 0; e < 4; ++e) {
#ifdef __CUDA_ARCH__
        q[e] = __fmul_rn(x[e], inv);
#else
        q[e] = x[e] * inv;
#endif
        all_safe = all_safe && e4m3_product_safe(q[e]);
    }
    if (!all_safe) {
#ifdef __CUDA_ARCH__
#pragma unroll
#endif
        for (int e = 0; e < 4; ++e)
            if (!e4m3_product_safe(q[e])) q[e] = e4m3_quotient_exact(x[e], s);
    }
}

}  // namespace fa
