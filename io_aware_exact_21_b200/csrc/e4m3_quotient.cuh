// e4m3_quotient.cuh -- the float32 value whose e4m3 conversion (round to
// nearest, ties to even, saturating at +-448) is the real quotient x / s
// rounded once to e4m3.
//
// The product q1 = x * inv with inv = RN(1 / s) is within two float32 steps
// of x / s, so it names the e4m3 interval [V, V'] that x / s lies in or
// borders.  Which way x / s rounds is decided by its side of that interval's
// midpoint M: the sign of M s - |x|, which one fused multiply-add gives
// exactly (the exact value is rounded once, and rounding keeps its sign and
// whether it is zero).  The returned magnitude is M moved one float32 step
// towards that side, or M itself on an exact tie, so its conversion gives V,
// V' or the even one of the two.  When x / s lies just across V or V' (in a
// neighbouring interval), it is close to that end and far from the
// neighbour's midpoint, and the same rule picks that end, which is correct.
//   normal range, |q1| >= 2^-6: M has q1's exponent and top three mantissa
//     bits followed by a one (e4m3 keeps three mantissa bits);
//   below 2^-6 (e4m3 subnormals, steps of 2^-9): M is the odd multiple of
//     2^-10 inside q1's step.
// Every step is exact arithmetic or one rounding, so no branch depends on how
// close q1 happens to fall to a midpoint.  Requires s > 0; exact while
// M s - |x| stays inside the float32 range (s >= 2^-100 suffices), which any
// block scale of bf16 data above 448 * 2^-100 in magnitude satisfies.
//
// Self-contained (no CUDA headers) so that the host test can build it.
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

namespace fa {

__host__ __device__ __forceinline__ uint32_t e4m3q_bits(float f) {
    uint32_t b;
    memcpy(&b, &f, 4);
    return b;
}

__host__ __device__ __forceinline__ float e4m3q_float(uint32_t b) {
    float f;
    memcpy(&f, &b, 4);
    return f;
}

// The e4m3 midpoint M (as float32 bits) of the interval of |q1| = ab.
__host__ __device__ __forceinline__ uint32_t e4m3q_mid_normal(uint32_t ab) {   // |q1| >= 2^-6
    return (ab & 0xFFF00000u) | 0x80000u;
}
__host__ __device__ __forceinline__ uint32_t e4m3q_mid_small(uint32_t ab) {    // |q1| < 2^-6
    // t * 2^-9 <= |q1| < (t + 1) * 2^-9, t in 0 .. 7; M = (t + 1/2) 2^-9
    const float t = floorf(e4m3q_float(ab) * 512.f);   // exact scaling by 2^9
    return e4m3q_bits((t + 0.5f) * 0.001953125f);      // exact: a 5-bit value times 2^-9
}
__host__ __device__ __forceinline__ uint32_t e4m3q_mid(uint32_t ab) {
    return ab >= 0x3C800000u ? e4m3q_mid_normal(ab) : e4m3q_mid_small(ab);
}

// M moved one float32 step towards x / s (r > 0: x / s below M, r < 0:
// above, r == 0: exactly M), with the sign of x.
__host__ __device__ __forceinline__ float e4m3q_finish(float x, float s, uint32_t sign, uint32_t mb) {
#ifdef __CUDA_ARCH__
    const float r = __fmaf_rn(e4m3q_float(mb), s, -fabsf(x));
#else
    const float r = fmaf(e4m3q_float(mb), s, -fabsf(x));
#endif
    mb = mb + (r < 0.f ? 1u : 0u) - (r > 0.f ? 1u : 0u);
    return e4m3q_float(mb | sign);
}

__host__ __device__ __forceinline__ float e4m3q_product(float x, float inv) {
#ifdef __CUDA_ARCH__
    return __fmul_rn(x, inv);
#else
    return x * inv;
#endif
}

// inv must be RN(1 / s).
__host__ __device__ __forceinline__ float e4m3_quotient(float x, float s, float inv) {
    const uint32_t qb = e4m3q_bits(e4m3q_product(x, inv));
    return e4m3q_finish(x, s, qb & 0x80000000u, e4m3q_mid(qb & 0x7FFFFFFFu));
}

// True when the rounded product q1 = RN(x * inv) alone decides the e4m3
// value: q1 lies in the normal e4m3 range (|q1| >= 2^-6) and more than 8
// float32 steps from the e4m3 midpoint of its interval.  x / s is within two
// float32 steps of q1 (two roundings of relative size 2^-24 each), so it then
// lies on the same side of every midpoint and e4m3(q1) = e4m3(x / s).
// (Normal-range midpoints have the low 20 mantissa bits 0x80000, and never
// sit at a binade boundary.)  A cheap test for data whose products rarely
// fall near a midpoint, so that the exact step runs only when one does.
__host__ __device__ __forceinline__ bool e4m3_product_decides(float q1) {
    const uint32_t b = e4m3q_bits(q1) & 0x7FFFFFFFu;
    return b >= 0x3C800000u && ((b & 0xFFFFFu) - 0x7FFF8u) > 16u;
}

// Four values with one scale (the quantiser's unit of work).
__host__ __device__ __forceinline__ void e4m3_quotient4(const float (&x)[4], float s, float inv,
                                                       float (&q)[4]) {
#ifdef __CUDA_ARCH__
#pragma unroll
#endif
    for (int e = 0; e < 4; ++e) q[e] = e4m3_quotient(x[e], s, inv);
}

}  // namespace fa
