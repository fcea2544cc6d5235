// Host build of the quantiser's quotient step (csrc/e4m3_quotient.cuh): for
// random values, bf16 values (whose products with a reciprocal fall near e4m3
// midpoints far more often than random ones), constructed double-rounding
// cases, exact ties, and scales from 2^-100 to 2^20, the e4m3 rounding of the
// returned float32 value must equal the real quotient x / s rounded once to
// e4m3 (nearest, ties to even, saturating).  The reference rounds the float64
// quotient (which lies on an e4m3 midpoint only when the real one does) by
// counting e4m3 steps; the value under test is rounded with integer bit
// arithmetic on its float32 pattern, as the conversion instruction would.
// The fast test e4m3_product_decides must never accept a product whose
// rounding differs from the exact one.
// Prints "ok".
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <random>

#define __host__
#define __device__
#define __forceinline__ inline
#include "e4m3_quotient.cuh"

// nearest e4m3 of a float64 by counting steps of the value's binade
static double ref_e4m3(double y) {
    const double a = std::fabs(y);
    if (a >= 448.0) return std::copysign(448.0, y);
    int e;
    std::frexp(a, &e);
    int E = e - 1;
    if (E < -6) E = -6;
    const double step = std::ldexp(1.0, E - 3);
    const double n = std::nearbyint(a / step);   // ties to even under the default mode
    return std::copysign(n * step, y);
}

// e4m3 rounding of a float32 by its bit pattern (ties to even), saturating
static double bits_e4m3(float q) {
    uint32_t b;
    std::memcpy(&b, &q, 4);
    const uint32_t sign = b & 0x80000000u;
    uint32_t m = b & 0x7FFFFFFFu;
    float a;
    std::memcpy(&a, &m, 4);
    double out;
    if (a >= 448.f) {
        out = 448.0;
    } else if (a >= 0.015625f) {
        const uint32_t lsb = (m >> 20) & 1u;
        m = (m + 0x7FFFFu + lsb) & ~0xFFFFFu;        // keep 3 mantissa bits
        float r;
        std::memcpy(&r, &m, 4);
        out = r > 448.f ? 448.0 : r;
    } else {
        out = std::nearbyint(static_cast<double>(a) * 512.0) / 512.0;
    }
    return sign ? -out : out;
}

int main() {
    std::mt19937_64 rng(12345);
    std::uniform_real_distribution<float> amax_d(1e-3f, 50.f), u(-1.f, 1.f);
    long fixups = 0, checked = 0, decided = 0, random_checked = 0;
    bool random_phase = true;
    auto check = [&](float x, float s) {
        const float inv = 1.f / s;
        const float q = fa::e4m3_quotient(x, s, inv);
        // the four-at-once form agrees element by element
        float xs4[4] = {x, x * 0.5f, -x, x * 3.0f}, q4[4];
        fa::e4m3_quotient4(xs4, s, inv, q4);
        for (int e = 0; e < 4; ++e)
            if (bits_e4m3(q4[e]) != ref_e4m3(static_cast<double>(xs4[e]) / static_cast<double>(s))) {
                std::printf("four-at-once: x=%a s=%a\n", xs4[e], s);
                std::exit(1);
            }
        const double want = ref_e4m3(static_cast<double>(x) / static_cast<double>(s));
        const double got = bits_e4m3(q);
        ++checked;
        if (got != want) {
            std::printf("x=%a s=%a got %.9g want %.9g\n", x, s, got, want);
            std::exit(1);
        }
        // cases where rounding the product x * inv alone would have been wrong
        if (bits_e4m3(x * inv) != want) ++fixups;
        // the fast test never claims such a case
        if (fa::e4m3_product_decides(x * inv) && bits_e4m3(x * inv) != want) {
            std::printf("product test: x=%a s=%a\n", x, s);
            std::exit(1);
        }
        if (random_phase && fa::e4m3_product_decides(x * inv)) ++decided;
    };
    auto bf16 = [](float f) {       // round to nearest bf16, ties to even
        uint32_t b;
        std::memcpy(&b, &f, 4);
        b = (b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u;
        std::memcpy(&f, &b, 4);
        return f;
    };
    // bf16 blocks as the quantiser sees them without the rotation: s from the
    // block's largest magnitude, itself a bf16 value
    std::normal_distribution<float> nd(0.f, 1.f);
    for (int blk = 0; blk < 400; ++blk) {
        float xs[1024], amax = 0.f;
        const float scale = std::ldexp(1.f, blk % 40 - 20);
        for (float& v : xs) {
            v = bf16(nd(rng) * scale);
            amax = std::fmax(amax, std::fabs(v));
        }
        const float s = amax / 448.f;
        for (float v : xs) check(v, s);
    }
    // scales across the exact range
    for (int E = -100; E <= 20; ++E)
        for (int n = 0; n < 2000; ++n) {
            const float s = std::ldexp(1.f + 0.999f * std::fabs(u(rng)), E);
            check(u(rng) * 448.f * s, s);
        }
    for (int n = 0; n < 2000000; ++n) {
        const float amax = amax_d(rng);
        const float s = amax / 448.f;
        check(u(rng) * amax, s);
    }
    random_checked = checked;
    random_phase = false;
    // constructed cases: x = fl(M * s) for an e4m3 midpoint M, so that the
    // float32 quotient often lands exactly on M while x / s does not
    std::uniform_int_distribution<int> mant(0, 7), expo(-9, 8);
    for (int n = 0; n < 2000000; ++n) {
        const float amax = amax_d(rng);
        const float s = amax / 448.f;
        const int E = expo(rng);
        double M;
        if (E < -6) M = (2 * (n % 8) + 1) * std::ldexp(1.0, -10);              // subnormal midpoints
        else M = (1.0 + (mant(rng) + 0.5) / 8.0) * std::ldexp(1.0, E);        // normal midpoints
        const float x = static_cast<float>(M * s) * ((n & 1) ? -1.f : 1.f);
        check(x, s);
        // and its float32 neighbours
        check(std::nextafter(x, 1e30f), s);
        check(std::nextafter(x, -1e30f), s);
    }
    // exact midpoints (power-of-two scales): ties go to the even code
    for (int E = -9; E <= 8; ++E)
        for (int k = 0; k < 8; ++k) {
            const double M = E < -6 ? (2 * k + 1) * std::ldexp(1.0, -10)
                                    : (1.0 + (k + 0.5) / 8.0) * std::ldexp(1.0, E);
            check(static_cast<float>(M * 0.25), 0.25f);
        }
    if (fixups == 0) {
        std::printf("no case needed more than the rounded product x * inv\n");
        return 1;
    }
    // on random values the fast test should decide nearly every case
    if (decided < random_checked * 99 / 100) {
        std::printf("the product test decided only %ld of %ld random cases\n", decided, random_checked);
        return 1;
    }
    std::printf("ok\n");
    return 0;
}
