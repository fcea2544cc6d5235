// fp8_quant.cuh -- block quantisation of bf16 Q, K, V to e4m3 for the FP8
// forward (FlashAttention encyclopedia page, FlashAttention-3 paragraph: the
// FP8 path quantises by blocks and adds a step that reduces quantisation
// error).
//
// One CTA per (sequence, head, block of 128 rows), 256 threads: warp w takes
// rows w, w + 8, ..., and lane l holds channels 4l .. 4l + 3 of each (d = 128).
//  * optional rotation (Q and K): multiply by a sign vector, then the
//    orthonormal Walsh-Hadamard transform -- butterflies (a, b) -> (a + b,
//    a - b) on channel pairs (j, j + h) for h = 1, 2, 4, ..., 64 in that
//    order (h = 1, 2 inside a lane, h >= 4 across lanes by shuffles), then a
//    factor 1/sqrt(128).  Every step is an explicitly rounded float32
//    operation, so the codes do not depend on how a compiler would contract
//    them.  q.k is unchanged by the rotation.
//  * scale s = amax / 448 over the block (1 for an all-zero block); codes are
//    e4m3(x / s), the real quotient rounded once to the nearest e4m3 value
//    (ties to even, saturating at +-448): see e4m3_quotient below.
//  * layout: Q and K codes keep the token-major [B, N, H, 128] layout; V codes
//    are written transposed, [B, H, 128, Np] with Np = N rounded up to 16 and
//    zeros past N, so the forward's PV GEMM reads a K-major operand.
#pragma once

#include "e4m3_quotient.cuh"
#include "sm100.cuh"

namespace fa {

struct QuantParams {
    const __nv_bfloat16* x;    // [B, N, H, 128]
    uint8_t* out;              // codes
    float* scales;             // [B, H, nb]
    const float* signs;        // 128 entries of +-1, or nullptr (no rotation)
    int B, N, H, nb, Np;
    int transpose;             // 1: write [B, H, 128, Np]
};

constexpr int kQuantRowPitch = 132;   // shared transpose tile: 128 keys + 4 bytes of padding

constexpr int kQuantWarps = 8;
constexpr int kQuantRows = 128 / kQuantWarps;   // rows per warp

__global__ void __launch_bounds__(32 * kQuantWarps)
quantize_fp8_kernel(const QuantParams p) {
    __shared__ float s_amax[kQuantWarps];
    __shared__ __align__(16) uint8_t s_t[128 * kQuantRowPitch];
    const int item = blockIdx.x;
    const int blk = item % p.nb;
    const int bh = item / p.nb;
    const int h = bh % p.H;
    const int b = bh / p.H;
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();
    const int r0 = blk * 128;

    float sg[4] = {1.f, 1.f, 1.f, 1.f};
    if (p.signs) {
#pragma unroll
        for (int e = 0; e < 4; ++e) sg[e] = p.signs[4 * lane + e];
    }
    // all row loads first, so they are in flight together
    uint2 raw[kQuantRows];
#pragma unroll
    for (int k = 0; k < kQuantRows; ++k) {
        const int r = r0 + warp + kQuantWarps * k;
        raw[k] = make_uint2(0u, 0u);
        if (r < p.N)
            raw[k] = __ldg(reinterpret_cast<const uint2*>(
                p.x + ((static_cast<size_t>(b) * p.N + r) * p.H + h) * 128 + 4 * lane));
    }
    float y[kQuantRows][4];
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < kQuantRows; ++k) {
        float x4[4];
        x4[0] = __uint_as_float(raw[k].x << 16);
        x4[1] = __uint_as_float(raw[k].x & 0xffff0000u);
        x4[2] = __uint_as_float(raw[k].y << 16);
        x4[3] = __uint_as_float(raw[k].y & 0xffff0000u);
        if (p.signs) {
#pragma unroll
            for (int e = 0; e < 4; ++e) x4[e] = __fmul_rn(x4[e], sg[e]);
            // h = 1 and h = 2 inside the lane
            float a = x4[0], c = x4[1];
            x4[0] = __fadd_rn(a, c);
            x4[1] = __fsub_rn(a, c);
            a = x4[2];
            c = x4[3];
            x4[2] = __fadd_rn(a, c);
            x4[3] = __fsub_rn(a, c);
            a = x4[0];
            c = x4[2];
            x4[0] = __fadd_rn(a, c);
            x4[2] = __fsub_rn(a, c);
            a = x4[1];
            c = x4[3];
            x4[1] = __fadd_rn(a, c);
            x4[3] = __fsub_rn(a, c);
            // h = 4 .. 64: partner lane l ^ (h / 4); the lower lane keeps a + b,
            // the upper a - b (a = the lower lane's value).  One fma with a
            // +-1 factor: the product is exact, so the single rounding gives
            // exactly the sum or the difference.
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const float sgn = (lane & m) ? -1.f : 1.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float o = __shfl_xor_sync(0xffffffffu, x4[e], m);
                    x4[e] = __fmaf_rn(sgn, x4[e], o);
                }
            }
            const float cnorm = 0.08838834764831845f;   // 1/sqrt(128), rounded to float
#pragma unroll
            for (int e = 0; e < 4; ++e) x4[e] = __fmul_rn(x4[e], cnorm);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            y[k][e] = x4[e];
            amax = fmaxf(amax, fabsf(x4[e]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) s_amax[warp] = amax;
    __syncthreads();
    amax = s_amax[0];
#pragma unroll
    for (int w = 1; w < kQuantWarps; ++w) amax = fmaxf(amax, s_amax[w]);
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const float inv = __fdiv_rn(1.f, sc);
    if (threadIdx.x == 0) p.scales[static_cast<size_t>(bh) * p.nb + blk] = sc;

#pragma unroll
    for (int k = 0; k < kQuantRows; ++k) {
        const int rr = warp + kQuantWarps * k;
        const int r = r0 + rr;
        float q4[4];
        e4m3_quotient4(y[k], sc, inv, q4);
        const uint32_t code = pack_e4m3x4(q4[0], q4[1], q4[2], q4[3]);
        if (!p.transpose) {
            if (r < p.N)
                *reinterpret_cast<uint32_t*>(
                    p.out + ((static_cast<size_t>(b) * p.N + r) * p.H + h) * 128 + 4 * lane) = code;
        } else {
            // rows past N hold zeros (their codes are 0)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                s_t[(4 * lane + e) * kQuantRowPitch + rr] = static_cast<uint8_t>(code >> (8 * e));
        }
    }
    if (p.transpose) {
        __syncthreads();
        // two threads per channel c, each writing half of the keys r0 .. r0 + 127
        // (those below Np)
        const int c = threadIdx.x >> 1;
        const int half = threadIdx.x & 1;
        const int nkeys = min(128, p.Np - r0);
        uint8_t* dst = p.out + (static_cast<size_t>(bh) * 128 + c) * p.Np + r0;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(s_t + c * kQuantRowPitch);
        for (int w = half; w < nkeys / 16; w += 2) {
            const uint4 v = make_uint4(src[4 * w], src[4 * w + 1], src[4 * w + 2], src[4 * w + 3]);
            *reinterpret_cast<uint4*>(dst + 16 * w) = v;
        }
    }
}

}  // namespace fa
