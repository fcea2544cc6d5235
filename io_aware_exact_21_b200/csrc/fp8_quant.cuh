// fp8_quant.cuh -- block quantisation of bf16 Q, K, V to e4m3 for the FP8
// forward (FlashAttention encyclopedia page, FlashAttention-3 paragraph: the
// FP8 path quantises by blocks and adds a step that reduces quantisation
// error).
//
// Persistent CTAs (two per SM, 256 threads) walk the (sequence, head, block of
// 128 rows) blocks; each block arrives in shared memory by TMA (two boxes of
// 64 channels x 128 rows, 128-byte swizzle) into one of two buffers, so the
// next block's load runs while this one is computed.  Eight lanes share a row,
// lane l of the eight holding channels 16 l .. 16 l + 15; a thread takes four
// consecutive rows.
//  * optional rotation (Q and K): multiply by a sign vector, then the
//    orthonormal Walsh-Hadamard transform -- butterflies (a, b) -> (a + b,
//    a - b) on channel pairs (j, j + h) for h = 1, 2, 4, ..., 64 in that
//    order (h <= 8 inside a lane, h = 16, 32, 64 across the row's lanes by
//    shuffles), then a factor 1/sqrt(128).  Every step is an explicitly
//    rounded float32 operation, so the codes do not depend on how a compiler
//    would contract them.  q.k is unchanged by the rotation.
//  * scale s = amax / 448 over the block (1 for an all-zero block); codes are
//    e4m3(x / s), the real quotient rounded once to the nearest e4m3 value
//    (ties to even, saturating at +-448): see e4m3_quotient.cuh.
//  * layout: Q and K codes keep the token-major [B, N, H, 128] layout; V codes
//    are written transposed, [B, H, 128, Np] with Np = N rounded up to 16 and
//    zeros past N, so the forward's PV GEMM reads a K-major operand.
#pragma once

#include "e4m3_quotient.cuh"
#include "sm100.cuh"

namespace fa {

struct QuantParams {
    const __nv_bfloat16* x;    // [B, N, H, 128] (read through the tensor map)
    uint8_t* out;              // codes
    float* scales;             // [B, H, nb]
    const float* signs;        // 128 entries of +-1, or nullptr (no rotation)
    int B, N, H, nb, Np;
    int transpose;             // 1: write [B, H, 128, Np] (selects the kernel)
    int* error_word;           // global: a wait that ran out records DEV_TIMEOUT
    uint64_t timeout_ns;
};

struct QuantCfg {
    static constexpr int RPT = 4;                         // rows per thread
    static constexpr int THREADS = 128 * 8 / RPT;         // eight lanes per row
    static constexpr int WARPS = THREADS / 32;
    static constexpr int BOX_BYTES = 128 * 128;           // 64 bf16 channels x 128 rows
    static constexpr int BLOCK_BYTES = 2 * BOX_BYTES;     // one block of 128 rows x 128 channels
    static constexpr int NBUF = 2;
    static constexpr int T_PITCH = 132;                   // transpose tile: 128 keys + 4 bytes
    static constexpr int OFF_BUF = 0;
    static constexpr int OFF_T = OFF_BUF + NBUF * BLOCK_BYTES;
    static constexpr int OFF_AMAX = OFF_T + 128 * T_PITCH;   // float[2][WARPS]
    static constexpr int OFF_SIGN = OFF_AMAX + 2 * WARPS * 4; // float[128]
    static constexpr int OFF_BAR = OFF_SIGN + 128 * 4;        // uint64_t[NBUF]
    static constexpr int OFF_MISC = OFF_BAR + NBUF * 8;      // abort flag
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
};

// Byte offset of the 16-byte chunk `j` (0..15) of row `r` in a block buffer:
// chunk j lies in box j / 8, at chunk j % 8 of the row's 128 bytes, XORed
// with r % 8 by the 128-byte swizzle.
__device__ __forceinline__ uint32_t quant_chunk_offset(int r, int j) {
    return static_cast<uint32_t>((j >> 3) * QuantCfg::BOX_BYTES + r * 128 + (((j & 7) ^ (r & 7)) << 4));
}

// 4 x 4 byte transpose: word e of the result holds byte e of a, b, c, d (in
// that order, lowest byte first).
__device__ __forceinline__ void transpose_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                                 uint32_t (&w)[4]) {
    const uint32_t ab_lo = __byte_perm(a, b, 0x5140), ab_hi = __byte_perm(a, b, 0x7362);
    const uint32_t cd_lo = __byte_perm(c, d, 0x5140), cd_hi = __byte_perm(c, d, 0x7362);
    w[0] = __byte_perm(ab_lo, cd_lo, 0x5410);
    w[1] = __byte_perm(ab_lo, cd_lo, 0x7632);
    w[2] = __byte_perm(ab_hi, cd_hi, 0x5410);
    w[3] = __byte_perm(ab_hi, cd_hi, 0x7632);
}

// Block `item` = (sequence b, head h, rows 128 blk ..) of x into a buffer:
// two boxes of 64 channels, completion on `bar`.
__device__ __forceinline__ void quant_issue_load(const CUtensorMap* tm, const QuantParams& p, int item,
                                                 uint8_t* dst, uint64_t* bar) {
    const int blk = item % p.nb;
    const int bh = item / p.nb;
    const int h = bh % p.H;
    const int b = bh / p.H;
    mbar_arrive_expect_tx(bar, QuantCfg::BLOCK_BYTES);
    tma_load_3d(dst, tm, bar, 0, h, b * p.N + blk * 128);
    tma_load_3d(dst + QuantCfg::BOX_BYTES, tm, bar, 64, h, b * p.N + blk * 128);
}

// kRotate: signs and the Walsh-Hadamard transform (p.signs non-null);
// kTranspose: the channel-major V layout (p.transpose = 1).
template <bool kRotate, bool kTranspose>
__global__ void __launch_bounds__(QuantCfg::THREADS, 2)
quantize_fp8_kernel(const __grid_constant__ CUtensorMap tm_x, const QuantParams p) {
    using C = QuantCfg;
    static_assert(C::RPT == 2 || C::RPT == 4, "two or four rows per thread");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    uint8_t* s_t = smem + C::OFF_T;
    float* s_amax = reinterpret_cast<float*>(smem + C::OFF_AMAX);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();
    const int g = lane >> 3;               // which of the warp's four row groups
    const int l8 = lane & 7;               // channels 16 l8 .. 16 l8 + 15
    const int nblocks = p.B * p.H * p.nb;

    if (threadIdx.x == 0) {
        for (int b = 0; b < C::NBUF; ++b) mbar_init(full + b, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_map(&tm_x);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 0; k < C::NBUF; ++k) {
            const int item = blockIdx.x + k * gridDim.x;
            if (item < nblocks) quant_issue_load(&tm_x, p, item, smem + C::OFF_BUF + k * C::BLOCK_BYTES, full + k);
        }
    }
    float* s_sign = reinterpret_cast<float*>(smem + C::OFF_SIGN);
    if (kRotate && threadIdx.x < 128) s_sign[threadIdx.x] = __ldg(p.signs + threadIdx.x);
    __syncthreads();
    const WaitCtl wc{abort_flag, p.error_word, p.timeout_ns};

    uint32_t k = 0;
    bool aborted = false;
    for (int item = blockIdx.x; item < nblocks; item += gridDim.x, ++k) {
        const int buf = k & (C::NBUF - 1);
        const bool ok = mbar_wait(full + buf, (k / C::NBUF) & 1, wc);
        if (!__syncthreads_and(ok)) {      // the same decision in every thread
            aborted = true;
            break;
        }
        const int blk = item % p.nb;
        const int bh = item / p.nb;
        const int h = bh % p.H;
        const int b = bh / p.H;
        const int r0 = blk * 128;
        const uint8_t* sb = smem + C::OFF_BUF + buf * C::BLOCK_BYTES;
        const int rbase = warp * 4 * C::RPT + g * C::RPT;   // this thread's rows: rbase .. + RPT - 1

        float y[C::RPT][16];
        float amax = 0.f;
#pragma unroll
        for (int kk = 0; kk < C::RPT; ++kk) {
            const int rr = rbase + kk;
            const uint4 u0 = *reinterpret_cast<const uint4*>(sb + quant_chunk_offset(rr, 2 * l8));
            const uint4 u1 = *reinterpret_cast<const uint4*>(sb + quant_chunk_offset(rr, 2 * l8 + 1));
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            float v[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[2 * e] = __uint_as_float(w[e] << 16);
                v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
            }
            if (r0 + rr >= p.N) {
                // past the sequence end: the box holds the next sequence's rows
                // (or the tensor map's zero fill); the block treats them as zeros
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = 0.f;
            }
            if constexpr (kRotate) {
                const float4* sg4 = reinterpret_cast<const float4*>(s_sign + 16 * l8);
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 sg = sg4[e4];
                    v[4 * e4] = __fmul_rn(v[4 * e4], sg.x);
                    v[4 * e4 + 1] = __fmul_rn(v[4 * e4 + 1], sg.y);
                    v[4 * e4 + 2] = __fmul_rn(v[4 * e4 + 2], sg.z);
                    v[4 * e4 + 3] = __fmul_rn(v[4 * e4 + 3], sg.w);
                }
                // h = 1, 2, 4, 8 inside the lane
#pragma unroll
                for (int hh = 1; hh < 16; hh <<= 1) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        if (e & hh) continue;
                        const float a = v[e], c = v[e + hh];
                        v[e] = __fadd_rn(a, c);
                        v[e + hh] = __fsub_rn(a, c);
                    }
                }
                // h = 16, 32, 64: partner lane l8 ^ (h / 16) of the same row; the
                // lower lane keeps a + b, the upper a - b (a = the lower lane's
                // value).  One fma with a +-1 factor: the product is exact, so
                // the single rounding gives exactly the sum or the difference.
#pragma unroll
                for (int m = 1; m < 8; m <<= 1) {
                    const float sgn = (l8 & m) ? -1.f : 1.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
                        v[e] = __fmaf_rn(sgn, v[e], o);
                    }
                }
                const float cnorm = 0.08838834764831845f;   // 1/sqrt(128), rounded to float
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = __fmul_rn(v[e], cnorm);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                y[kk][e] = v[e];
                amax = fmaxf(amax, fabsf(v[e]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        float* sa = s_amax + (k & 1) * C::WARPS;
        if (lane == 0) sa[warp] = amax;
        __syncthreads();   // the block's amax is complete and its buffer has been read
        if (threadIdx.x == 0) {
            const int next = item + C::NBUF * gridDim.x;
            if (next < nblocks)
                quant_issue_load(&tm_x, p, next, smem + C::OFF_BUF + buf * C::BLOCK_BYTES, full + buf);
        }
        amax = sa[0];
#pragma unroll
        for (int w = 1; w < C::WARPS; ++w) amax = fmaxf(amax, sa[w]);
        const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        const float inv = __fdiv_rn(1.f, sc);
        if (threadIdx.x == 0) p.scales[static_cast<size_t>(bh) * p.nb + blk] = sc;

        uint32_t code[C::RPT][4];  // [row][four channels]
#pragma unroll
        for (int kk = 0; kk < C::RPT; ++kk) {
            if constexpr (kRotate) {
                // rotated values are full float32 numbers whose products rarely
                // fall near an e4m3 midpoint: the rounded product decides unless
                // some lane of the warp has such a value in this row, and only
                // then does the warp take the exact step for the row
                float qv[16];
                bool slow = false;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    qv[e] = __fmul_rn(y[kk][e], inv);
                    slow = slow || !e4m3_product_decides(qv[e]);
                }
                if (__any_sync(0xffffffffu, slow)) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) qv[e] = e4m3_quotient(y[kk][e], sc, inv);
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    code[kk][c4] = pack_e4m3x4(qv[4 * c4], qv[4 * c4 + 1], qv[4 * c4 + 2], qv[4 * c4 + 3]);
            } else {
                // bf16 values put 0.6 % of their products near a midpoint, so
                // every value takes the exact step (no branch)
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const float x4[4] = {y[kk][4 * c4], y[kk][4 * c4 + 1], y[kk][4 * c4 + 2], y[kk][4 * c4 + 3]};
                    float q4[4];
                    e4m3_quotient4(x4, sc, inv, q4);
                    code[kk][c4] = pack_e4m3x4(q4[0], q4[1], q4[2], q4[3]);
                }
            }
            if constexpr (!kTranspose) {
                const int r = r0 + rbase + kk;
                if (r < p.N)
                    *reinterpret_cast<uint4*>(p.out + ((static_cast<size_t>(b) * p.N + r) * p.H + h) * 128 +
                                              16 * l8) =
                        make_uint4(code[kk][0], code[kk][1], code[kk][2], code[kk][3]);
            }
        }
        if constexpr (kTranspose) {
            // channel-major tile: row c holds the codes of channel c for keys
            // r0 .. r0 + 127 (rows past N hold zeros, their codes are 0)
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                if constexpr (C::RPT == 4) {
                    uint32_t w[4];
                    transpose_bytes4(code[0][c4], code[1][c4], code[2][c4], code[3][c4], w);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<uint32_t*>(s_t + (16 * l8 + 4 * c4 + e) * C::T_PITCH + rbase) = w[e];
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)   // byte e of both rows' words
                        *reinterpret_cast<uint16_t*>(s_t + (16 * l8 + 4 * c4 + e) * C::T_PITCH + rbase) =
                            static_cast<uint16_t>(__byte_perm(code[0][c4], code[1][c4], 0x40 + 0x11 * e));
                }
            }
            __syncthreads();
            // THREADS / 128 threads per channel c, each writing every such
            // 16-key chunk of the keys r0 .. r0 + 127 (those below Np); the
            // next block's tile writes come after that block's barriers
            constexpr int TPC = C::THREADS / 128;
            const int c = threadIdx.x / TPC;
            const int part = threadIdx.x % TPC;
            const int nkeys = min(128, p.Np - r0);
            uint8_t* dst = p.out + (static_cast<size_t>(bh) * 128 + c) * p.Np + r0;
            const uint32_t* src = reinterpret_cast<const uint32_t*>(s_t + c * C::T_PITCH);
            for (int w = part; w < nkeys / 16; w += TPC) {
                const uint4 v4 = make_uint4(src[4 * w], src[4 * w + 1], src[4 * w + 2], src[4 * w + 3]);
                *reinterpret_cast<uint4*>(dst + 16 * w) = v4;
            }
        }
    }
    if (aborted && threadIdx.x == 0) {
        // copies still in flight (this block's and the next one's) land before
        // the CTA's shared memory is released; each wait is bounded
        volatile int no_abort = 0;
        const WaitCtl dw{&no_abort, p.error_word, 200000000ull};
        for (uint32_t x = k; x < k + C::NBUF; ++x) {
            if (blockIdx.x + x * gridDim.x < static_cast<uint32_t>(nblocks))
                mbar_wait(full + (x & (C::NBUF - 1)), (x / C::NBUF) & 1, dw);
        }
    }
}

}  // namespace fa
