// decode_kernel.cuh -- a few new queries per sequence against a long cache of
// keys and values (per-token decode, speculative decode, and short prompt
// chunks), split along the keys.
//
// The pages separate this shape from training and prefill (IO-aware essay,
// section on training, prefill and per-token decode, and its scenario table):
// each step adds few queries that must read the whole accumulated K/V cache,
// so the work is bound by the cache's bandwidth, not by matrix throughput, and
// inference with cached keys and values is one of the interfaces the pages
// list (FlashAttention encyclopedia page, "software integration").  With one
// FMA per loaded element for each of QK^T and PV there is nothing for the
// tensor cores to do: the design goal is to keep enough cache bytes in flight
// to run HBM at its copy bandwidth.
//
// One CTA = one (sequence, head, key split).  The cache is [B, Nk, H, d] with
// sequence b using its first nk_b rows; its Nq queries are the last Nq
// positions of those nk_b keys (bottom-right alignment; causal and window
// rules apply at position nk_b - Nq + i).  The key tiles of the (sequence,
// head) are cut into `nsplit` contiguous ranges; each split runs the online
// softmax of the tiled method over its range (same page, "tiled computation
// and online normalisation") and, when nsplit > 1, writes its normalised
// partial output and base-2 log-sum-exp, which combine_kernel merges with the
// same rule the online update uses for two blocks.
//
// Roles (160 threads, two CTAs per SM):
//   warp 0 lane 0   TMA producer: K and V tiles of 64 keys into a 3-stage ring
//   warps 1-4       compute: S = q k^T with one thread per (key, half of the
//                   channels); max and sums through shuffles and a named
//                   barrier; O += p v with one thread per (channel pair, key
//                   group), 8 keys per unrolled step.
#pragma once

#include "sm100.cuh"

namespace fa {

constexpr int kDecMaxQ = 16;     // queries per sequence
constexpr int kDecMaxSplits = 32;

struct DecodeParams {
    const __nv_bfloat16* q;    // [B, Nq, H, D]
    __nv_bfloat16* o;          // [B, Nq, H, D]
    float* lse;                // [B, H, Nq], natural log
    float* o_part;             // nsplit > 1: [nsplit, B*Nq, H, D], each split's O / its own sum
    float* lse_part;           // nsplit > 1: [nsplit, H, B*Nq], each split's base-2 log-sum-exp
    const int* seqlens_k;      // [B] used cache rows per sequence, or nullptr (all Nk)
    int B, H, Nq, Nk;
    int causal, window, nsplit;
    float scale_log2;          // scale * log2(e)
    int* error_word;
    uint64_t timeout_ns;
    int fault_skip;            // test hook: the producer leaves its first tile unloaded
};

template <int D>
struct DecCfg {
    static constexpr int BN = 64;                    // keys per tile
    static constexpr int NSTAGE = 3;
    static constexpr int BOX_BYTES = BN * 128;       // one TMA box: 64 keys x 64 channels
    static constexpr int NBOX = D / 64;
    static constexpr int TILE_BYTES = BN * D * 2;    // one K or V tile
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int THREADS = 160;
    static constexpr int NCT = 128;                  // compute threads
    static constexpr int KGROUPS = NCT / (D / 2);    // PV: key groups (thread = channel pair)
    static constexpr int KPG = BN / KGROUPS;         // keys per group
    static constexpr int OFF_ST = 0;
    // q as fp32 [kDecMaxQ][D]; after the key loop the q and p areas together
    // hold the key groups' partial outputs [KGROUPS - 1][kDecMaxQ][D]
    static constexpr int Q_AREA = (KGROUPS - 1) * kDecMaxQ * D * 4 - kDecMaxQ * BN * 4 > kDecMaxQ * D * 4
                                      ? (KGROUPS - 1) * kDecMaxQ * D * 4 - kDecMaxQ * BN * 4
                                      : kDecMaxQ * D * 4;
    static constexpr int OFF_Q = OFF_ST + NSTAGE * STAGE_BYTES;
    static constexpr int OFF_P = OFF_Q + Q_AREA;                       // fp32 [kDecMaxQ][BN]
    static constexpr int OFF_RED = OFF_P + kDecMaxQ * BN * 4;          // fp32 [4][kDecMaxQ]
    static constexpr int OFF_BAR = OFF_RED + 4 * kDecMaxQ * 4;
    static constexpr int OFF_MISC = OFF_BAR + 2 * NSTAGE * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    // the key groups' partial outputs are summed through the q and p areas
    static_assert((KGROUPS - 1) * kDecMaxQ * D * 4 <= OFF_RED - OFF_Q, "reduction space");
};

// Named barrier over the 128 compute threads (id 1) that also ORs a predicate
// across them, so that every compute thread takes the same branch afterwards.
__device__ __forceinline__ bool compute_barrier_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred))
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void compute_barrier() {
    asm volatile("barrier.cta.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Key-tile range [tb, te) of split `split` for a sequence with nk used keys
// and nq queries; false for a split that has no tiles.
__device__ __forceinline__ bool decode_split_range(int nk, int nq, int causal, int window, int BN,
                                                   int nsplit, int split, int& tb, int& te) {
    (void)causal;   // the last query sits at position nk - 1: causal keeps every key below nk
    int k_lo = 0;
    if (window > 0) k_lo = max(0, nk - nq - window + 1);
    const int t0 = k_lo / BN;
    const int t1 = (nk + BN - 1) / BN;
    const int n = t1 - t0;
    const int ns = min(nsplit, n);
    if (split >= ns) return false;
    tb = t0 + static_cast<int>(static_cast<int64_t>(split) * n / ns);
    te = t0 + static_cast<int>(static_cast<int64_t>(split + 1) * n / ns);
    return true;
}

// NQ: compile-time bound on the queries per sequence (1, 2, 4, 8 or 16); the
// runtime count nq <= NQ masks the rest.
template <int D, int NQ>
__global__ void __launch_bounds__(DecCfg<D>::THREADS, 2)
decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const DecodeParams p) {
    using C = DecCfg<D>;
    // the merge launched after this grid (programmatic dependent launch) may
    // be scheduled now; it waits for this grid's completion before reading
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    float* sq = reinterpret_cast<float*>(smem + C::OFF_Q);
    float* sp = reinterpret_cast<float*>(smem + C::OFF_P);
    float* sred = reinterpret_cast<float*>(smem + C::OFF_RED);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + C::NSTAGE;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);

    const int H = p.H, nq = p.Nq;
    const int item = blockIdx.x;
    const int b = item / (H * p.nsplit);
    const int rem = item - b * H * p.nsplit;
    const int h = rem / p.nsplit;
    const int split = rem - h * p.nsplit;
    const int nk = p.seqlens_k ? min(max(p.seqlens_k[b], 0), p.Nk) : p.Nk;
    const int rows = p.B * nq;                     // query rows of the whole batch
    const int qpos0 = nk - nq;                     // key position of query 0
    const float kNegInf = -INFINITY;

    int tb = 0, te = 0;
    if (!decode_split_range(nk, nq, p.causal, p.window, C::BN, p.nsplit, split, tb, te)) {
        // A split without keys: its queries see nothing here.
        for (int i = threadIdx.x; i < nq; i += blockDim.x) {
            const int row = b * nq + i;
            if (p.nsplit > 1) {
                p.lse_part[(static_cast<size_t>(split) * H + h) * rows + row] = kNegInf;
            } else {
                p.lse[(static_cast<size_t>(b) * H + h) * nq + i] = kNegInf;
            }
        }
        if (p.nsplit == 1)
            for (int e = threadIdx.x; e < nq * D; e += blockDim.x) {
                const int i = e / D, c = e - i * D;
                p.o[((static_cast<size_t>(b) * nq + i) * H + h) * D + c] = __float2bfloat16(0.f);
            }
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 4);                 // one arrival per compute warp
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    // queries of this (sequence, head) as fp32 in shared memory (zero past nq)
    for (int e = threadIdx.x; e < NQ * D; e += blockDim.x) {
        const int i = e / D, c = e - i * D;
        sq[i * D + c] = i < nq ? __bfloat162float(p.q[((static_cast<size_t>(b) * nq + i) * H + h) * D + c])
                               : 0.f;
    }
    __syncthreads();
    const WaitCtl wc{abort_flag, p.error_word, p.timeout_ns};
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            tma_prefetch_map(&tm_k);
            tma_prefetch_map(&tm_v);
            uint32_t cnt = 0;
            uint32_t skipped_at = 0xffffffffu;
            bool ok = true;
            for (int t = tb; t < te; ++t, ++cnt) {
                const int slot = cnt % C::NSTAGE;
                if (!mbar_wait(empty + slot, ((cnt / C::NSTAGE) & 1) ^ 1, wc)) { ok = false; break; }
                mbar_arrive_expect_tx(full + slot, C::STAGE_BYTES);
                if (p.fault_skip && cnt == 0) {
                    skipped_at = cnt;           // test hook: this stage never fills
                    continue;
                }
                uint8_t* st = smem + C::OFF_ST + slot * C::STAGE_BYTES;
                const int row = b * p.Nk + t * C::BN;
                for (int bx = 0; bx < C::NBOX; ++bx) {
                    tma_load_3d(st + bx * C::BOX_BYTES, &tm_k, full + slot, bx * 64, h, row);
                    tma_load_3d(st + C::TILE_BYTES + bx * C::BOX_BYTES, &tm_v, full + slot, bx * 64, h,
                                row);
                }
            }
            if (!ok || skipped_at != 0xffffffffu) {
                // let the copies in flight land before the CTA exits
                for (uint32_t x = cnt > C::NSTAGE ? cnt - C::NSTAGE : 0; x < cnt; ++x) {
                    if (x == skipped_at) continue;
                    volatile int no_abort = 0;
                    WaitCtl dw{&no_abort, p.error_word, 200000000ull};
                    mbar_wait(full + x % C::NSTAGE, (x / C::NSTAGE) & 1, dw);
                }
            }
        }
        return;
    }

    // ------------------------------------------------------------ compute --
    const int ct = threadIdx.x - 32;               // 0..127
    const int cw = ct >> 5;                        // compute warp 0..3
    // S phase: key kk of the tile, channels [hf * D/2, hf * D/2 + D/2)
    const int kk = ct >> 1;
    const int hf = ct & 1;
    // PV phase: channel pair cp (channels 2cp, 2cp+1), keys of group g
    const int cp = ct % (D / 2);
    const int g = ct / (D / 2);
    const int c2 = 2 * cp;
    const uint32_t v_off = C::TILE_BYTES + (c2 >> 6) * C::BOX_BYTES + (c2 & 7) * 2;
    const int v_cr = (c2 & 63) >> 3;

    // With one query its half row of q stays in registers.
    float qreg[NQ == 1 ? D / 2 : 1];
    if (NQ == 1) {
#pragma unroll
        for (int e = 0; e < D / 2; ++e) qreg[e] = sq[hf * (D / 2) + e];
    }

    float m_run[NQ], l_part[NQ], o0[NQ], o1[NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        m_run[i] = kNegInf;
        l_part[i] = 0.f;
        o0[i] = 0.f;
        o1[i] = 0.f;
    }
    bool aborted = false;
    uint32_t cnt = 0;
    for (int t = tb; t < te; ++t, ++cnt) {
        const int slot = cnt % C::NSTAGE;
        const bool got = mbar_wait(full + slot, (cnt / C::NSTAGE) & 1, wc);
        const uint8_t* st = smem + C::OFF_ST + slot * C::STAGE_BYTES;
        const int k0 = t * C::BN;
        // ---- S = q k^T for key kk (two threads per key, half the channels each)
        float acc[NQ];
#pragma unroll
        for (int i = 0; i < NQ; ++i) acc[i] = 0.f;
#pragma unroll
        for (int u = 0; u < D / 16; ++u) {
            const int c0 = hf * (D / 2) + u * 8;
            const int bx = c0 >> 6, cr = (c0 & 63) >> 3;
            const uint4 kv = *reinterpret_cast<const uint4*>(st + bx * C::BOX_BYTES + kk * 128 +
                                                             ((cr ^ (kk & 7)) << 4));
            const float k8[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                                 bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
            if (NQ == 1) {
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[0] = fmaf(qreg[u * 8 + e], k8[e], acc[0]);
            } else {
#pragma unroll
                for (int i = 0; i < NQ; ++i) {
                    const float4 qa = *reinterpret_cast<const float4*>(sq + i * D + c0);
                    const float4 qb = *reinterpret_cast<const float4*>(sq + i * D + c0 + 4);
                    acc[i] = fmaf(qa.x, k8[0], acc[i]);
                    acc[i] = fmaf(qa.y, k8[1], acc[i]);
                    acc[i] = fmaf(qa.z, k8[2], acc[i]);
                    acc[i] = fmaf(qa.w, k8[3], acc[i]);
                    acc[i] = fmaf(qb.x, k8[4], acc[i]);
                    acc[i] = fmaf(qb.y, k8[5], acc[i]);
                    acc[i] = fmaf(qb.z, k8[6], acc[i]);
                    acc[i] = fmaf(qb.w, k8[7], acc[i]);
                }
            }
        }
        const int kpos = k0 + kk;
        float x[NQ];
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            const float full_dot = acc[i] + __shfl_xor_sync(0xffffffffu, acc[i], 1);
            const int qp = qpos0 + i;
            const bool allowed = i < nq && kpos < nk && (!p.causal || kpos <= qp) &&
                                 (p.window <= 0 || kpos > qp - p.window);
            x[i] = allowed ? full_dot * p.scale_log2 : kNegInf;
            // tile maximum within the warp (lane pairs hold the same key)
            float m = x[i];
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
            if (lane == 0) sred[cw * kDecMaxQ + i] = m;
        }
        if (compute_barrier_or(!got || *abort_flag)) { aborted = true; break; }
        // ---- online softmax update (every compute thread holds the row state)
        float alpha[NQ];
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            const float mt = fmaxf(fmaxf(sred[i], sred[kDecMaxQ + i]),
                                   fmaxf(sred[2 * kDecMaxQ + i], sred[3 * kDecMaxQ + i]));
            const float m_new = fmaxf(m_run[i], mt);
            alpha[i] = 1.f;
            float pv = 0.f;
            if (m_new != kNegInf) {
                alpha[i] = ex2(m_run[i] - m_new);      // 0 while m_run is -inf
                m_run[i] = m_new;
                pv = ex2(x[i] - m_new);                // masked: ex2(-inf) = 0
            }
            l_part[i] = fmaf(l_part[i], alpha[i], hf == 0 ? pv : 0.f);
            if (hf == 0) sp[i * C::BN + kk] = pv;
        }
        compute_barrier();
        // ---- O += p v: channel pair cp, keys of group g; keys past nk are never read
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            o0[i] *= alpha[i];
            o1[i] *= alpha[i];
        }
        const int kb = g * C::KPG;
        const int ke = min(C::BN, nk - k0);       // valid keys of the tile (k0 < nk)
        const uint8_t* vbase = st + v_off;
        if (ke >= kb + C::KPG) {
            // whole group valid: unrolled in chunks of 8 keys
#pragma unroll
            for (int j0 = 0; j0 < C::KPG; j0 += 8) {
                float va[8], vb[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = kb + j0 + e;
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(
                        vbase + j * 128 + ((v_cr ^ (j & 7)) << 4));
                    va[e] = bf16_lo(w);
                    vb[e] = bf16_hi(w);
                }
#pragma unroll
                for (int i = 0; i < NQ; ++i) {
                    const float4 pa = *reinterpret_cast<const float4*>(sp + i * C::BN + kb + j0);
                    const float4 pb = *reinterpret_cast<const float4*>(sp + i * C::BN + kb + j0 + 4);
                    const float pp[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        o0[i] = fmaf(pp[e], va[e], o0[i]);
                        o1[i] = fmaf(pp[e], vb[e], o1[i]);
                    }
                }
            }
        } else {
            const int je = min(ke, kb + C::KPG);
            for (int j = kb; j < je; ++j) {
                const uint32_t w = *reinterpret_cast<const uint32_t*>(
                    vbase + j * 128 + ((v_cr ^ (j & 7)) << 4));
                const float va = bf16_lo(w), vb = bf16_hi(w);
#pragma unroll
                for (int i = 0; i < NQ; ++i) {
                    const float pp = sp[i * C::BN + j];
                    o0[i] = fmaf(pp, va, o0[i]);
                    o1[i] = fmaf(pp, vb, o1[i]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + slot);
    }
    if (aborted) return;

    // -------------------------------------------------------- epilogue --
    compute_barrier();                 // every thread is done with q, p and the tiles
    // row sums: l_part lives on the hf == 0 threads
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        float l = l_part[i];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (lane == 0) sred[cw * kDecMaxQ + i] = l;
    }
    // key groups 1.. hand their partial sums to group 0 (through the q/p area)
    float* sgrp = sq;
    if (g > 0) {
#pragma unroll
        for (int i = 0; i < NQ; ++i)
            *reinterpret_cast<float2*>(sgrp + ((g - 1) * kDecMaxQ + i) * D + c2) =
                make_float2(o0[i], o1[i]);
    }
    compute_barrier();
    if (g != 0) return;
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        if (i < nq) {
            const float l = (sred[i] + sred[kDecMaxQ + i]) + (sred[2 * kDecMaxQ + i] + sred[3 * kDecMaxQ + i]);
            float a0 = o0[i], a1 = o1[i];
#pragma unroll
            for (int gg = 1; gg < C::KGROUPS; ++gg) {
                const float2 t2 = *reinterpret_cast<const float2*>(sgrp + ((gg - 1) * kDecMaxQ + i) * D + c2);
                a0 += t2.x;
                a1 += t2.y;
            }
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int row = b * nq + i;
            if (p.nsplit == 1) {
                *reinterpret_cast<uint32_t*>(p.o + (static_cast<size_t>(row) * H + h) * D + c2) =
                    pack_bf16(a0 * inv, a1 * inv);
                if (cp == 0)
                    p.lse[(static_cast<size_t>(b) * H + h) * nq + i] =
                        l > 0.f ? (m_run[i] + __log2f(l)) * 0.6931471805599453f : kNegInf;
            } else {
                *reinterpret_cast<float2*>(p.o_part + ((static_cast<size_t>(split) * rows + row) * H + h) * D + c2) =
                    make_float2(a0 * inv, a1 * inv);
                if (cp == 0)
                    p.lse_part[(static_cast<size_t>(split) * H + h) * rows + row] =
                        l > 0.f ? m_run[i] + __log2f(l) : kNegInf;
            }
        }
    }
}

// Merge the splits of each (query row, head): with M the largest split
// log-sum-exp (base 2) and w_s = 2^(lse_s - M), O = sum_s w_s O_s / sum_s w_s
// and LSE = ln 2 * (M + log2 sum_s w_s) -- the two-block case of the online
// normalisation update.  One warp per (row, head); splits with no allowed key
// (lse_s = -inf) carry weight 0 and their O_s is not read.
template <int D>
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
               __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int rows, int H, int Nq,
               int nsplit) {
    // launched as a programmatic dependent of the split kernel: wait until it
    // has completed and its partials are visible (returns at once otherwise)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = lane_id();
    if (warp_global >= rows * H) return;
    const int row = warp_global / H;
    const int h = warp_global - row * H;
    const float l2 = lane < nsplit ? lse_part[(static_cast<size_t>(lane) * H + h) * rows + row]
                                   : -INFINITY;
    float M = l2;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, s));
    const float w = (l2 == -INFINITY) ? 0.f : ex2(l2 - M);
    float W = w;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) W += __shfl_xor_sync(0xffffffffu, W, s);
    constexpr int CPL = D / 32;                  // channels per lane
    float acc[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float ws = __shfl_sync(0xffffffffu, w, s);
        if (ws == 0.f) continue;
        const float* src = o_part + ((static_cast<size_t>(s) * rows + row) * H + h) * D + lane * CPL;
        if (CPL == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            acc[0] = fmaf(ws, v.x, acc[0]);
            acc[1] = fmaf(ws, v.y, acc[1]);
            acc[2] = fmaf(ws, v.z, acc[2]);
            acc[3] = fmaf(ws, v.w, acc[3]);
        } else {
#pragma unroll
            for (int e = 0; e < CPL; ++e) acc[e] = fmaf(ws, src[e], acc[e]);
        }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    __nv_bfloat16* dst = o + (static_cast<size_t>(row) * H + h) * D + lane * CPL;
#pragma unroll
    for (int e = 0; e < CPL; ++e) dst[e] = __float2bfloat16(acc[e] * inv);
    if (lane == 0) {
        const int bq = row / Nq, i = row - bq * Nq;
        lse[(static_cast<size_t>(bq) * H + h) * Nq + i] =
            W > 0.f ? (M + __log2f(W)) * 0.6931471805599453f : -INFINITY;
    }
}

}  // namespace fa
