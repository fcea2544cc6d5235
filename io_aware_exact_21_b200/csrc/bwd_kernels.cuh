// bwd_kernels.cuh -- backward pass of exact attention for sm_100a.
//
// The pages only say that the backward pass keeps compact normalisation
// statistics from the forward and recomputes the attention blocks it needs
// instead of storing the probability matrix (FlashAttention encyclopedia page,
// "training and complexity").  With the forward's per-row log-sum-exp L_i the
// probabilities are recomputed exactly, P_ij = exp(scale s_ij - L_i), and the
// gradients follow from the definition O = softmax(scale Q K^T) V:
//   D_i   = sum_j P_ij (dO_i . v_j) = dO_i . O_i
//   dV_j  = sum_i P_ij dO_i
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dK_j  = scale * sum_i dS_ij q_i
//   dQ_i  = scale * sum_j dS_ij k_j
//
// Three kernels on the caller's stream:
//   1. dot_kernel : D_i = rowsum(dO_i * O_i) in fp32, one row per group of
//      d/8 lanes reading 16-byte vectors, reduced with warp shuffles.
//   2. dkdv_kernel: a CTA owns 128 keys of one (sequence, head) and streams
//      the query tiles (64 rows) that can see them.  Per query tile:
//        S^T = K Q^T and dP^T = V dO^T        (tcgen05, both operands in smem)
//        P^T = 2^(S^T scale log2e - L log2e), dS^T = P^T (dP^T - D)   (fp32)
//        dV += P^T dO and dK += dS^T Q        (tcgen05, P^T / dS^T from TMEM)
//   3. dq_kernel  : a CTA owns 128 queries and streams the key tiles (64 keys):
//        S = Q K^T, dP = dO V^T, P, dS as above, dQ += dS K.
// Both big kernels use the forward's role split (TMA warp, MMA warp, two
// element-wise warpgroups, each taking one 32-column half of every score
// tile) and double-buffer the score tiles in TMEM, so the element-wise work
// of one tile overlaps the GEMMs of the next.  Deterministic: no atomics.
#pragma once

#include "schedule.cuh"
#include "sm100.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
    Geometry g;
    const float* lse;       // layout: fixed [B, H, N], packed [H, T]
    const float* dsum;      // D, same layout
    __nv_bfloat16* out0;    // dK (dkdv_kernel) or dQ (dq_kernel)
    __nv_bfloat16* out1;    // dV (dkdv_kernel)
    float scale;
    float scale_log2;
    int* error_word;
    uint64_t timeout_ns;
};

// Index of row i of sequence s, head h in an LSE-shaped array.
__device__ __forceinline__ size_t rowstat_index(const Geometry& g, int s, int h, int start, int i) {
    return g.cu_seqlens ? static_cast<size_t>(h) * g.T + start + i
                        : (static_cast<size_t>(s) * g.H + h) * g.N + i;
}

// ------------------------------------------------------------ D pre-pass --
template <int D>
__global__ void __launch_bounds__(256)
dot_kernel(const __nv_bfloat16* __restrict__ dO, const __nv_bfloat16* __restrict__ O,
           float* __restrict__ dsum, Geometry g) {
    constexpr int LPR = D / 8;                 // lanes per row (16-byte vectors)
    constexpr int RPW = 32 / LPR;              // rows per warp per iteration
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR;
    const int part = lane % LPR;
    const int64_t rows = static_cast<int64_t>(g.T) * g.H;
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t base = warp_global * RPW; base < rows; base += nwarps * RPW) {
        const int64_t r = base + sub;
        float acc = 0.f;
        if (r < rows) {
            const uint4 a = *reinterpret_cast<const uint4*>(dO + r * D + part * 8);
            const uint4 b = *reinterpret_cast<const uint4*>(O + r * D + part * 8);
            const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fa2 = __bfloat1622float2(pa[e]);
                const float2 fb2 = __bfloat1622float2(pb[e]);
                acc = fmaf(fa2.x, fb2.x, acc);
                acc = fmaf(fa2.y, fb2.y, acc);
            }
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (r < rows && part == 0) {
            const int64_t token = r / g.H;
            const int h = static_cast<int>(r - token * g.H);
            size_t idx;
            if (g.cu_seqlens) {
                idx = static_cast<size_t>(h) * g.T + token;
            } else {
                const int64_t s = token / g.N;
                idx = (static_cast<size_t>(s) * g.H + h) * g.N + (token - s * g.N);
            }
            dsum[idx] = acc;
        }
    }
}

// --------------------------------------------------- shared configuration --
template <int D>
struct BwdCfg {
    static constexpr int BM = 128;               // rows the CTA owns (keys or queries)
    static constexpr int BS = 64;                // rows streamed per step
    static constexpr int NSTAGE = 4;
    static constexpr int NBOX = D / 64;
    static constexpr int FBOX = 128 * 128;       // 128 rows x 128 B
    static constexpr int SBOX = 64 * 128;        // 64 rows x 128 B
    static constexpr int FIX_BYTES = BM * D * 2;
    static constexpr int STR_BYTES = BS * D * 2;
    static constexpr int THREADS = 384;
    static constexpr uint32_t COL_ACC0 = 0, COL_ACC1 = 128;
    __host__ __device__ static constexpr uint32_t col_s(int b) { return 256 + 128 * b; }
    __host__ __device__ static constexpr uint32_t col_dp(int b) { return 256 + 128 * b + 64; }
    static constexpr int OFF_FA = 0;
    static constexpr int OFF_FB = FIX_BYTES;
    static constexpr int OFF_ST = 2 * FIX_BYTES;                  // stage: X then Y
    static constexpr int OFF_VEC = OFF_ST + NSTAGE * 2 * STR_BYTES;  // stage: 64 nl + 64 D
    static constexpr int OFF_BAR = OFF_VEC + NSTAGE * 2 * BS * 4;
    static constexpr int NBAR = 2 + 2 * NSTAGE + 2 + 2 + 2 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_SCRATCH = OFF_MISC + 16;
    static constexpr int OFF_PREFIX = OFF_SCRATCH + THREADS * 4;
    static constexpr int SMEM_BYTES = OFF_PREFIX + (kMaxVarlenSeqs + 1) * 4 + 1024;
};

// Query-tile range [ib, ie) (tiles of BS rows) whose rows can see some key of
// [k_lo, k_hi) in a sequence of length n.
__device__ __forceinline__ void query_tile_range(int k_lo, int k_hi, int n, int causal, int window,
                                                 int BS, int& ib, int& ie) {
    const int q_lo = causal ? k_lo : 0;
    int q_hi = n;
    if (window > 0) q_hi = min(n, k_hi - 1 + window);
    ib = q_lo / BS;
    ie = (q_hi + BS - 1) / BS;
    if (ie < ib) ie = ib;
}

struct BwdBarriers {
    uint64_t *fix_full, *fix_empty, *stage_full, *stage_empty, *s_full, *ready, *acc_final,
        *acc_empty, *drain;
};

template <int D>
__device__ __forceinline__ BwdBarriers carve_barriers(uint8_t* smem) {
    using C = BwdCfg<D>;
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    BwdBarriers r;
    r.fix_full = b;
    r.fix_empty = b + 1;
    r.stage_full = b + 2;
    r.stage_empty = b + 2 + C::NSTAGE;
    r.s_full = b + 2 + 2 * C::NSTAGE;
    r.ready = r.s_full + 2;
    r.acc_final = r.ready + 2;
    r.acc_empty = r.acc_final + 1;
    r.drain = r.acc_empty + 1;
    return r;
}

template <int D>
__device__ __forceinline__ void init_barriers(const BwdBarriers& br, volatile int* abort_flag) {
    using C = BwdCfg<D>;
    mbar_init(br.fix_full, 1);
    mbar_init(br.fix_empty, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
        mbar_init(br.stage_full + s, 1);
        mbar_init(br.stage_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
        mbar_init(br.s_full + b, 1);
        mbar_init(br.ready + b, 8);     // all eight element-wise warps (both halves of a tile)
    }
    mbar_init(br.acc_final, 1);
    mbar_init(br.acc_empty, 8);         // all eight element-wise warps
    mbar_init(br.drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
}

// A-operand (K-major, 128 rows) and B-operand (K-major, 64 rows) descriptors
// for k-step kk of a d-deep contraction: 16 channels = 32 bytes inside the
// 128-byte swizzled rows, next 64-channel box after four steps.
template <int D>
__device__ __forceinline__ void issue_ss_pair(uint32_t d_tmem, uint32_t a_base, uint32_t b_base,
                                              uint32_t idesc) {
    using C = BwdCfg<D>;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t ka = (kk >> 2) * C::FBOX + (kk & 3) * 32;
        const uint32_t kb = (kk >> 2) * C::SBOX + (kk & 3) * 32;
        umma_ss(d_tmem, sw128_desc(a_base + ka, 16, 1024), sw128_desc(b_base + kb, 16, 1024), idesc,
                kk > 0);
    }
}

// Column of the packed bf16 operand for 16-row k-step kk: each element-wise
// warpgroup packs its 32-column half h of a score tile into the first 16 of
// that half's columns (h * 32 ... h * 32 + 15), which it has already read.
__host__ __device__ constexpr uint32_t packed_col(int kk) { return (kk >> 1) * 32 + (kk & 1) * 8; }

// acc[128 x D] (+)= A[tmem, 128 x 64 bf16] * B[smem, 64 x D, MN-major].
template <int D>
__device__ __forceinline__ void issue_ts_acc(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base,
                                             uint32_t idesc, bool accumulate) {
    using C = BwdCfg<D>;
#pragma unroll
    for (int kk = 0; kk < C::BS / 16; ++kk)
        umma_ts(d_tmem, a_tmem + packed_col(kk), sw128_desc(b_base + kk * 2048, C::SBOX, 1024),
                idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* error_word) {
    volatile int no_abort = 0;
    WaitCtl dw{&no_abort, error_word, 200000000ull};
    mbar_wait(bar, parity, dw);
}

// Store one 32-column chunk of a TMEM row (fp32) to bf16 global memory.
__device__ __forceinline__ void store_row_chunk(uint32_t taddr, float mul, __nv_bfloat16* dst,
                                                bool valid) {
    uint32_t r[32];
    tmem_ld32(taddr, r);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
        pk[e] = pack_bf16(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
    if (valid) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int v = 0; v < 4; ++v) d4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
}

// --------------------------------------------------------- dK/dV kernel --
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
            const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const BwdBarriers br = carve_barriers<D>(smem);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    int* scratch = reinterpret_cast<int*>(smem + C::OFF_SCRATCH);
    int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);
    float* vec = reinterpret_cast<float*>(smem + C::OFF_VEC);
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();

    if (threadIdx.x == 0) init_barriers<D>(br, abort_flag);
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_do);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    Schedule sch;
    sch.g = p.g;
    sch.rows_per_item = C::BM;
    sch.heavy_first = 0;       // under a causal mask the first key block sees the most queries
    sch.prefix = prefix;
    sch.total_items = build_schedule_prefix(p.g, C::BM, prefix, scratch);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtl wc{abort_flag, p.error_word, p.timeout_ns};
    const int H = p.g.H;

    if (warp < 4) {
        regs_dealloc<104>();
        if (warp == 0) {
            // ---------------------------------- producer (whole warp) --
            uint32_t cnt = 0, item_it = 0, fix_issued = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < sch.total_items && ok; w += gridDim.x, ++item_it) {
                int s, h, blk;
                sch.item(w, s, h, blk);
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int k0 = blk * C::BM;
                int ib, ie;
                query_tile_range(k0, min(n, k0 + C::BM), n, p.g.causal, p.g.window, C::BS, ib, ie);
                if (lane == 0) {
                    ok = mbar_wait(br.fix_empty, (item_it & 1) ^ 1, wc);
                    if (ok) {
                        mbar_arrive_expect_tx(br.fix_full, 2 * C::FIX_BYTES);
                        for (int b = 0; b < C::NBOX; ++b) {
                            tma_load_3d(smem + C::OFF_FA + b * C::FBOX, &tm_k, br.fix_full, b * 64, h,
                                        sp.start + k0);
                            tma_load_3d(smem + C::OFF_FB + b * C::FBOX, &tm_v, br.fix_full, b * 64, h,
                                        sp.start + k0);
                        }
                        ++fix_issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                for (int i = ib; i < ie && ok; ++i, ++cnt) {
                    const int slot = cnt % C::NSTAGE;
                    if (lane == 0) ok = mbar_wait(br.stage_empty + slot, ((cnt / C::NSTAGE) & 1) ^ 1, wc);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    // per-query statistics of this tile: -L*log2(e) and D (query rows
                    // outside the sequence get -inf, which zeroes their P)
                    float* vs = vec + slot * 2 * C::BS;
#pragma unroll
                    for (int e = 0; e < C::BS / 32; ++e) {
                        const int q = i * C::BS + e * 32 + lane;
                        float nl = -INFINITY, dd = 0.f;
                        if (q < n) {
                            const size_t idx = rowstat_index(p.g, s, h, sp.start, q);
                            nl = -p.lse[idx] * kLog2e;
                            dd = p.dsum[idx];
                        }
                        vs[e * 32 + lane] = nl;
                        vs[C::BS + e * 32 + lane] = dd;
                    }
                    __threadfence_block();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_expect_tx(br.stage_full + slot, 2 * C::STR_BYTES);
                        uint8_t* st = smem + C::OFF_ST + slot * 2 * C::STR_BYTES;
                        for (int b = 0; b < C::NBOX; ++b) {
                            tma_load_3d(st + b * C::SBOX, &tm_q, br.stage_full + slot, b * 64, h,
                                        sp.start + i * C::BS);
                            tma_load_3d(st + C::STR_BYTES + b * C::SBOX, &tm_do, br.stage_full + slot,
                                        b * 64, h, sp.start + i * C::BS);
                        }
                    }
                }
            }
            if (!ok && lane == 0) {
                for (uint32_t x = cnt > C::NSTAGE ? cnt - C::NSTAGE : 0; x < cnt; ++x)
                    drain_wait(br.stage_full + x % C::NSTAGE, (x / C::NSTAGE) & 1, p.error_word);
                if (fix_issued) drain_wait(br.fix_full, (fix_issued - 1) & 1, p.error_word);
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA --
            constexpr uint32_t IDESC_S = idesc_bf16(128, C::BS, false, false);
            constexpr uint32_t IDESC_ACC = idesc_bf16(128, D, false, true);
            const uint32_t fa_addr = smem_u32(smem + C::OFF_FA);
            const uint32_t fb_addr = smem_u32(smem + C::OFF_FB);
            const uint32_t st_addr = smem_u32(smem + C::OFF_ST);
            uint32_t cnt = 0, item_it = 0;
            bool ok = true;
            auto issue_scores = [&](int b, uint32_t slot) {
                const uint32_t x = st_addr + slot * 2 * C::STR_BYTES;
                issue_ss_pair<D>(tmem + C::col_s(b), fa_addr, x, IDESC_S);              // K Q^T
                issue_ss_pair<D>(tmem + C::col_dp(b), fb_addr, x + C::STR_BYTES, IDESC_S); // V dO^T
                umma_commit(br.s_full + b);
            };
            for (int w = blockIdx.x; w < sch.total_items && ok; w += gridDim.x, ++item_it) {
                int s, h, blk;
                sch.item(w, s, h, blk);
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int k0 = blk * C::BM;
                int ib, ie;
                query_tile_range(k0, min(n, k0 + C::BM), n, p.g.causal, p.g.window, C::BS, ib, ie);
                if (!mbar_wait(br.fix_full, item_it & 1, wc)) { ok = false; break; }
                if (!mbar_wait(br.acc_empty, (item_it & 1) ^ 1, wc)) { ok = false; break; }
                if (!mbar_wait(br.stage_full + cnt % C::NSTAGE, (cnt / C::NSTAGE) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_scores(cnt & 1, cnt % C::NSTAGE);
                for (int i = ib; i < ie; ++i, ++cnt) {
                    const int b = cnt & 1;
                    const bool last = (i + 1 == ie);
                    const uint32_t slot = cnt % C::NSTAGE;
                    if (!last) {
                        const uint32_t nslot = (cnt + 1) % C::NSTAGE;
                        if (!mbar_wait(br.stage_full + nslot, ((cnt + 1) / C::NSTAGE) & 1, wc)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_scores(b ^ 1, nslot);
                    }
                    if (!mbar_wait(br.ready + b, (cnt >> 1) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t x = st_addr + slot * 2 * C::STR_BYTES;
                    issue_ts_acc<D>(tmem + C::COL_ACC1, tmem + C::col_s(b), x + C::STR_BYTES, IDESC_ACC,
                                    i > ib);                                          // dV += P^T dO
                    issue_ts_acc<D>(tmem + C::COL_ACC0, tmem + C::col_dp(b), x, IDESC_ACC,
                                    i > ib);                                          // dK += dS^T Q
                    umma_commit(br.stage_empty + slot);
                    if (last) {
                        umma_commit(br.acc_final);
                        umma_commit(br.fix_empty);
                    }
                }
            }
            if (!ok) {
                umma_commit(br.drain);
                drain_wait(br.drain, 0, p.error_word);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------ element-wise warpgroups --
        regs_alloc<200>();
        const int g = (warp >> 2) - 1;
        const int wq = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const int row = wq * 32 + lane;
        const float sl2 = p.scale_log2;
        uint32_t cnt = 0, item_it = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < sch.total_items && ok; w += gridDim.x, ++item_it) {
            int s, h, blk;
            sch.item(w, s, h, blk);
            const SeqSpan sp = sch.span(s);
            const int n = sp.len;
            const int k0 = blk * C::BM;
            const int j = k0 + row;               // this thread's key
            int ib, ie;
            query_tile_range(k0, min(n, k0 + C::BM), n, p.g.causal, p.g.window, C::BS, ib, ie);
            for (int i = ib; i < ie; ++i, ++cnt) {
                const int b = cnt & 1;
                if (!mbar_wait(br.s_full + b, (cnt >> 1) & 1, wc)) { ok = false; break; }
                // The producer wrote this stage's row statistics with ordinary stores
                // before arriving on stage_full: wait on it too so they are visible.
                if (!mbar_wait(br.stage_full + cnt % C::NSTAGE, (cnt / C::NSTAGE) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // this warpgroup's half of the tile: queries q0 + 32g ... q0 + 32g + 31
                const float* vs = vec + (cnt % C::NSTAGE) * 2 * C::BS + 32 * g;
                const int q0 = i * C::BS + 32 * g;
                const bool need_mask = (k0 + C::BM > n) || (p.g.causal && k0 + C::BM - 1 > q0) ||
                                       (p.g.window > 0 && q0 + 31 - k0 >= p.g.window);
                const uint32_t tS = tmem + lane_base + C::col_s(b) + 32 * g;
                const uint32_t tP = tmem + lane_base + C::col_dp(b) + 32 * g;
                uint32_t sr[32], dr[32];
                tmem_ld32(tS, sr);
                tmem_ld32(tP, dr);
                tmem_wait_ld();
                uint32_t pp[16], dd[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float pv[2], dv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int col = e + u;
                        float pr = ex2(fmaf(__uint_as_float(sr[col]), sl2, vs[col]));
                        if (need_mask && !key_allowed(q0 + col, j, n, p.g.causal, p.g.window))
                            pr = 0.f;
                        pv[u] = pr;
                        dv[u] = pr * (__uint_as_float(dr[col]) - vs[C::BS + col]);
                    }
                    pp[e / 2] = pack_bf16(pv[0], pv[1]);
                    dd[e / 2] = pack_bf16(dv[0], dv[1]);
                }
                tmem_st16(tS, pp);     // P^T packed over the first 16 columns of this half
                tmem_st16(tP, dd);     // dS^T likewise in the dP^T half
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(br.ready + b);
            }
            if (!ok) break;
            // ------------------------------------------------ epilogue --
            if (!mbar_wait(br.acc_final, item_it & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool valid = j < n;
            const size_t off = (static_cast<size_t>(sp.start) + j) * H * D + static_cast<size_t>(h) * D;
            if (g == 0) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c)
                    store_row_chunk(tmem + lane_base + C::COL_ACC1 + c * 32, 1.f, p.out1 + off + c * 32,
                                    valid);
            } else {
#pragma unroll
                for (int c = 0; c < D / 32; ++c)
                    store_row_chunk(tmem + lane_base + C::COL_ACC0 + c * 32, p.scale,
                                    p.out0 + off + c * 32, valid);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(br.acc_empty);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------- dQ kernel --
template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
          const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const BwdBarriers br = carve_barriers<D>(smem);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    int* scratch = reinterpret_cast<int*>(smem + C::OFF_SCRATCH);
    int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();

    if (threadIdx.x == 0) init_barriers<D>(br, abort_flag);
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_do);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    Schedule sch;
    sch.g = p.g;
    sch.rows_per_item = C::BM;
    sch.heavy_first = p.g.causal;   // the last query block sees the most keys
    sch.prefix = prefix;
    sch.total_items = build_schedule_prefix(p.g, C::BM, prefix, scratch);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtl wc{abort_flag, p.error_word, p.timeout_ns};
    const int H = p.g.H;

    if (warp < 4) {
        regs_dealloc<104>();
        if (warp == 0 && lane == 0) {
            // -------------------------------------------------- producer --
            uint32_t cnt = 0, item_it = 0, fix_issued = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < sch.total_items && ok; w += gridDim.x, ++item_it) {
                int s, h, blk;
                sch.item(w, s, h, blk);
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int q0 = blk * C::BM;
                int jb, je;
                key_tile_range(q0, min(n, q0 + C::BM), n, p.g.causal, p.g.window, C::BS, jb, je);
                if (!mbar_wait(br.fix_empty, (item_it & 1) ^ 1, wc)) { ok = false; break; }
                mbar_arrive_expect_tx(br.fix_full, 2 * C::FIX_BYTES);
                for (int b = 0; b < C::NBOX; ++b) {
                    tma_load_3d(smem + C::OFF_FA + b * C::FBOX, &tm_q, br.fix_full, b * 64, h,
                                sp.start + q0);
                    tma_load_3d(smem + C::OFF_FB + b * C::FBOX, &tm_do, br.fix_full, b * 64, h,
                                sp.start + q0);
                }
                ++fix_issued;
                for (int j = jb; j < je; ++j, ++cnt) {
                    const int slot = cnt % C::NSTAGE;
                    if (!mbar_wait(br.stage_empty + slot, ((cnt / C::NSTAGE) & 1) ^ 1, wc)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(br.stage_full + slot, 2 * C::STR_BYTES);
                    uint8_t* st = smem + C::OFF_ST + slot * 2 * C::STR_BYTES;
                    for (int b = 0; b < C::NBOX; ++b) {
                        tma_load_3d(st + b * C::SBOX, &tm_k, br.stage_full + slot, b * 64, h,
                                    sp.start + j * C::BS);
                        tma_load_3d(st + C::STR_BYTES + b * C::SBOX, &tm_v, br.stage_full + slot,
                                    b * 64, h, sp.start + j * C::BS);
                    }
                }
            }
            if (!ok) {
                for (uint32_t x = cnt > C::NSTAGE ? cnt - C::NSTAGE : 0; x < cnt; ++x)
                    drain_wait(br.stage_full + x % C::NSTAGE, (x / C::NSTAGE) & 1, p.error_word);
                if (fix_issued) drain_wait(br.fix_full, (fix_issued - 1) & 1, p.error_word);
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA --
            constexpr uint32_t IDESC_S = idesc_bf16(128, C::BS, false, false);
            constexpr uint32_t IDESC_ACC = idesc_bf16(128, D, false, true);
            const uint32_t fa_addr = smem_u32(smem + C::OFF_FA);
            const uint32_t fb_addr = smem_u32(smem + C::OFF_FB);
            const uint32_t st_addr = smem_u32(smem + C::OFF_ST);
            uint32_t cnt = 0, item_it = 0;
            bool ok = true;
            auto issue_scores = [&](int b, uint32_t slot) {
                const uint32_t x = st_addr + slot * 2 * C::STR_BYTES;
                issue_ss_pair<D>(tmem + C::col_s(b), fa_addr, x, IDESC_S);              // Q K^T
                issue_ss_pair<D>(tmem + C::col_dp(b), fb_addr, x + C::STR_BYTES, IDESC_S); // dO V^T
                umma_commit(br.s_full + b);
            };
            for (int w = blockIdx.x; w < sch.total_items && ok; w += gridDim.x, ++item_it) {
                int s, h, blk;
                sch.item(w, s, h, blk);
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int q0 = blk * C::BM;
                int jb, je;
                key_tile_range(q0, min(n, q0 + C::BM), n, p.g.causal, p.g.window, C::BS, jb, je);
                if (!mbar_wait(br.fix_full, item_it & 1, wc)) { ok = false; break; }
                if (!mbar_wait(br.acc_empty, (item_it & 1) ^ 1, wc)) { ok = false; break; }
                if (!mbar_wait(br.stage_full + cnt % C::NSTAGE, (cnt / C::NSTAGE) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_scores(cnt & 1, cnt % C::NSTAGE);
                for (int j = jb; j < je; ++j, ++cnt) {
                    const int b = cnt & 1;
                    const bool last = (j + 1 == je);
                    const uint32_t slot = cnt % C::NSTAGE;
                    if (!last) {
                        const uint32_t nslot = (cnt + 1) % C::NSTAGE;
                        if (!mbar_wait(br.stage_full + nslot, ((cnt + 1) / C::NSTAGE) & 1, wc)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_scores(b ^ 1, nslot);
                    }
                    if (!mbar_wait(br.ready + b, (cnt >> 1) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t x = st_addr + slot * 2 * C::STR_BYTES;
                    issue_ts_acc<D>(tmem + C::COL_ACC0, tmem + C::col_dp(b), x, IDESC_ACC,
                                    j > jb);                                          // dQ += dS K
                    umma_commit(br.stage_empty + slot);
                    if (last) {
                        umma_commit(br.acc_final);
                        umma_commit(br.fix_empty);
                    }
                }
            }
            if (!ok) {
                umma_commit(br.drain);
                drain_wait(br.drain, 0, p.error_word);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------ element-wise warpgroups --
        regs_alloc<200>();
        const int g = (warp >> 2) - 1;
        const int wq = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const int row = wq * 32 + lane;
        const float sl2 = p.scale_log2;
        uint32_t cnt = 0, item_it = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < sch.total_items && ok; w += gridDim.x, ++item_it) {
            int s, h, blk;
            sch.item(w, s, h, blk);
            const SeqSpan sp = sch.span(s);
            const int n = sp.len;
            const int q0 = blk * C::BM;
            const int q = q0 + row;               // this thread's query row
            int jb, je;
            key_tile_range(q0, min(n, q0 + C::BM), n, p.g.causal, p.g.window, C::BS, jb, je);
            float nl = -INFINITY, dq_d = 0.f;
            if (q < n) {
                const size_t idx = rowstat_index(p.g, s, h, sp.start, q);
                nl = -p.lse[idx] * kLog2e;
                dq_d = p.dsum[idx];
            }
            for (int j = jb; j < je; ++j, ++cnt) {
                const int b = cnt & 1;
                if (!mbar_wait(br.s_full + b, (cnt >> 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                // this warpgroup's half of the tile: keys kb ... kb + 31
                const int kb = j * C::BS + 32 * g;
                const bool need_mask = tile_needs_mask(q0, C::BM, kb, 32, n, p.g.causal, p.g.window);
                const uint32_t tS = tmem + lane_base + C::col_s(b) + 32 * g;
                const uint32_t tP = tmem + lane_base + C::col_dp(b) + 32 * g;
                uint32_t sr[32], dr[32];
                tmem_ld32(tS, sr);
                tmem_ld32(tP, dr);
                tmem_wait_ld();
                uint32_t dd[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float dv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int col = e + u;
                        float pr = ex2(fmaf(__uint_as_float(sr[col]), sl2, nl));
                        if (need_mask && !key_allowed(q, kb + col, n, p.g.causal, p.g.window))
                            pr = 0.f;
                        dv[u] = pr * (__uint_as_float(dr[col]) - dq_d);
                    }
                    dd[e / 2] = pack_bf16(dv[0], dv[1]);
                }
                tmem_st16(tP, dd);     // dS packed over the first 16 columns of this half
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(br.ready + b);
            }
            if (!ok) break;
            // ------------------------------------------------ epilogue --
            if (!mbar_wait(br.acc_final, item_it & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool valid = q < n;
            const size_t off = (static_cast<size_t>(sp.start) + q) * H * D + static_cast<size_t>(h) * D;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                const int col = g * (D / 2) + c * 32;
                store_row_chunk(tmem + lane_base + C::COL_ACC0 + col, p.scale, p.out0 + off + col, valid);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(br.acc_empty);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------ host side --
struct BwdMaps {
    CUtensorMap q64, do64, k128, v128;   // dK/dV kernel
    CUtensorMap q128, do128, k64, v64;   // dQ kernel
};

struct BwdArgs {
    Geometry g;
    int d;
    const void *o, *dO;
    const float* lse;
    void *dq, *dk, *dv;
    float* dsum;
    float scale;
    int num_sms;
    int* error_word;
    uint64_t timeout_ns;
};

inline size_t bwd_workspace_bytes(int64_t rows, int H) {
    return static_cast<size_t>((rows * H * 4 + 255) / 256 * 256);
}

inline cudaError_t bwd_set_smem_limits() {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(dkdv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BwdCfg<64>::SMEM_BYTES)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(dkdv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BwdCfg<128>::SMEM_BYTES)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BwdCfg<64>::SMEM_BYTES)) != cudaSuccess)
        return e;
    return cudaFuncSetAttribute(dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BwdCfg<128>::SMEM_BYTES);
}

// Optional timing callbacks around each launch (kind 1 = D pre-pass,
// 2 = dK/dV, 3 = dQ): start returns a slot that stop closes.
struct BwdHooks {
    int (*start)(int kind, cudaStream_t stream);
    void (*stop)(int kind, int slot, cudaStream_t stream);
};

template <int D>
cudaError_t bwd_launch_d(const BwdArgs& a, const BwdMaps& m, cudaStream_t stream,
                         const BwdHooks& hk) {
    using C = BwdCfg<D>;
    {
        const int slot = hk.start(1, stream);
        const int64_t rows = static_cast<int64_t>(a.g.T) * a.g.H;
        const int rows_per_block = 8 * (32 / (D / 8));
        int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
        const int64_t cap = static_cast<int64_t>(a.num_sms) * 8;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        dot_kernel<D><<<static_cast<int>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a.dO), static_cast<const __nv_bfloat16*>(a.o),
            a.dsum, a.g);
        hk.stop(1, slot, stream);
    }
    BwdParams p;
    p.g = a.g;
    p.lse = a.lse;
    p.dsum = a.dsum;
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    p.error_word = a.error_word;
    p.timeout_ns = a.timeout_ns;
    int grid = a.num_sms;
    if (!a.g.cu_seqlens) {
        const int64_t items = static_cast<int64_t>(a.g.B) * a.g.H * ((a.g.N + C::BM - 1) / C::BM);
        if (items < grid) grid = static_cast<int>(items);
    }
    p.out0 = static_cast<__nv_bfloat16*>(a.dk);
    p.out1 = static_cast<__nv_bfloat16*>(a.dv);
    int slot = hk.start(2, stream);
    dkdv_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(m.k128, m.v128, m.q64, m.do64, p);
    hk.stop(2, slot, stream);
    p.out0 = static_cast<__nv_bfloat16*>(a.dq);
    p.out1 = nullptr;
    slot = hk.start(3, stream);
    dq_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(m.q128, m.do128, m.k64, m.v64, p);
    hk.stop(3, slot, stream);
    return cudaGetLastError();
}

inline cudaError_t bwd_launch(const BwdArgs& a, const BwdMaps& m, cudaStream_t stream,
                              const BwdHooks& hk) {
    return a.d == 64 ? bwd_launch_d<64>(a, m, stream, hk) : bwd_launch_d<128>(a, m, stream, hk);
}

}  // namespace fa
