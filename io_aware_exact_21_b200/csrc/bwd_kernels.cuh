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
//   1. stats_kernel: D_i = rowsum(dO_i * O_i) in fp32 (one row per group of
//      d/8 lanes reading 16-byte vectors, reduced with warp shuffles), stored
//      with -LSE_i log2(e) in a 128-row padded layout.
//   2. dkdv_kernel: a CTA owns 128 keys of one (sequence, head) and streams
//      the 128-row query tiles that can see them.  Per query tile:
//        S^T = K Q^T and dP^T = V dO^T        (tcgen05, both operands in smem)
//        P^T = 2^(S^T scale log2e - L log2e), dS^T = P^T (dP^T - D)   (fp32)
//        dV += P^T dO and dK += dS^T Q        (tcgen05, P^T / dS^T from TMEM)
//   3. dq_kernel  : a CTA owns 128 queries and streams 128-key tiles:
//        S = Q K^T, dP = dO V^T, P, dS as above, dQ += dS K.
// Every GEMM is 128 x 128 (x 128): on sm_100a an MMA with N = 64 costs as
// much tensor time as one with N = 128, so 64-wide score tiles would run the
// tensor core at half rate.  Both big kernels use the forward's role split
// (TMA warp, MMA warp, two element-wise warpgroups, each taking one 64-column
// half of every score tile).  The score tiles are single-buffered in TMEM
// (dK, dV or dQ take the other columns) and the element-wise warps release
// their results in two steps -- P first (the dV GEMM and the next S^T start),
// dS second -- so GEMMs and element-wise work overlap.  Deterministic: no
// atomics.
#pragma once

#include "schedule.cuh"
#include "dead_rows.cuh"
#include "sm100.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;

// Per-row statistics the two gradient kernels read, written by the pre-pass
// into the workspace: x_i = -LSE_i * log2(e) and y_i = -D_i for each
// (sequence, head, row), in a layout padded to 128-row blocks so that a
// streamed tile's statistics are one aligned 1 KB bulk copy, and split within
// each block (its 128 x values, then its 128 y values) so that consecutive
// rows' values sit next to each other for packed float32x2 arithmetic.  Row i
// of a (sequence, head) whose rows start at row index R (a multiple of 128):
//   fixed length: R = (s * H + h) * stride,           stride = N rounded up to 128
//   packed:       R = h * stride + 128 * blocks(s),    blocks(s) = sum over earlier
//                 sequences of ceil(len / 128), stride >= 128 * blocks(B)
//   x at float 2 (R + i - i % 128) + i % 128, y 128 floats further.
// Entries of padding rows are never written; readers mask them.
struct BwdParams {
    Geometry g;
    const float* stats;
    int64_t stats_stride;
    const __nv_bfloat16* qrows;   // Q and dO (the dQ kernel reads its own rows directly)
    const __nv_bfloat16* dorows;
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

// Float index of x for row i of sequence s, head h in the padded statistics
// array (y is 128 floats further); `blocks_before` = 128-row blocks of the
// sequences before s (packed only).  For i a multiple of 128 it is the start
// of that block's 1 KB.
__device__ __forceinline__ size_t stats_index(const Geometry& g, int64_t stride, int s, int h,
                                              int blocks_before, int i) {
    const size_t R = g.cu_seqlens ? static_cast<size_t>(h) * stride + static_cast<size_t>(blocks_before) * 128
                                  : (static_cast<size_t>(s) * g.H + h) * stride;
    return 2 * (R + (i & ~127)) + (i & 127);
}

// ------------------------------------------------------------ pre-pass --
// stats[row] = {-LSE * log2(e), D = rowsum(dO * O)}: each warp takes 32 rows
// in the LSE array's order (so their LSE reads and statistics writes are
// whole lines); a row's dO and O are read by a group of d/8 lanes in 16-byte
// vectors and the dot product is reduced with warp shuffles.  Packed
// batches: each CTA first builds the per-sequence block prefix and a copy of
// cu_seqlens in shared memory to place each token.
// With dq_acc non-null (the fused backward) it also zeroes that fp32 [rows, d]
// accumulator, row by row.
constexpr int kStatsUnroll = 4;        // load steps a warp has in flight
constexpr int kStatsCtasPerSm = 4;     // 256-thread CTAs resident per SM (64 registers)

template <int D>
__global__ void __launch_bounds__(256, kStatsCtasPerSm)
stats_kernel(const __nv_bfloat16* __restrict__ dO, const __nv_bfloat16* __restrict__ O,
             const float* __restrict__ lse, float* __restrict__ stats, int64_t stride,
             Geometry g, float* __restrict__ dq_acc) {
    constexpr int LPR = D / 8;                 // lanes per row (16-byte vectors)
    constexpr int RPW = 32 / LPR;              // rows per warp per iteration
    extern __shared__ int pre_smem[];
    int* prefix = pre_smem;                    // B + 1 block prefix (packed only)
    int* uprefix = prefix + kMaxVarlenSeqs + 1;
    int* cu = uprefix + kMaxVarlenSeqs + 1;    // B + 1
    int* scratch = cu + kMaxVarlenSeqs + 1;    // 2 * blockDim
    if (g.cu_seqlens) {
        for (int i = threadIdx.x; i <= g.B; i += blockDim.x) cu[i] = g.cu_seqlens[i];
        build_schedule_prefix(g, 128, prefix, uprefix, scratch, false);   // __syncthreads inside
    }
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR;
    const int part = lane % LPR;
    const int64_t rows = static_cast<int64_t>(g.T) * g.H;
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const bool narrow = rows <= 0x7fffffff;    // row numbers fit 32-bit division
    // Rows are walked in the LSE array's own order -- r = (s * H + h) * N + i
    // for fixed length, h * T + token for packed batches -- 32 per warp, so
    // the warp reads its 32 LSE values and writes its 32 statistics pairs as
    // whole lines (consecutive rows of one (sequence, head)); each row's dO
    // and O are read by d / 8 lanes in 16-byte vectors, RPW rows per load
    // step, kStatsUnroll steps' loads in flight.
    for (int64_t base = warp_global * 32; base < rows; base += nwarps * 32) {
        // this lane's row: its place, its LSE, and its token row in dO / O
        const int64_t r = base + lane;
        bool out = false;
        float l = 0.f;
        size_t xi = 0;
        long long src = -1;                     // (token * H + h), or -1: no row
        if (r < rows) {
            if (g.cu_seqlens) {
                int h, token;
                if (narrow) {
                    const uint32_t h32 = static_cast<uint32_t>(r) / static_cast<uint32_t>(g.T);
                    h = static_cast<int>(h32);
                    token = static_cast<int>(static_cast<uint32_t>(r) - h32 * static_cast<uint32_t>(g.T));
                } else {
                    h = static_cast<int>(r / g.T);
                    token = static_cast<int>(r - static_cast<int64_t>(h) * g.T);
                }
                src = static_cast<long long>(token) * g.H + h;
                if (token < cu[g.B]) {                 // else a row outside every sequence
                    int lo = 0, hi = g.B - 1;          // last s with cu[s] <= token
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (cu[mid] <= token) lo = mid; else hi = mid - 1;
                    }
                    out = true;
                    xi = stats_index(g, stride, lo, h, prefix[lo], token - cu[lo]);
                }
            } else {
                int64_t sh;
                int i;
                if (narrow) {
                    const uint32_t sh32 = static_cast<uint32_t>(r) / static_cast<uint32_t>(g.N);
                    sh = sh32;
                    i = static_cast<int>(static_cast<uint32_t>(r) - sh32 * static_cast<uint32_t>(g.N));
                } else {
                    sh = r / g.N;
                    i = static_cast<int>(r - sh * g.N);
                }
                const int s_ = static_cast<int>(sh / g.H);
                const int h = static_cast<int>(sh - static_cast<int64_t>(s_) * g.H);
                src = (static_cast<long long>(s_) * g.N + i) * g.H + h;
                out = true;
                xi = stats_index(g, stride, s_, h, 0, i);
            }
            l = lse[r];
        }
        float dsum = 0.f;                       // D of this lane's row, once gathered
#pragma unroll 1
        for (int k0 = 0; k0 < 32 / RPW; k0 += kStatsUnroll) {
            uint4 a[kStatsUnroll], b[kStatsUnroll];
#pragma unroll
            for (int u = 0; u < kStatsUnroll; ++u) {
                const long long rs = __shfl_sync(0xffffffffu, src, (k0 + u) * RPW + sub);
                a[u] = make_uint4(0u, 0u, 0u, 0u);
                b[u] = make_uint4(0u, 0u, 0u, 0u);
                if (rs >= 0) {
                    a[u] = *reinterpret_cast<const uint4*>(dO + rs * D + part * 8);
                    b[u] = *reinterpret_cast<const uint4*>(O + rs * D + part * 8);
                    if (dq_acc) {
                        float4* z = reinterpret_cast<float4*>(dq_acc + rs * D + part * 8);
                        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
                        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kStatsUnroll; ++u) {
                float acc = 0.f;
                const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
                const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b[u]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 fa2 = __bfloat1622float2(pa[e]);
                    const float2 fb2 = __bfloat1622float2(pb[e]);
                    acc = fmaf(fa2.x, fb2.x, acc);
                    acc = fmaf(fa2.y, fb2.y, acc);
                }
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                // every lane of group q now holds row (k0 + u) * RPW + q's D
#pragma unroll
                for (int q = 0; q < RPW; ++q) {
                    const float t = __shfl_sync(0xffffffffu, acc, q * LPR);
                    if (lane == (k0 + u) * RPW + q) dsum = t;
                }
            }
        }
        if (out) {
            stats[xi] = -l * 1.4426950408889634f;
            stats[xi + 128] = -dsum;
        }
    }
}

// --------------------------------------------------- shared configuration --
template <int D>
struct BwdCfg {
    static constexpr int BM = 128;               // rows the CTA owns (keys or queries)
    static constexpr int BS = 128;               // rows streamed per step
    static constexpr int NSTAGE = 2;
    static constexpr int NBOX = D / 64;
    static constexpr int BOX = 128 * 128;        // one TMA box: 128 rows x 128 B
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int THREADS = 384;
    // TMEM columns: accumulators, then the score tile and its gradient tile
    static constexpr uint32_t COL_ACC0 = 0, COL_ACC1 = 128, COL_S = 256, COL_DP = 384;
    static constexpr int OFF_FA = 0;                               // fixed tile A (K or Q)
    static constexpr int OFF_FB = TILE_BYTES;                      // fixed tile B (V or dO)
    static constexpr int OFF_ST = 2 * TILE_BYTES;                  // stages: X then Y
    static constexpr int OFF_VEC = OFF_ST + NSTAGE * 2 * TILE_BYTES;  // stage stats: float2[BS]
    static constexpr int VEC_BYTES = BS * 8;
    static constexpr int OFF_BAR = OFF_VEC + NSTAGE * VEC_BYTES;
    static constexpr int NBAR = 2 + 2 * NSTAGE + 6 + 2 + 1 + NSTAGE;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_SCRATCH = OFF_MISC + 16;
    static constexpr int OFF_PREFIX = OFF_SCRATCH + 2 * THREADS * 4;   // block and unit prefixes
    // block prefix, unit prefix, then the rank order (short[kMaxSortedSeqs])
    static constexpr int SMEM_BYTES = OFF_PREFIX + 2 * (kMaxVarlenSeqs + 1) * 4 + kMaxSortedSeqs * 2 + 1024;
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

// Barriers.  s_full / dp_full: the score GEMM and the gradient GEMM of a step
// have completed.  mid: the element-wise warps are done with the first half
// of their work (dK/dV kernel: P^T written, in two parts; dQ kernel: S read,
// part 0 only).  ready: dS written, in two parts.  A part is the first or the
// second 32 columns of each warpgroup's 64-column half, so the accumulating
// GEMM can start on part 0 while part 1 is computed.  Each barrier completes
// once per step, so its parity is the step count's.
struct BwdBarriers {
    uint64_t *fix_full, *fix_empty, *stage_full, *stage_empty, *s_full, *dp_full, *mid, *ready,
        *acc_final, *acc_empty, *drain, *land;
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
    r.dp_full = r.s_full + 1;
    r.mid = r.dp_full + 1;          // [2 parts]
    r.ready = r.mid + 2;            // [2 parts]
    r.acc_final = r.ready + 2;
    r.acc_empty = r.acc_final + 1;
    r.drain = r.acc_empty + 1;
    r.land = r.drain + 1;           // [NSTAGE]: stages with rows past a packed batch
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
    mbar_init(br.s_full, 1);
    mbar_init(br.dp_full, 1);
    for (int part = 0; part < 2; ++part) {
        mbar_init(br.mid + part, 8);    // all eight element-wise warps
        mbar_init(br.ready + part, 8);
    }
    mbar_init(br.acc_final, 1);
    mbar_init(br.acc_empty, 8);
    mbar_init(br.drain, 1);
    for (int s = 0; s < C::NSTAGE; ++s) mbar_init(br.land + s, 1);
    *abort_flag = 0;
    fence_barrier_init();
}

// D[128 x 128] = A[smem 128 x d, K-major] * B[smem 128 x d, K-major]^T.
// k-step kk covers channels 16kk..16kk+15: 32 bytes inside the 128-byte
// swizzled rows, the next 64-channel box after four steps.
template <int D>
__device__ __forceinline__ void issue_scores_ss(uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
    using C = BwdCfg<D>;
    constexpr uint32_t IDESC = idesc_bf16(128, C::BS, false, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
        umma_ss(d_tmem, sw128_desc(a_base + off, 16, 1024), sw128_desc(b_base + off, 16, 1024),
                IDESC, kk > 0);
    }
}

// Column of the packed bf16 operand for 16-row k-step kk: each element-wise
// warpgroup packs its 64-column half h of a score tile into the first 32 of
// that half's columns (h * 64 ... h * 64 + 31), which it has already read.
__host__ __device__ constexpr uint32_t packed_col(int kk) { return (kk >> 2) * 64 + (kk & 3) * 8; }

// acc[128 x D] (+)= A[tmem, rows of `part`, bf16 packed] * B[smem, same rows, MN-major]:
// part 0 covers k-steps {0, 1, 4, 5} (streamed rows 0-31 and 64-95), part 1
// covers {2, 3, 6, 7}.  `accumulate` false only for the first part of a tile's
// first step.
template <int D>
__device__ __forceinline__ void issue_acc_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base,
                                             bool accumulate, int part) {
    constexpr uint32_t IDESC = idesc_bf16(128, D, false, true);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int kk = (i >> 1) * 4 + part * 2 + (i & 1);
        umma_ts(d_tmem, a_tmem + packed_col(kk), sw128_desc(b_base + kk * 2048, BwdCfg<D>::BOX, 1024),
                IDESC, (accumulate || i > 0) ? 1u : 0u);
    }
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

// Load 64 consecutive TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}

__device__ __forceinline__ void arrive_warp(uint64_t* bar) {
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane_id() == 0) mbar_arrive(bar);
}

// Common prologue of both big kernels: barriers, TMEM, schedule.
template <int D>
__device__ __forceinline__ uint32_t bwd_prologue(uint8_t* smem, const BwdBarriers& br,
                                                 volatile int* abort_flag, const BwdParams& p,
                                                 Schedule& sch,
                                                 const CUtensorMap* maps[4]) {
    using C = BwdCfg<D>;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    int* scratch = reinterpret_cast<int*>(smem + C::OFF_SCRATCH);
    int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) init_barriers<D>(br, abort_flag);
    if (warp == 0 && lane_id() == 0)
        for (int i = 0; i < 4; ++i) tma_prefetch_map(maps[i]);
    if (warp == 1) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    sch.g = p.g;
    sch.rows_per_item = C::BM;
    sch.order = schedule_order(p.g, 0);     // key blocks: fewer queries see later keys
    sch.bprefix = prefix;
    sch.uprefix = prefix + kMaxVarlenSeqs + 1;
    sch.total_units = build_schedule_prefix(p.g, C::BM, prefix, prefix + kMaxVarlenSeqs + 1,
                                            scratch);   // __syncthreads inside
    schedule_split_tail(sch);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *tmem_holder;
}

template <int D>
__device__ __forceinline__ void bwd_epilogue_sync(uint32_t tmem) {
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
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
    uint8_t* smem = align_smem_1024(smem_raw);
    const BwdBarriers br = carve_barriers<D>(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    float* vec = reinterpret_cast<float*>(smem + C::OFF_VEC);   // per stage: x[128], y[128]
    const CUtensorMap* maps[4] = {&tm_k, &tm_v, &tm_q, &tm_do};
    Schedule sch;
    const uint32_t tmem = bwd_prologue<D>(smem, br, abort_flag, p, sch, maps);
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();
    const WaitCtl wc{abort_flag, p.error_word, p.timeout_ns};
    const int H = p.g.H;

    if (warp < 4) {
        regs_dealloc<104>();
        if (warp == 0) {
            // ---------------------------------- producer (whole warp) --
            uint32_t cnt = 0, item_it = 0, fix_issued = 0;
            LandTrack lt;
            bool ok = true;
            ItemIter<true> it;
            int s, h, blk;
            for (; ok && it.next(sch, s, h, blk); ++item_it) {
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int k0 = blk * C::BM;
                int ib, ie;
                query_tile_range(k0, min(n, k0 + C::BM), n, p.g.causal, p.g.window, C::BS, ib, ie);
                if (lane == 0) {
                    ok = mbar_wait(br.fix_empty, (item_it & 1) ^ 1, wc);
                    if (ok) {
                        mbar_arrive_expect_tx(br.fix_full, 2 * C::TILE_BYTES);
                        for (int b = 0; b < C::NBOX; ++b) {
                            tma_load_3d(smem + C::OFF_FA + b * C::BOX, &tm_k, br.fix_full, b * 64, h,
                                        sp.start + k0);
                            tma_load_3d(smem + C::OFF_FB + b * C::BOX, &tm_v, br.fix_full, b * 64, h,
                                        sp.start + k0);
                        }
                        ++fix_issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                const int blocks_before = sch.blocks_before(s);
                // packed batches: the first row of the item's last query tile past
                // the batch's last sequence (128: none); that stage lands on
                // land[slot] for the fixer warp
                const int dead_r0 =
                    ie > ib ? first_dead_row(p.g.cu_seqlens, p.g.B, sp.start + (ie - 1) * C::BS) : 128;
                for (int i = ib; i < ie && ok; ++i, ++cnt) {
                    const int slot = cnt % C::NSTAGE;
                    if (lane == 0) {
                        ok = mbar_wait(br.stage_empty + slot, ((cnt / C::NSTAGE) & 1) ^ 1, wc);
                        if (ok) {
                            const bool to_land = i + 1 == ie && dead_r0 < 128;
                            uint64_t* full = to_land ? br.land + slot : br.stage_full + slot;
                            lt.note(slot, to_land);
                            mbar_arrive_expect_tx(full, 2 * C::TILE_BYTES + C::VEC_BYTES);
                            uint8_t* st = smem + C::OFF_ST + slot * 2 * C::TILE_BYTES;
                            for (int b = 0; b < C::NBOX; ++b) {
                                tma_load_3d(st + b * C::BOX, &tm_q, full, b * 64, h, sp.start + i * C::BS);
                                tma_load_3d(st + C::TILE_BYTES + b * C::BOX, &tm_do, full, b * 64, h,
                                            sp.start + i * C::BS);
                            }
                            // the tile's per-query statistics, one aligned 1 KB copy
                            bulk_load(vec + slot * 2 * C::BS,
                                      p.stats + stats_index(p.g, p.stats_stride, s, h, blocks_before,
                                                            i * C::BS),
                                      C::VEC_BYTES, full);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                }
            }
            if (!ok && lane == 0) {
                for (uint32_t x = cnt > C::NSTAGE ? cnt - C::NSTAGE : 0; x < cnt; ++x) {
                    const int sl = x % C::NSTAGE;
                    if (lt.landed(sl))
                        drain_wait(br.land + sl, lt.land_parity(sl), p.error_word);
                    else
                        drain_wait(br.stage_full + sl, (x / C::NSTAGE) & 1, p.error_word);
                }
                if (fix_issued) drain_wait(br.fix_full, (fix_issued - 1) & 1, p.error_word);
            }
        } else if (warp == 2) {
            // ------------------------------------------------------- fixer --
            // packed batches: zeroes the Q and dO rows past the batch's last
            // sequence in each stage the producer sent to land[slot] (they meet
            // dS = 0 and P = 0 in the dK and dV GEMMs), then releases the stage
            // on stage_full[slot]
            if (p.g.cu_seqlens) {
                uint32_t cnt = 0, land_par = 0;
                ItemIter<true> it;
                int s, h, blk;
                while (it.next(sch, s, h, blk)) {
                    const SeqSpan sp = sch.span(s);
                    const int n = sp.len;
                    const int k0 = blk * C::BM;
                    int ib, ie;
                    query_tile_range(k0, min(n, k0 + C::BM), n, p.g.causal, p.g.window, C::BS, ib, ie);
                    const int dead_r0 =
                        ie > ib ? first_dead_row(p.g.cu_seqlens, p.g.B, sp.start + (ie - 1) * C::BS) : 128;
                    if (dead_r0 < 128) {
                        const int slot = (cnt + (ie - 1 - ib)) % C::NSTAGE;
                        // every lane waits; the warp leaves together if any lane gave up
                        if (!__all_sync(0xffffffffu, mbar_wait(br.land + slot, (land_par >> slot) & 1u, wc))) break;
                        land_par ^= 1u << slot;
                        uint8_t* st = smem + C::OFF_ST + slot * 2 * C::TILE_BYTES;
                        zero_tile_rows(st, C::NBOX, dead_r0, lane, 32);
                        zero_tile_rows(st + C::TILE_BYTES, C::NBOX, dead_r0, lane, 32);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(br.stage_full + slot);
                    }
                    cnt += ie - ib;
                }
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA --
            // per step i:  S^T_i, dP^T_i  ->  [P^T_i written] dV += P^T_i dO_i, S^T_{i+1}
            //              ->  [dS^T_i written] dK += dS^T_i Q_i, dP^T_{i+1}
            const uint32_t fa_addr = smem_u32(smem + C::OFF_FA);
            const uint32_t fb_addr = smem_u32(smem + C::OFF_FB);
            const uint32_t st_addr = smem_u32(smem + C::OFF_ST);
            uint32_t cnt = 0, item_it = 0;
            bool ok = true;
            ItemIter<true> it;
            int s, h, blk;
            for (; ok && it.next(sch, s, h, blk); ++item_it) {
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int k0 = blk * C::BM;
                int ib, ie;
                query_tile_range(k0, min(n, k0 + C::BM), n, p.g.causal, p.g.window, C::BS, ib, ie);
                // the item's first S^T and dP^T do not touch the accumulators, so
                // they run while the element-wise warps still store the previous
                // item's dK and dV; the accumulators are awaited before the first dV
                if (!mbar_wait(br.fix_full, item_it & 1, wc)) { ok = false; break; }
                if (!mbar_wait(br.stage_full + cnt % C::NSTAGE, (cnt / C::NSTAGE) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                {
                    const uint32_t x = st_addr + (cnt % C::NSTAGE) * 2 * C::TILE_BYTES;
                    issue_scores_ss<D>(tmem + C::COL_S, fa_addr, x);                  // K Q^T
                    umma_commit(br.s_full);
                    issue_scores_ss<D>(tmem + C::COL_DP, fb_addr, x + C::TILE_BYTES);  // V dO^T
                    umma_commit(br.dp_full);
                    if (ib + 1 == ie) umma_commit(br.fix_empty);   // K and V read for the last time
                }
                if (!mbar_wait(br.acc_empty, (item_it & 1) ^ 1, wc)) { ok = false; break; }
                tc_fence_after();
                for (int i = ib; i < ie; ++i, ++cnt) {
                    const bool last = (i + 1 == ie);
                    const uint32_t slot = cnt % C::NSTAGE;
                    const uint32_t x = st_addr + slot * 2 * C::TILE_BYTES;
                    const uint32_t xn = st_addr + ((cnt + 1) % C::NSTAGE) * 2 * C::TILE_BYTES;
                    bool mok = true;
                    for (int part = 0; part < 2 && mok; ++part) {
                        if (!mbar_wait(br.mid + part, cnt & 1, wc)) { mok = false; break; }
                        tc_fence_after();
                        issue_acc_ts<D>(tmem + C::COL_ACC1, tmem + C::COL_S, x + C::TILE_BYTES,
                                        i > ib || part > 0, part);                      // dV
                    }
                    if (!mok) { ok = false; break; }
                    if (!last) {
                        if (!mbar_wait(br.stage_full + (cnt + 1) % C::NSTAGE, ((cnt + 1) / C::NSTAGE) & 1, wc)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_scores_ss<D>(tmem + C::COL_S, fa_addr, xn);             // next K Q^T
                        umma_commit(br.s_full);
                    }
                    for (int part = 0; part < 2 && mok; ++part) {
                        if (!mbar_wait(br.ready + part, cnt & 1, wc)) { mok = false; break; }
                        tc_fence_after();
                        issue_acc_ts<D>(tmem + C::COL_ACC0, tmem + C::COL_DP, x, i > ib || part > 0,
                                        part);                                          // dK
                    }
                    if (!mok) { ok = false; break; }
                    umma_commit(br.stage_empty + slot);
                    if (!last) {
                        issue_scores_ss<D>(tmem + C::COL_DP, fb_addr, xn + C::TILE_BYTES);  // next V dO^T
                        umma_commit(br.dp_full);
                        // K and V read for the last time: the producer may load the
                        // next item's while this one finishes
                        if (i + 2 == ie) umma_commit(br.fix_empty);
                    } else {
                        umma_commit(br.acc_final);
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
        const int g = (warp >> 2) - 1;             // 64-column half of each tile
        const int wq = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const int row = wq * 32 + lane;
        const float sl2 = p.scale_log2;
        const uint32_t tS = tmem + lane_base + C::COL_S + 64 * g;
        const uint32_t tP = tmem + lane_base + C::COL_DP + 64 * g;
        uint32_t cnt = 0, item_it = 0;
        bool ok = true;
        ItemIter<true> it;
        int s, h, blk;
        for (; ok && it.next(sch, s, h, blk); ++item_it) {
            const SeqSpan sp = sch.span(s);
            const int n = sp.len;
            const int k0 = blk * C::BM;
            const int j = k0 + row;               // this thread's key
            int ib, ie;
            query_tile_range(k0, min(n, k0 + C::BM), n, p.g.causal, p.g.window, C::BS, ib, ie);
            for (int i = ib; i < ie; ++i, ++cnt) {
                if (!mbar_wait(br.s_full, cnt & 1, wc)) { ok = false; break; }
                // The producer wrote this stage's row statistics with ordinary stores
                // before arriving on stage_full: wait on it too so they are visible.
                if (!mbar_wait(br.stage_full + cnt % C::NSTAGE, (cnt / C::NSTAGE) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float* xs = vec + (cnt % C::NSTAGE) * 2 * C::BS + 64 * g;   // -L log2e
                const float* ys = xs + C::BS;                                     // -D
                const int q0 = i * C::BS + 64 * g;     // this half's first query
                const bool need_mask = (k0 + C::BM > n) || (q0 + 64 > n) ||
                                       (p.g.causal && k0 + C::BM - 1 > q0) ||
                                       (p.g.window > 0 && q0 + 63 - k0 >= p.g.window);
                uint32_t r[64];
                tmem_ld64(tS, r);
                tmem_wait_ld();
                float pf[64];
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    if (!need_mask) {
                        // pairs of queries: the argument in packed float32x2
#pragma unroll
                        for (int c = 32 * part; c < 32 * part + 32; c += 2) {
                            const float2 a = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])),
                                                   make_float2(sl2, sl2),
                                                   *reinterpret_cast<const float2*>(xs + c));
                            pf[c] = ex2(a.x);
                            pf[c + 1] = ex2(a.y);
                        }
                    } else {
                        // masked pairs, and query rows past the sequence end (their
                        // statistics are padding), get P = 0: this key's allowed
                        // queries of the half are columns [c_lo, c_hi)
                        int c_lo, c_hi;
                        tile_query_bounds(j, q0, n, p.g.causal, p.g.window, 64, c_lo, c_hi);
#pragma unroll
                        for (int c = 32 * part; c < 32 * part + 32; ++c) {
                            const float x = ex2(fmaf(__uint_as_float(r[c]), sl2, xs[c]));
                            pf[c] = (c >= c_lo && c < c_hi) ? x : 0.f;
                        }
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        pk[c] = pack_bf16(pf[32 * part + 2 * c], pf[32 * part + 2 * c + 1]);
                    tmem_st16(tS + 16 * part, pk);   // P^T packed over the first 32 columns of this half
                    arrive_warp(br.mid + part);
                }
                if (!mbar_wait(br.dp_full, cnt & 1, wc)) { ok = false; break; }
                tc_fence_after();
                tmem_ld64(tP, r);
                tmem_wait_ld();
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t pk[16];
                    if (!need_mask) {
                        // dS = P (dP - D), pairs of queries in packed float32x2
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int k = 32 * part + 2 * c;
                            const float2 d = fmul2(make_float2(pf[k], pf[k + 1]),
                                                   fadd2(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])),
                                                         *reinterpret_cast<const float2*>(ys + k)));
                            pk[c] = pack_bf16(d.x, d.y);
                        }
                    } else {
                        // P = 0 must give dS = 0 even where the padding D is not finite
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int k = 32 * part + 2 * c;
                            const float d0 = pf[k] * (__uint_as_float(r[k]) + ys[k]);
                            const float d1 = pf[k + 1] * (__uint_as_float(r[k + 1]) + ys[k + 1]);
                            pk[c] = pack_bf16(pf[k] != 0.f ? d0 : 0.f, pf[k + 1] != 0.f ? d1 : 0.f);
                        }
                    }
                    tmem_st16(tP + 16 * part, pk);   // dS^T packed over the first 32 columns of this half
                    arrive_warp(br.ready + part);
                }
            }
            if (!ok) break;
            // ------------------------------------------------ epilogue --
            if (!mbar_wait(br.acc_final, item_it & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool valid = j < n;
            const size_t off = (static_cast<size_t>(sp.start) + j) * H * D + static_cast<size_t>(h) * D;
            if (g == 0) {
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    store_line_bf16(tmem + lane_base + C::COL_ACC1 + c * 64, 1.f, p.out1 + off + c * 64, valid);
            } else {
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    store_line_bf16(tmem + lane_base + C::COL_ACC0 + c * 64, p.scale, p.out0 + off + c * 64,
                                    valid);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(br.acc_empty);
        }
    }
    bwd_epilogue_sync<D>(tmem);
}

// ------------------------------------------------------------- dQ kernel --
// The CTA's own operands Q and dO live in TMEM (packed bf16, written by the
// element-wise warps straight from global memory), so the score GEMMs read
// their A operand from TMEM and all shared memory goes to a 3-deep ring of
// K/V tiles: a tile's refill then starts a step earlier than with two stages.
template <int D>
struct DqCfg {
    static constexpr int BM = 128;               // queries the CTA owns
    static constexpr int BS = 128;               // keys streamed per step
    static constexpr int NSTAGE = 3;
    static constexpr int NBOX = D / 64;
    static constexpr int BOX = 128 * 128;
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int THREADS = 384;
    // TMEM columns: dQ, Q (packed), dO (packed), S, dP
    static constexpr uint32_t COL_DQ = 0, COL_Q = 128, COL_DO = 192, COL_S = 256, COL_DP = 384;
    static constexpr int OFF_ST = 0;                                  // stages: K then V
    static constexpr int OFF_BAR = NSTAGE * 2 * TILE_BYTES;
    static constexpr int NBAR = 2 * NSTAGE + 1 + 2 + 1 + 2 + 2 + 1 + NSTAGE;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_SCRATCH = OFF_MISC + 16;
    static constexpr int OFF_PREFIX = OFF_SCRATCH + 2 * THREADS * 4;
    // block prefix, unit prefix, then the rank order (short[kMaxSortedSeqs])
    static constexpr int SMEM_BYTES = OFF_PREFIX + 2 * (kMaxVarlenSeqs + 1) * 4 + kMaxSortedSeqs * 2 + 1024;
};

struct DqBarriers {
    uint64_t *stage_full, *stage_empty, *fix_ready, *s_full, *dp_full, *mid, *ready, *acc_final,
        *acc_empty, *drain, *land;
};

// D[128 x 128] = A[tmem 128 x d, packed bf16] * B[smem 128 x d, K-major]^T.
template <int D>
__device__ __forceinline__ void issue_scores_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base) {
    constexpr uint32_t IDESC = idesc_bf16(128, DqCfg<D>::BS, false, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * DqCfg<D>::BOX + (kk & 3) * 32;
        umma_ts(d_tmem, a_tmem + kk * 8, sw128_desc(b_base + off, 16, 1024), IDESC, kk > 0);
    }
}

template <int D>
__global__ void __launch_bounds__(DqCfg<D>::THREADS, 1)
dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
          const BwdParams p) {
    using C = DqCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    uint64_t* bb = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    DqBarriers br;
    br.stage_full = bb;
    br.stage_empty = bb + C::NSTAGE;
    br.fix_ready = bb + 2 * C::NSTAGE;
    br.s_full = br.fix_ready + 1;
    br.dp_full = br.s_full + 1;
    br.mid = br.dp_full + 1;
    br.ready = br.mid + 2;          // [2 parts]
    br.acc_final = br.ready + 2;
    br.acc_empty = br.acc_final + 1;
    br.drain = br.acc_empty + 1;
    br.land = br.drain + 1;         // [NSTAGE]: stages with rows past a packed batch
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    int* scratch = reinterpret_cast<int*>(smem + C::OFF_SCRATCH);
    int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NSTAGE; ++i) {
            mbar_init(br.stage_full + i, 1);
            mbar_init(br.stage_empty + i, 1);
        }
        mbar_init(br.fix_ready, 8);      // all eight element-wise warps
        mbar_init(br.s_full, 1);
        mbar_init(br.dp_full, 1);
        mbar_init(br.mid, 8);
        mbar_init(br.ready, 8);
        mbar_init(br.ready + 1, 8);
        mbar_init(br.acc_final, 1);
        mbar_init(br.acc_empty, 8);
        mbar_init(br.drain, 1);
        for (int i = 0; i < C::NSTAGE; ++i) mbar_init(br.land + i, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
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
    sch.order = schedule_order(p.g, 1);     // query blocks: later queries see more keys
    sch.bprefix = prefix;
    sch.uprefix = prefix + kMaxVarlenSeqs + 1;
    sch.total_units = build_schedule_prefix(p.g, C::BM, prefix, prefix + kMaxVarlenSeqs + 1,
                                            scratch);   // __syncthreads inside
    schedule_split_tail(sch);
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
            uint32_t cnt = 0;
            LandTrack lt;
            bool ok = true;
            ItemIter<true> it;
            int s, h, blk;
            while (ok && it.next(sch, s, h, blk)) {
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int q0 = blk * C::BM;
                int jb, je;
                key_tile_range(q0, min(n, q0 + C::BM), n, p.g.causal, p.g.window, C::BS, jb, je);
                // packed batches: the first row of the item's last key tile past the
                // batch's last sequence (128: none); that stage lands on land[slot]
                // for the fixer warp
                const int dead_r0 = first_dead_row(p.g.cu_seqlens, p.g.B, sp.start + (je - 1) * C::BS);
                for (int j = jb; j < je; ++j, ++cnt) {
                    const int slot = cnt % C::NSTAGE;
                    if (!mbar_wait(br.stage_empty + slot, ((cnt / C::NSTAGE) & 1) ^ 1, wc)) {
                        ok = false;
                        break;
                    }
                    const bool to_land = j + 1 == je && dead_r0 < 128;
                    uint64_t* full = to_land ? br.land + slot : br.stage_full + slot;
                    lt.note(slot, to_land);
                    mbar_arrive_expect_tx(full, 2 * C::TILE_BYTES);
                    uint8_t* st = smem + C::OFF_ST + slot * 2 * C::TILE_BYTES;
                    for (int b = 0; b < C::NBOX; ++b) {
                        tma_load_3d(st + b * C::BOX, &tm_k, full, b * 64, h, sp.start + j * C::BS);
                        tma_load_3d(st + C::TILE_BYTES + b * C::BOX, &tm_v, full, b * 64, h,
                                    sp.start + j * C::BS);
                    }
                }
            }
            if (!ok) {
                for (uint32_t x = cnt > C::NSTAGE ? cnt - C::NSTAGE : 0; x < cnt; ++x) {
                    const int sl = x % C::NSTAGE;
                    if (lt.landed(sl))
                        drain_wait(br.land + sl, lt.land_parity(sl), p.error_word);
                    else
                        drain_wait(br.stage_full + sl, (x / C::NSTAGE) & 1, p.error_word);
                }
            }
        } else if (warp == 2) {
            // ------------------------------------------------------- fixer --
            // packed batches: zeroes the K and V rows past the batch's last
            // sequence in each stage the producer sent to land[slot] (they meet
            // P = 0 in dP's use and dS = 0 in the dQ GEMM), then releases the
            // stage on stage_full[slot]
            if (p.g.cu_seqlens) {
                uint32_t cnt = 0, land_par = 0;
                ItemIter<true> it;
                int s, h, blk;
                while (it.next(sch, s, h, blk)) {
                    const SeqSpan sp = sch.span(s);
                    const int n = sp.len;
                    const int q0 = blk * C::BM;
                    int jb, je;
                    key_tile_range(q0, min(n, q0 + C::BM), n, p.g.causal, p.g.window, C::BS, jb, je);
                    const int dead_r0 = first_dead_row(p.g.cu_seqlens, p.g.B, sp.start + (je - 1) * C::BS);
                    if (dead_r0 < 128) {
                        const int slot = (cnt + (je - 1 - jb)) % C::NSTAGE;
                        // every lane waits; the warp leaves together if any lane gave up
                        if (!__all_sync(0xffffffffu, mbar_wait(br.land + slot, (land_par >> slot) & 1u, wc))) break;
                        land_par ^= 1u << slot;
                        uint8_t* st = smem + C::OFF_ST + slot * 2 * C::TILE_BYTES;
                        zero_tile_rows(st, C::NBOX, dead_r0, lane, 32);
                        zero_tile_rows(st + C::TILE_BYTES, C::NBOX, dead_r0, lane, 32);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(br.stage_full + slot);
                    }
                    cnt += je - jb;
                }
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA --
            // per step j:  S_j, dP_j  ->  [S_j read] S_{j+1}  ->  [dS_j written]
            //              dQ += dS_j K_j, dP_{j+1}
            const uint32_t st_addr = smem_u32(smem + C::OFF_ST);
            uint32_t cnt = 0, item_it = 0;
            bool ok = true;
            ItemIter<true> it;
            int s, h, blk;
            for (; ok && it.next(sch, s, h, blk); ++item_it) {
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int q0 = blk * C::BM;
                int jb, je;
                key_tile_range(q0, min(n, q0 + C::BM), n, p.g.causal, p.g.window, C::BS, jb, je);
                // the block's first S and dP do not touch the dQ accumulator, so
                // they run during the previous block's epilogue; the
                // accumulator is awaited before the first dQ GEMM
                if (!mbar_wait(br.fix_ready, item_it & 1, wc)) { ok = false; break; }
                if (!mbar_wait(br.stage_full + cnt % C::NSTAGE, (cnt / C::NSTAGE) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                {
                    const uint32_t x = st_addr + (cnt % C::NSTAGE) * 2 * C::TILE_BYTES;
                    issue_scores_ts<D>(tmem + C::COL_S, tmem + C::COL_Q, x);                // Q K^T
                    umma_commit(br.s_full);
                    issue_scores_ts<D>(tmem + C::COL_DP, tmem + C::COL_DO, x + C::TILE_BYTES);  // dO V^T
                    umma_commit(br.dp_full);
                }
                if (!mbar_wait(br.acc_empty, (item_it & 1) ^ 1, wc)) { ok = false; break; }
                tc_fence_after();
                for (int j = jb; j < je; ++j, ++cnt) {
                    const bool last = (j + 1 == je);
                    const uint32_t slot = cnt % C::NSTAGE;
                    const uint32_t x = st_addr + slot * 2 * C::TILE_BYTES;
                    const uint32_t xn = st_addr + ((cnt + 1) % C::NSTAGE) * 2 * C::TILE_BYTES;
                    if (!last) {
                        if (!mbar_wait(br.stage_full + (cnt + 1) % C::NSTAGE, ((cnt + 1) / C::NSTAGE) & 1, wc)) {
                            ok = false;
                            break;
                        }
                        if (!mbar_wait(br.mid, cnt & 1, wc)) { ok = false; break; }
                        tc_fence_after();
                        issue_scores_ts<D>(tmem + C::COL_S, tmem + C::COL_Q, xn);           // next Q K^T
                        umma_commit(br.s_full);
                    }
                    bool mok = true;
                    for (int part = 0; part < 2 && mok; ++part) {
                        if (!mbar_wait(br.ready + part, cnt & 1, wc)) { mok = false; break; }
                        tc_fence_after();
                        issue_acc_ts<D>(tmem + C::COL_DQ, tmem + C::COL_DP, x, j > jb || part > 0,
                                        part);                                          // dQ += dS K
                    }
                    if (!mok) { ok = false; break; }
                    umma_commit(br.stage_empty + slot);
                    if (!last) {
                        issue_scores_ts<D>(tmem + C::COL_DP, tmem + C::COL_DO, xn + C::TILE_BYTES);  // next dO V^T
                        umma_commit(br.dp_full);
                    } else {
                        umma_commit(br.acc_final);
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
        const uint32_t tS = tmem + lane_base + C::COL_S + 64 * g;
        const uint32_t tP = tmem + lane_base + C::COL_DP + 64 * g;
        uint32_t cnt = 0, item_it = 0;
        bool ok = true;
        // this thread's row of Q (warpgroup 0) or dO (warpgroup 1) of block
        // (s, h, blk) into TMEM as packed bf16 pairs; rows past the sequence
        // end are zero.  Called before the first block, and for every later
        // block once the previous block's last S and dP have completed (the
        // only GEMMs that read these columns), ahead of that block's epilogue.
        auto load_rows = [&](int s_, int h_, int blk_) {
            const SeqSpan sp_ = sch.span(s_);
            const int qr = blk_ * C::BM + row;
            const __nv_bfloat16* src = (g == 0 ? p.qrows : p.dorows) +
                                       ((static_cast<size_t>(sp_.start) + qr) * H + h_) * D;
            uint32_t r[D / 2];
#pragma unroll
            for (int v = 0; v < D / 8; ++v) {
                uint4 x4 = make_uint4(0, 0, 0, 0);
                if (qr < sp_.len) x4 = __ldg(reinterpret_cast<const uint4*>(src) + v);
                r[4 * v] = x4.x;
                r[4 * v + 1] = x4.y;
                r[4 * v + 2] = x4.z;
                r[4 * v + 3] = x4.w;
            }
            const uint32_t dst = tmem + lane_base + (g == 0 ? C::COL_Q : C::COL_DO);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
                tmem_st32(dst + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
            arrive_warp(br.fix_ready);
        };
        ItemIter<true> it;
        int s, h, blk;
        bool have = it.next(sch, s, h, blk);
        if (have) load_rows(s, h, blk);
        for (; ok && have; ++item_it) {
            const SeqSpan sp = sch.span(s);
            const int n = sp.len;
            const int q0 = blk * C::BM;
            const int q = q0 + row;               // this thread's query row
            int jb, je;
            key_tile_range(q0, min(n, q0 + C::BM), n, p.g.causal, p.g.window, C::BS, jb, je);
            float nl = -INFINITY, neg_d = 0.f;     // -L log2e, -D of this row
            if (q < n) {
                const size_t xi = stats_index(p.g, p.stats_stride, s, h, sch.blocks_before(s), q);
                nl = p.stats[xi];
                neg_d = p.stats[xi + 128];
            }
            for (int j = jb; j < je; ++j, ++cnt) {
                if (!mbar_wait(br.s_full, cnt & 1, wc)) { ok = false; break; }
                tc_fence_after();
                const int kb = j * C::BS + 64 * g;     // this half's first key
                const bool need_mask = tile_needs_mask(q0, C::BM, kb, 64, n, p.g.causal, p.g.window);
                uint32_t r[64];
                tmem_ld64(tS, r);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(br.mid);     // S read: the next S may overwrite it
                float pf[64];
                if (!need_mask) {
                    // pairs of keys: the argument in packed float32x2
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const float2 a = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])),
                                               make_float2(sl2, sl2), make_float2(nl, nl));
                        pf[c] = ex2(a.x);
                        pf[c + 1] = ex2(a.y);
                    }
                } else {
                    // this row's allowed keys of the tile are columns [c_lo, c_hi)
                    int c_lo, c_hi;
                    tile_key_bounds(q, kb, n, p.g.causal, p.g.window, 64, c_lo, c_hi);
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        const float x = ex2(fmaf(__uint_as_float(r[c]), sl2, nl));
                        pf[c] = (c >= c_lo && c < c_hi) ? x : 0.f;
                    }
                }
                if (!mbar_wait(br.dp_full, cnt & 1, wc)) { ok = false; break; }
                tc_fence_after();
                tmem_ld64(tP, r);
                tmem_wait_ld();
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int k = 32 * part + 2 * c;
                        const float2 d = fmul2(make_float2(pf[k], pf[k + 1]),
                                               fadd2(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])),
                                                     make_float2(neg_d, neg_d)));
                        pk[c] = pack_bf16(d.x, d.y);
                    }
                    tmem_st16(tP + 16 * part, pk);   // dS packed over the first 32 columns of this half
                    arrive_warp(br.ready + part);
                }
            }
            if (!ok) break;
            // the next block's rows first, so that its first S and dP run
            // during this block's epilogue
            int s_next, h_next, blk_next;
            const bool have_next = it.next(sch, s_next, h_next, blk_next);
            if (have_next) load_rows(s_next, h_next, blk_next);
            // ------------------------------------------------ epilogue --
            if (!mbar_wait(br.acc_final, item_it & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool valid = q < n;
            const size_t off = (static_cast<size_t>(sp.start) + q) * H * D + static_cast<size_t>(h) * D;
            if constexpr (D == 128) {
                // this group's 64 columns: one 128-byte line of the row
                store_line_bf16(tmem + lane_base + C::COL_DQ + g * 64, p.scale, p.out0 + off + g * 64, valid);
            } else {
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    const int col = g * (D / 2) + c * 32;
                    store_row_chunk(tmem + lane_base + C::COL_DQ + col, p.scale, p.out0 + off + col, valid);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(br.acc_empty);
            s = s_next;
            h = h_next;
            blk = blk_next;
            have = have_next;
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
    CUtensorMap q, k, v, dO;   // 128-row boxes
};

struct BwdArgs {
    Geometry g;
    int d;
    const void *q, *o, *dO;
    const float* lse;
    void *dq, *dk, *dv;
    float* stats;            // workspace
    int64_t stats_stride;
    float scale;
    int num_sms;
    int* error_word;
    uint64_t timeout_ns;
};

// Row stride of the padded statistics array (see BwdParams).
inline int64_t bwd_stats_stride(int B, int N, int64_t packed_rows, bool packed) {
    if (!packed) return (static_cast<int64_t>(N) + 127) / 128 * 128;
    return (packed_rows + 127 * static_cast<int64_t>(B) + 127) / 128 * 128;
}

// Workspace bytes: the padded statistics array, 8 bytes per entry.
inline size_t bwd_workspace_bytes(int B, int H, int64_t stride, bool packed) {
    const int64_t entries = packed ? static_cast<int64_t>(H) * stride
                                   : static_cast<int64_t>(B) * H * stride;
    return static_cast<size_t>((entries * 8 + 255) / 256 * 256);
}

constexpr int kStatsSmem = (3 * (kMaxVarlenSeqs + 1) + 2 * 256) * 4;

inline cudaError_t bwd_set_smem_limits() {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(stats_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kStatsSmem)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(stats_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kStatsSmem)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(dkdv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BwdCfg<64>::SMEM_BYTES)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(dkdv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BwdCfg<128>::SMEM_BYTES)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  DqCfg<64>::SMEM_BYTES)) != cudaSuccess)
        return e;
    return cudaFuncSetAttribute(dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                DqCfg<128>::SMEM_BYTES);
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
        const int rows_per_block = 8 * 32;
        int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
        const int64_t cap = static_cast<int64_t>(a.num_sms) * kStatsCtasPerSm;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        stats_kernel<D><<<static_cast<int>(blocks), 256, a.g.cu_seqlens ? kStatsSmem : 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a.dO), static_cast<const __nv_bfloat16*>(a.o), a.lse,
            a.stats, a.stats_stride, a.g, nullptr);
        hk.stop(1, slot, stream);
    }
    BwdParams p;
    p.g = a.g;
    p.stats = a.stats;
    p.stats_stride = a.stats_stride;
    p.qrows = static_cast<const __nv_bfloat16*>(a.q);
    p.dorows = static_cast<const __nv_bfloat16*>(a.dO);
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
    dkdv_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(m.k, m.v, m.q, m.dO, p);
    hk.stop(2, slot, stream);
    p.out0 = static_cast<__nv_bfloat16*>(a.dq);
    p.out1 = nullptr;
    slot = hk.start(3, stream);
    dq_kernel<D><<<grid, DqCfg<D>::THREADS, DqCfg<D>::SMEM_BYTES, stream>>>(m.k, m.v, p);
    hk.stop(3, slot, stream);
    return cudaGetLastError();
}

inline cudaError_t bwd_launch(const BwdArgs& a, const BwdMaps& m, cudaStream_t stream,
                              const BwdHooks& hk) {
    return a.d == 64 ? bwd_launch_d<64>(a, m, stream, hk) : bwd_launch_d<128>(a, m, stream, hk);
}

}  // namespace fa
