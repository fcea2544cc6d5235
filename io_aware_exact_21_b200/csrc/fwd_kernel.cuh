// fwd_kernel.cuh -- fused, tiled exact attention forward for sm_100a.
//
// What it computes: O = softmax(scale * Q K^T) V per (sequence, head), plus
// the per-row log-sum-exp, without ever writing the score or probability
// matrix to HBM (FlashAttention encyclopedia page, "attention and the memory
// bottleneck" and "tiled computation and online normalisation"; the IO-aware
// essay, "let a block do more work on chip", whose flow chart is: load a Q
// block, stream K/V blocks, form local scores, update row statistics,
// accumulate the output, write the final output once).
//
// Online update per key tile (encyclopedia page, update equations), here in
// base 2 with s' = s * scale * log2(e):
//     m' = max(m, max_j s'_j),  l' = 2^(m-m') l + sum_j 2^(s'_j - m'),
//     u' = 2^(m-m') u + sum_j 2^(s'_j - m') v_j,   O = u / l,
//     LSE = ln 2 * (m + log2 l).
// The rescale is applied only when the running maximum grows by more than
// kRescaleLog2 (a factor 256): the update is exact for any reference value
// used consistently in l and u, the maximum only keeps 2^(s'-m) bounded
// (same page: subtracting the maximum is for numerical stability).
//
// CTA = two query tiles of 128 rows (256 rows) of one (sequence, head); both
// tiles share one stream of K/V tiles of 128 keys.  Roles (384 threads):
//   warp 0        TMA producer: Q tiles, then K_j, V_j into a ring of smem slots
//   warp 1        TMEM owner and MMA issuer (one elected thread):
//                 S_t = Q_t K_j^T (both operands in smem), O_t += P_t V_j
//                 (P_t read from TMEM, V_j from smem)
//   warps 2-3     idle
//   warps 4-7     softmax + correction + epilogue of tile 0 (one thread per row)
//   warps 8-11    the same for tile 1
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D).
// P_t is written as packed bf16 over the first 64 columns of S_t, in two
// halves of 64 keys that are released to the MMA warp one at a time.
// The MMA thread issues S_t(j+1) right after O_t += P_t(j) V_j, so while one
// softmax warpgroup works on its tile the tensor core runs the other's GEMMs.
//
// kF8 = true instantiates the block-quantised FP8 variant (FlashAttention
// encyclopedia page, FlashAttention-3 paragraph: an FP8 path with block
// quantisation, kept apart from the exact path).  Q and K are e4m3 codes with
// one scale per 128-row block of a head, V is e4m3 stored transposed
// ([B, H, d, keys], so both GEMMs read K-major operands) with one scale per
// 128-key block.  Both GEMMs are kind::f8f6f4 MMAs; the score tile is scaled
// by scale * log2(e) * s_q * s_k in the softmax, and P is written to TMEM as
// e4m3 after multiplying by r = s_v(block) / max s_v (so one accumulator
// serves every V block; O is multiplied back by max s_v at the end).  The row
// sum uses the unrounded P.  Fixed-length sequences and d = 128 only.
//
// kCache = true instantiates the padded K/V cache variant (fixed-length
// queries; sequence s uses the first seqused_k[s] rows of its Nk-row cache
// slice).  With nsplit > 1 it also cuts the key tiles of every block into
// `nsplit` contiguous ranges that run as separate work items (the schedule
// sees H * nsplit heads), so that few, long blocks still spread over all SMs;
// each item then writes O / l as fp32 and the base-2 log-sum-exp of its range
// to the split buffers ([nsplit, rows, H, D] and [nsplit, H, rows]), which
// combine_kernel merges.  A split with no tiles writes -inf and is skipped by
// the merge.  Cache rows past a sequence's used length are never read: K and V
// come through 4-D maps [B, Nk, H, d] (coordinates channel, head, row,
// sequence), and a key tile that would reach past the used length nk is read
// right-aligned instead, as keys [nk - 128, nk) -- rows before 0 are outside
// the map and arrive as zeros -- with the keys below the tile's own start
// (those of the tile before it) masked out in the softmax.
//
// kSingles = true (always with kCache; also instantiated for packed cached-KV
// prefill) walks every 256-row block as its own work unit instead of pairs of
// blocks of one head (ItemIter's kSingles walk): where each head's keys far
// outnumber its queries, pairs keep twice as many heads' K/V in flight as
// singles do, more than L2 holds.
#pragma once

#include "dead_rows.cuh"
#include "schedule.cuh"
#include "sm100.cuh"

namespace fa {

constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

struct FwdParams {
    Geometry g;
    __nv_bfloat16* o;
    float* lse;
    float scale_log2;       // scale * log2(e)
    int* error_word;
    uint64_t timeout_ns;
    int fault_skip_v;       // test hook: producer skips the first V load
    // Variant parameters; the FP8 and padded-cache variants never coexist, so
    // they share storage (a larger parameter block changed the plain kernel's
    // register allocation for the worse).
    struct F8 {                 // FP8: block scales [B, H, nb] of Q, K, V, nb = ceil(N / 128)
        const float* sq;
        const float* sk;
        const float* sv;
    };
    struct Cache {              // padded cache: used rows per sequence, split outputs
        const int* seqused_k;   // or nullptr (all Nk rows in use)
        float* o_part;          // [nsplit, B * N, H, D]
        float* lse_part;        // [nsplit, H, B * N], base 2
    };
    union {
        F8 f8;
        Cache kv;
    };
    union {
        int nb;                 // FP8
        int nsplit;             // padded cache
    };
};

// Tiles [jb, je) of split `split` out of `nsplit` for a block whose key range
// is [jb, je); false when the split has none.
__device__ __forceinline__ bool split_tile_range(int nsplit, int split, int& jb, int& je) {
    const int n = je - jb;
    const int ns = min(nsplit, n);
    if (split >= ns) return false;
    const int b0 = jb;
    jb = b0 + split * n / ns;
    je = b0 + (split + 1) * n / ns;
    return true;
}

// 4-D tiled load, box coordinates (c0 innermost), into this CTA's shared
// memory (the padded cache's maps: channel, head, row, sequence).
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
          "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// First key of cache tile j as read (128 keys): j * 128, or nk - 128 for the
// tile that would reach past the used length nk (negative when nk < 128).
__device__ __forceinline__ int cache_tile_key0(int j, int nk) {
    return (j + 1) * 128 > nk ? nk - 128 : j * 128;
}

template <int D, bool kF8 = false>
struct FwdCfg {
    static constexpr int BM = 128;              // rows per query tile
    static constexpr int BN = 128;              // keys per key tile
    static constexpr int ROWS = 2 * BM;         // rows per CTA work item
    static constexpr int ESIZE = kF8 ? 1 : 2;   // bytes per element
    static constexpr int BOX_BYTES = 128 * 128; // one TMA box: 128 rows x 128 bytes
    static constexpr int TILE_BYTES = BM * D * ESIZE;
    static constexpr int NSLOT = kF8 ? 8 : 4;   // K/V ring depth (128 KB either way)
    static constexpr int NBOX = D * ESIZE / 128;
    static constexpr int KSTEPS = D * ESIZE / 32;   // MMA k-steps of 32 bytes over d
    static constexpr int THREADS = 384;
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 384;
    // shared memory carve-up (offsets from a 1024-byte aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_KV + NSLOT * TILE_BYTES;
    static constexpr int NBAR = 2 + 2 * NSLOT + 8 + 1 + NSLOT;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_SCRATCH = OFF_MISC + 16;
    static constexpr int OFF_PREFIX = OFF_SCRATCH + 2 * THREADS * 4;   // block and unit prefixes
    // block prefix, unit prefix, then the rank order (short[kMaxSortedSeqs])
    static constexpr int SMEM_BYTES = OFF_PREFIX + 2 * (kMaxVarlenSeqs + 1) * 4 + kMaxSortedSeqs * 2 + 1024;
};

template <int D, bool kF8 = false, bool kCache = false, bool kSingles = kCache>
__global__ void __launch_bounds__(FwdCfg<D, kF8>::THREADS, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdCfg<D, kF8>;
    static_assert(!kF8 || D == 128, "the FP8 variant is built for d = 128");
    static_assert(!(kF8 && kCache), "no FP8 cache variant");
    static_assert(!kCache || C::BN == 128, "cache_tile_key0 assumes 128-key tiles");
    static_assert(!kCache || kSingles, "the cache variant walks single blocks");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sKV = smem + C::OFF_KV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* slot_full = bars + 2;
    uint64_t* slot_empty = bars + 2 + C::NSLOT;
    uint64_t* s_full = bars + 2 + 2 * C::NSLOT;     // [2]
    uint64_t* p_full = s_full + 2;                  // [2 tiles x 2 halves]
    uint64_t* o_final = p_full + 4;                 // [2]
    uint64_t* drain = o_final + 2;
    uint64_t* land = drain + 1;                    // [NSLOT]: tiles with rows past the batch
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    int* scratch = reinterpret_cast<int*>(smem + C::OFF_SCRATCH);
    int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);

    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();
    unsigned long long* t_start = reinterpret_cast<unsigned long long*>(smem + C::OFF_MISC + 8);

    if (threadIdx.x == 0) {
        *t_start = global_timer_ns();         // this CTA's start (profiling: CTA balance)
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(slot_full + s, 1);
            mbar_init(slot_empty + s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full + t, 1);
            mbar_init(p_full + 2 * t, 4);       // one arrival per softmax warp, per half
            mbar_init(p_full + 2 * t + 1, 4);
            mbar_init(o_final + t, 1);
        }
        mbar_init(drain, 1);
        for (int s = 0; s < C::NSLOT; ++s) mbar_init(land + s, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    Schedule sch;
    sch.g = p.g;
    sch.rows_per_item = C::ROWS;
    // fixed length under a causal or window mask: pairs, then the last
    // round's blocks one by one, heaviest first (query blocks grow in cost
    // with their index); pairs alone otherwise
    sch.order = kCache ? 0 : schedule_order(p.g, 1);
    sch.bprefix = prefix;
    sch.uprefix = prefix + kMaxVarlenSeqs + 1;
    if constexpr (kCache) {
        // (head, split) pairs; one block per unit (ItemIter's kSingles walk)
        sch.g.H = p.g.H * p.nsplit;
        sch.total_units = sch.g.B * sch.g.H * sch.blocks_of(sch.g.N);
    } else {
        sch.total_units = build_schedule_prefix(p.g, C::ROWS, prefix, prefix + kMaxVarlenSeqs + 1,
                                                scratch, true, kSingles);  // has __syncthreads
    }
    schedule_split_tail(sch);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const WaitCtl wc{abort_flag, p.error_word, p.timeout_ns};
    const int H = p.g.H;

    // register split: 120 per thread for the producer / MMA warpgroup, 192 for
    // the two softmax warpgroups: 120 * 128 + 192 * 256 = 64512, the launch's
    // 168 * 384 (at 104 / 200 the producer and MMA code spilled)
    if (warp < 4) {
        regs_dealloc<120>();
        if (warp == 0 && lane == 0) {
            // ------------------------------------------------ TMA producer --
            uint32_t cnt = 0, item_it = 0;
            uint32_t q_issued = 0;
            LandTrack lt;
            bool ok = true;
            bool skipped = false;
            uint32_t skipped_at = 0xffffffffu;
            ItemIter<true, kSingles, !kCache> it;
            int s, h, blk;
            for (; ok && it.next(sch, s, h, blk); ++item_it) {
                [[maybe_unused]] int split = 0;
                if constexpr (kCache) {
                    split = h % p.nsplit;
                    h /= p.nsplit;
                }
                const SeqSpan sp = sch.span(s);
                const SeqSpan kp = kCache ? sch.kspan_used(s, p.kv.seqused_k) : sch.kspan(s);
                const int off = kp.len - sp.len;        // key position of query row 0
                const int r_lo = blk * C::ROWS;
                const int r_hi = min(sp.len, r_lo + C::ROWS);
                int jb, je;
                key_tile_range(r_lo + off, r_hi + off, kp.len, p.g.causal, p.g.window, C::BN, jb, je);
                if constexpr (kCache) {
                    if (!split_tile_range(p.nsplit, split, jb, je)) {
                        --item_it;          // no tiles: no barrier phase for this item
                        continue;
                    }
                }
                // packed batches: the first row of the item's last key tile past
                // the batch's last sequence (128: none); that tile's V lands on
                // land[slot] for the fixer warp
                int dead_r0 = 128;
                if constexpr (!kF8 && !kCache)
                    dead_r0 = first_dead_row(p.g.cu_seqlens_k, p.g.B, kp.start + (je - 1) * C::BN);
                if (!mbar_wait(q_empty, (item_it & 1) ^ 1, wc)) { ok = false; break; }
                mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
                for (int t = 0; t < 2; ++t)
                    for (int b = 0; b < C::NBOX; ++b)
                        tma_load_3d(sQ + t * C::TILE_BYTES + b * C::BOX_BYTES, &tm_q, q_full,
                                    b * 128 / C::ESIZE, h, sp.start + r_lo + t * C::BM);
                ++q_issued;
                for (int j = jb; j < je && ok; ++j) {
                    for (int kv = 0; kv < 2; ++kv) {
                        const int slot = cnt % C::NSLOT;
                        if (!mbar_wait(slot_empty + slot, ((cnt / C::NSLOT) & 1) ^ 1, wc)) {
                            ok = false;
                            break;
                        }
                        if (kv == 1 && p.fault_skip_v && !skipped) {
                            skipped = true;   // test hook: this slot never fills
                            skipped_at = cnt;
                        } else {
                            const bool to_land = kv == 1 && j + 1 == je && dead_r0 < 128;
                            uint64_t* full = to_land ? land + slot : slot_full + slot;
                            lt.note(slot, to_land);
                            mbar_arrive_expect_tx(full, C::TILE_BYTES);
                            uint8_t* dst = sKV + slot * C::TILE_BYTES;
                            if (kF8 && kv == 1) {
                                // V^T tile: d rows of this (sequence, head), 128 keys
                                tma_load_2d(dst, &tm_v, full, j * C::BN, (s * H + h) * D);
                            } else if constexpr (kCache) {
                                const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
                                const int k0 = cache_tile_key0(j, kp.len);
                                for (int b = 0; b < C::NBOX; ++b)
                                    tma_load_4d(dst + b * C::BOX_BYTES, tm, full, b * 128 / C::ESIZE, h,
                                                k0, s);
                            } else {
                                const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
                                for (int b = 0; b < C::NBOX; ++b)
                                    tma_load_3d(dst + b * C::BOX_BYTES, tm, full, b * 128 / C::ESIZE, h,
                                                kp.start + j * C::BN);
                            }
                        }
                        ++cnt;
                    }
                }
            }
            if (!ok) {
                // Let the copies already in flight land before the CTA exits.
                WaitCtl dw{abort_flag, p.error_word, 200000000ull};
                volatile int no_abort = 0;
                dw.abort_flag = &no_abort;
                // The latest phase of every slot is one of the last NSLOT loads.
                for (uint32_t x = cnt > C::NSLOT ? cnt - C::NSLOT : 0; x < cnt; ++x) {
                    if (x == skipped_at) continue;
                    const int sl = x % C::NSLOT;
                    if (lt.landed(sl))
                        mbar_wait(land + sl, lt.land_parity(sl), dw);
                    else
                        mbar_wait(slot_full + sl, (x / C::NSLOT) & 1, dw);
                }
                if (q_issued) mbar_wait(q_full, (q_issued - 1) & 1, dw);
            }
        } else if (warp == 2) {
            // ------------------------------------------------------- fixer --
            // packed batches: zeroes the V rows past the batch's last sequence in
            // each tile the producer sent to land[slot], then releases the tile
            // on slot_full[slot] (walks the items and ring slots as the MMA
            // issuer does)
            if constexpr (!kF8 && !kCache) {
                if (p.g.cu_seqlens_k) {
                    uint32_t cnt = 0, land_par = 0;
                    ItemIter<true, kSingles, !kCache> it;
                    int s, h, blk;
                    while (it.next(sch, s, h, blk)) {
                        const SeqSpan sp = sch.span(s);
                        const SeqSpan kp = sch.kspan(s);
                        const int off = kp.len - sp.len;
                        const int r_lo = blk * C::ROWS;
                        const int r_hi = min(sp.len, r_lo + C::ROWS);
                        int jb, je;
                        key_tile_range(r_lo + off, r_hi + off, kp.len, p.g.causal, p.g.window, C::BN, jb, je);
                        const int dead_r0 = first_dead_row(p.g.cu_seqlens_k, p.g.B, kp.start + (je - 1) * C::BN);
                        if (dead_r0 < 128) {
                            const int slot = (cnt + 2 * (je - 1 - jb) + 1) % C::NSLOT;
                            // every lane waits; the warp leaves together if any lane gave up
                            if (!__all_sync(0xffffffffu, mbar_wait(land + slot, (land_par >> slot) & 1u, wc))) break;
                            land_par ^= 1u << slot;
                            zero_tile_rows(sKV + slot * C::TILE_BYTES, C::NBOX, dead_r0, lane, 32);
                            __syncwarp();
                            if (lane == 0) mbar_arrive(slot_full + slot);
                        }
                        cnt += 2 * (je - jb);
                    }
                }
            }
        } else if (warp == 1 && lane == 0) {
            // --------------------------------------------------- MMA issuer --
            constexpr uint32_t IDESC_S = kF8 ? idesc_e4m3(128, C::BN) : idesc_bf16(128, C::BN, false, false);
            constexpr uint32_t IDESC_O = kF8 ? idesc_e4m3(128, D) : idesc_bf16(128, D, false, true);
            const uint32_t q_addr = smem_u32(sQ);
            const uint32_t kv_addr = smem_u32(sKV);
            uint32_t cnt = 0, step = 0, item_it = 0;
            bool ok = true;
            auto issue_s = [&](int t, uint32_t kslot) {
                const uint32_t d_tmem = tmem + (t ? C::COL_S1 : C::COL_S0);
                const uint32_t a0 = q_addr + t * C::TILE_BYTES;
                const uint32_t b0 = kv_addr + kslot * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                    if constexpr (kF8)
                        umma_ss_f8(d_tmem, sw128_desc(a0 + off, 16, 1024),
                                   sw128_desc(b0 + off, 16, 1024), IDESC_S, kk > 0);
                    else
                        umma_ss(d_tmem, sw128_desc(a0 + off, 16, 1024),
                                sw128_desc(b0 + off, 16, 1024), IDESC_S, kk > 0);
                }
            };
            // O_t (+)= P_t[:, keys of half] V_j[keys of half, :]  (half = 64 keys)
            auto issue_pv = [&](int t, uint32_t vslot, uint32_t accumulate, int half) {
                const uint32_t d_tmem = tmem + (t ? C::COL_O1 : C::COL_O0);
                const uint32_t a_tmem = tmem + (t ? C::COL_S1 : C::COL_S0);
                const uint32_t b0 = kv_addr + vslot * C::TILE_BYTES;
                if constexpr (kF8) {
                    // P: 4 e4m3 per TMEM column, 32 keys (8 columns) per k-step;
                    // V^T K-major: 32 keys = 32 bytes along its 128-byte rows
#pragma unroll
                    for (int k = 0; k < C::BN / 64; ++k) {
                        const int kk = half * (C::BN / 64) + k;
                        umma_ts_f8(d_tmem, a_tmem + kk * 8, sw128_desc(b0 + kk * 32, 16, 1024),
                                   IDESC_O, (accumulate | kk) != 0);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < C::BN / 32; ++k) {
                        const int kk = half * (C::BN / 32) + k;
                        umma_ts(d_tmem, a_tmem + kk * 8,
                                sw128_desc(b0 + kk * 2048, C::BOX_BYTES, 1024), IDESC_O,
                                (accumulate | kk) != 0);
                    }
                }
            };
            ItemIter<true, kSingles, !kCache> it;
            int s, h, blk;
            for (; ok && it.next(sch, s, h, blk); ++item_it) {
                [[maybe_unused]] int split = 0;
                if constexpr (kCache) {
                    split = h % p.nsplit;
                    h /= p.nsplit;
                }
                const SeqSpan sp = sch.span(s);
                const SeqSpan kp = kCache ? sch.kspan_used(s, p.kv.seqused_k) : sch.kspan(s);
                const int off = kp.len - sp.len;
                const int r_lo = blk * C::ROWS;
                const int r_hi = min(sp.len, r_lo + C::ROWS);
                int jb, je;
                key_tile_range(r_lo + off, r_hi + off, kp.len, p.g.causal, p.g.window, C::BN, jb, je);
                if constexpr (kCache) {
                    if (!split_tile_range(p.nsplit, split, jb, je)) {
                        --item_it;          // no tiles: no barrier phase for this item
                        continue;
                    }
                }
                if (!mbar_wait(q_full, item_it & 1, wc)) { ok = false; break; }
                // first key tile
                uint32_t kslot = cnt % C::NSLOT;
                if (!mbar_wait(slot_full + kslot, (cnt / C::NSLOT) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                issue_s(0, kslot);
                umma_commit(s_full + 0);
                issue_s(1, kslot);
                umma_commit(s_full + 1);
                umma_commit(slot_empty + kslot);
                if (jb + 1 == je) umma_commit(q_empty);   // the item's last S: Q is free
                ++cnt;
                for (int j = jb; j < je; ++j, ++step) {
                    const bool last = (j + 1 == je);
                    const uint32_t vslot = cnt % C::NSLOT;
                    const uint32_t kslot_n = (cnt + 1) % C::NSLOT;
                    if (!mbar_wait(slot_full + vslot, (cnt / C::NSLOT) & 1, wc)) { ok = false; break; }
                    if (!mbar_wait(p_full + 0, step & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(0, vslot, j > jb, 0);
                    if (!mbar_wait(p_full + 1, step & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(0, vslot, 1, 1);
                    if (last) umma_commit(o_final + 0);
                    if (!last) {
                        if (!mbar_wait(slot_full + kslot_n, ((cnt + 1) / C::NSLOT) & 1, wc)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_s(0, kslot_n);
                        umma_commit(s_full + 0);
                    }
                    if (!mbar_wait(p_full + 2, step & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(1, vslot, j > jb, 0);
                    if (!mbar_wait(p_full + 3, step & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(1, vslot, 1, 1);
                    if (last) umma_commit(o_final + 1);
                    umma_commit(slot_empty + vslot);
                    if (!last) {
                        issue_s(1, kslot_n);
                        umma_commit(s_full + 1);
                        umma_commit(slot_empty + kslot_n);
                        if (j + 2 == je) umma_commit(q_empty);   // the item's last S: Q is free
                        cnt += 2;
                    } else {
                        cnt += 1;
                    }
                }
            }
            if (!ok) {
                umma_commit(drain);
                WaitCtl dw{abort_flag, p.error_word, 200000000ull};
                volatile int no_abort = 0;
                dw.abort_flag = &no_abort;
                mbar_wait(drain, 0, dw);
            }
        }
        __syncwarp();
    } else {
        // --------------------------------------------- softmax warpgroups --
        regs_alloc<192>();
        const int t = (warp >> 2) - 1;               // query tile 0 or 1
        const int wq = warp & 3;                     // TMEM lane quarter
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + (t ? C::COL_S1 : C::COL_S0);
        const uint32_t tO = tmem + lane_base + (t ? C::COL_O1 : C::COL_O0);
        const int row_in_tile = wq * 32 + lane;
        const float sl2 = p.scale_log2;
        uint32_t step = 0, item_it = 0;
        bool ok = true;
        ItemIter<true, kSingles, !kCache> it;
        int s, h, blk;
        for (; ok && it.next(sch, s, h, blk); ++item_it) {
            [[maybe_unused]] int split = 0;
            if constexpr (kCache) {
                split = h % p.nsplit;
                h /= p.nsplit;
            }
            const SeqSpan sp = sch.span(s);
            const SeqSpan kp = kCache ? sch.kspan_used(s, p.kv.seqused_k) : sch.kspan(s);
            const int n = sp.len;
            const int nk = kp.len;
            const int off = nk - n;                     // key position of query row 0
            const int r_lo = blk * C::ROWS;
            const int r_hi = min(n, r_lo + C::ROWS);
            int jb, je;
            key_tile_range(r_lo + off, r_hi + off, nk, p.g.causal, p.g.window, C::BN, jb, je);
            const int r0 = r_lo + t * C::BM;            // first row of this tile
            const int i = r0 + row_in_tile;             // this thread's row
            if constexpr (kCache) {
                if (!split_tile_range(p.nsplit, split, jb, je)) {
                    if (i < n)
                        p.kv.lse_part[(static_cast<size_t>(split) * H + h) * p.g.T + sp.start + i] =
                            -INFINITY;
                    --item_it;
                    continue;
                }
            }
            float m_ref = -INFINITY;
            float l = 0.f;
            // FP8: the Q tile's scale, and the largest V block scale of the head
            float sq_t = 1.f, sv_max = 1.f;
            const float* skh = nullptr;
            const float* svh = nullptr;
            if constexpr (kF8) {
                const size_t base = (static_cast<size_t>(s) * H + h) * p.nb;
                skh = p.f8.sk + base;
                svh = p.f8.sv + base;
                sq_t = p.f8.sq[base + min(r0 / C::BM, p.nb - 1)];
                float mv = 0.f;
                for (int b = lane; b < p.nb; b += 32) mv = fmaxf(mv, svh[b]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
                sv_max = mv > 0.f ? mv : 1.f;
            }
            for (int j = jb; j < je; ++j, ++step) {
                float sl2j = sl2, r_j = 1.f;
                if constexpr (kF8) {
                    sl2j = sl2 * sq_t * skh[j];
                    r_j = fminf(1.f, svh[j] / sv_max);
                }
                if (!mbar_wait(s_full + t, step & 1, wc)) { ok = false; break; }
                tc_fence_after();
                float sv[C::BN];
                {
                    uint32_t r[C::BN];
#pragma unroll
                    for (int c = 0; c < C::BN / 32; ++c)
                        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < C::BN; ++e) sv[e] = __uint_as_float(r[e]);
                }
                const int k0 = j * C::BN;
                const bool masked = tile_needs_mask_pos(r0 + off, min(r0 + C::BM, n) + off, k0, C::BN,
                                                        nk, p.g.causal, p.g.window);
                if (masked) {
                    // this row's allowed keys of the tile are columns [c_lo, c_hi)
                    int c_lo, c_hi;
                    if constexpr (kCache) {
                        // the tile holds keys from k0r on; those below k0 belong to
                        // the tile before it
                        const int k0r = cache_tile_key0(j, nk);
                        tile_key_bounds(i + off, k0r, nk, p.g.causal, p.g.window, C::BN, c_lo, c_hi);
                        c_lo = max(c_lo, min(k0 - k0r, C::BN));
                        c_hi = max(c_hi, c_lo);
                    } else {
                        tile_key_bounds(i + off, k0, nk, p.g.causal, p.g.window, C::BN, c_lo, c_hi);
                    }
#pragma unroll
                    for (int c = 0; c < C::BN; ++c) sv[c] = (c >= c_lo && c < c_hi) ? sv[c] : -INFINITY;
                }
                // row maximum as a tree of three-input maxima (the max is exact
                // in any order), so the compares are not one dependent chain
                const float mx = row_max<C::BN>(sv);
                const float m_new = fmaxf(m_ref, mx * sl2j);
                const bool resc = m_new > m_ref + kRescaleLog2;
                float alpha = 1.f;
                if (resc) {
                    alpha = ex2(m_ref - m_new);
                    l *= alpha;
                    m_ref = m_new;
                }
                const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                float lsum = 0.f;
                // P in two halves of 64 keys, each released to the MMA warp as soon
                // as it is in TMEM, so O += P V for the first half overlaps the
                // exponentials of the second.  Masked keys hold -inf: ex2 gives 0.
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if constexpr (kF8) {
                        // 64 keys -> 16 columns of four e4m3 values, scaled by r_j
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int k = half * 64 + 4 * e;
                            const float p0 = ex2(fmaf(sv[k], sl2j, neg_m));
                            const float p1 = ex2(fmaf(sv[k + 1], sl2j, neg_m));
                            const float p2 = ex2(fmaf(sv[k + 2], sl2j, neg_m));
                            const float p3 = ex2(fmaf(sv[k + 3], sl2j, neg_m));
                            lsum += (p0 + p1) + (p2 + p3);
                            pk[e] = pack_e4m3x4(p0 * r_j, p1 * r_j, p2 * r_j, p3 * r_j);
                        }
                        tmem_st16(tS + half * 16, pk);
                    } else {
                        // pairs of keys: the argument and the row sum in packed
                        // float32x2 arithmetic (two sums, added at the end)
                        float2 ls = make_float2(0.f, 0.f);
#pragma unroll
                        for (int c = half * (C::BN / 64); c < (half + 1) * (C::BN / 64); ++c) {
                            uint32_t pk[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const float2 a = ffma2(make_float2(sv[c * 32 + 2 * e], sv[c * 32 + 2 * e + 1]),
                                                       make_float2(sl2, sl2), make_float2(neg_m, neg_m));
                                const float p0 = ex2(a.x);
                                const float p1 = ex2(a.y);
                                ls = fadd2(ls, make_float2(p0, p1));
                                pk[e] = pack_bf16(p0, p1);
                            }
                            tmem_st16(tS + c * 16, pk);
                        }
                        lsum += ls.x + ls.y;
                    }
                    if (half == 0 && j > jb && __any_sync(0xffffffffu, resc)) {
                        // O_t *= alpha before the first O_t += P V of this step.  The
                        // previous one has completed because S_t(j), which the MMA
                        // thread issued after it, has.
                        uint32_t r[32];
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            tmem_ld32(tO + c * 32, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                            tmem_st32(tO + c * 32, r);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(p_full + 2 * t + half);
                }
                l += lsum;
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue --
            if (!mbar_wait(o_final + t, item_it & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool valid = i < n;
            const float inv_l = l > 0.f ? (kF8 ? sv_max : 1.f) / l : 0.f;
            if constexpr (kCache) if (p.nsplit > 1) {
                // this split's O / l (fp32) and base-2 log-sum-exp
                float* prow = p.kv.o_part + ((static_cast<size_t>(split) * p.g.T + sp.start + i) * H + h) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tO + c * 32, r);
                    tmem_wait_ld();
                    if (valid) {
                        float4* dst = reinterpret_cast<float4*>(prow + c * 32);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_float4(__uint_as_float(r[4 * v]) * inv_l,
                                                 __uint_as_float(r[4 * v + 1]) * inv_l,
                                                 __uint_as_float(r[4 * v + 2]) * inv_l,
                                                 __uint_as_float(r[4 * v + 3]) * inv_l);
                    }
                }
                if (valid)
                    p.kv.lse_part[(static_cast<size_t>(split) * H + h) * p.g.T + sp.start + i] =
                        l > 0.f ? m_ref + __log2f(l) : -INFINITY;
                tc_fence_before();
                continue;
            }
            __nv_bfloat16* orow = p.o + (static_cast<size_t>(sp.start) + i) * H * D +
                                  static_cast<size_t>(h) * D;
            // 64 columns (one 128-byte line of the row) at a time, whole lines
            // per store instruction
#pragma unroll
            for (int c = 0; c < D / 64; ++c) store_line_bf16(tO + c * 64, inv_l, orow + c * 64, valid);
            if (valid) {
                const float lse = l > 0.f ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
                const size_t idx = p.g.cu_seqlens
                                       ? static_cast<size_t>(h) * p.g.T + sp.start + i
                                       : (static_cast<size_t>(s) * H + h) * p.g.N + i;
                p.lse[idx] = lse;
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0) {
        unsigned long long* const cta_clock = g_cta_clock;
        if (cta_clock && blockIdx.x < 4096) {
            if (blockIdx.x == 0) cta_clock[0] = gridDim.x;
            cta_clock[1 + 2 * blockIdx.x] = *t_start;
            cta_clock[2 + 2 * blockIdx.x] = global_timer_ns();
        }
    }
}

}  // namespace fa
