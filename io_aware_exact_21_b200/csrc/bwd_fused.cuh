// bwd_fused.cuh -- single-kernel backward pass (dK, dV and dQ in one kernel)
// for sm_100a, d = 128.
//
// The two-kernel backward (bwd_kernels.cuh) recomputes the score and gradient
// tiles twice: once in the dK/dV kernel and once in the dQ kernel, seven
// 128 x 128 GEMMs per (key tile, query tile) pair for the five the gradients
// need.  This kernel does the five once: a CTA owns 128 keys of a (sequence,
// head), streams the query tiles that can see them, and per query tile runs
//   S^T = K Q^T, dP^T = V dO^T                       (tcgen05, smem operands)
//   P^T, dS^T                                        (element-wise warps)
//   dV += P^T dO, dK += dS^T Q                        (tcgen05, TMEM operands)
//   dQ_part = dS K                                    (tcgen05, smem operands)
// and adds each tile's dQ part (fp32, 128 x 128) into an fp32 dQ accumulator
// in global memory with the bulk-copy unit's reduction
// (cp.reduce.async.bulk ... .add.f32); a last kernel scales the accumulator
// into bf16 dQ.  The gradient formulas and the recomputation from the
// log-sum-exp are those of bwd_kernels.cuh (FlashAttention encyclopedia page,
// "training and complexity": compact statistics plus recomputation).
//
// Cost on the other side: every (key tile, query tile) pair adds 64 KB of fp32
// into the accumulator, so the backward moves (N / 128) times the size of dQ
// in fp32 through the L2's reduction units; whether that is cheaper than the
// dQ kernel's two recomputed GEMMs is what this kernel measures.
//
// Per step, TMEM holds dK [0,128), dV [128,256), S^T [256,384) and dP^T
// [384,512) as in the dK/dV kernel; dQ_part is written over the dP^T columns
// once dK has consumed dS^T from them, and the element-wise warps read it out
// before the next dP^T.  dS (queries x keys) is the A operand of the dQ GEMM,
// so the element-wise warps also write it to shared memory, MN-major with the
// 128-byte swizzle, over the step's dO tile once the dV GEMM has read that
// tile; the whole stage (Q and dO tiles, 64 KB) then stages the fp32 dQ part
// for the bulk reduction before the stage is handed back to the loader.
#pragma once

#include "bwd_kernels.cuh"

namespace fa {

struct FusedCfg {
    static constexpr int D = 128;
    using B = BwdCfg<128>;
    static constexpr int NSTAGE = B::NSTAGE;
    static constexpr int TILE_BYTES = B::TILE_BYTES;    // 32 KB
    static constexpr int BOX = B::BOX;
    static constexpr int NBOX = B::NBOX;
    static constexpr int THREADS = B::THREADS;
    static constexpr uint32_t COL_ACC0 = B::COL_ACC0, COL_ACC1 = B::COL_ACC1, COL_S = B::COL_S,
                              COL_DP = B::COL_DP;
    static constexpr int OFF_FA = B::OFF_FA, OFF_FB = B::OFF_FB, OFF_ST = B::OFF_ST,
                         OFF_VEC = B::OFF_VEC;
    static constexpr int VEC_BYTES = B::VEC_BYTES;
    static constexpr int OFF_BAR = B::OFF_BAR;
    static constexpr int NBAR = 2 + 2 * NSTAGE + 6 + 3 + 3;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_SCRATCH = OFF_MISC + 16;
    static constexpr int OFF_PREFIX = OFF_SCRATCH + 2 * THREADS * 4;
    // block prefix, unit prefix, then the rank order (short[kMaxSortedSeqs])
    static constexpr int SMEM_BYTES = OFF_PREFIX + 2 * (kMaxVarlenSeqs + 1) * 4 + kMaxSortedSeqs * 2 + 1024;
};

struct FusedParams {
    BwdParams b;       // out0 = dK, out1 = dV
    float* dq_acc;     // [rows, H, 128] fp32, zeroed by the pre-pass
};

__global__ void __launch_bounds__(FusedCfg::THREADS, 1)
dkdvq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
             const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
             const FusedParams fp) {
    using C = FusedCfg;
    constexpr int D = 128;
    const BwdParams& p = fp.b;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    uint64_t* bb = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* fix_full = bb;
    uint64_t* fix_empty = bb + 1;
    uint64_t* stage_full = bb + 2;
    uint64_t* stage_empty = bb + 2 + C::NSTAGE;
    uint64_t* s_full = bb + 2 + 2 * C::NSTAGE;
    uint64_t* dp_full = s_full + 1;
    uint64_t* mid = dp_full + 1;          // [2 parts]
    uint64_t* ready = mid + 2;            // [2 parts]
    uint64_t* dv_done = ready + 2;        // the dV GEMM of the step has read dO
    uint64_t* dq_full = dv_done + 1;      // the step's dQ part is in TMEM
    uint64_t* drained = dq_full + 1;      // ... and has been read out of it
    uint64_t* acc_final = drained + 1;
    uint64_t* acc_empty = acc_final + 1;
    uint64_t* drain = acc_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    int* scratch = reinterpret_cast<int*>(smem + C::OFF_SCRATCH);
    int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);
    float* vec = reinterpret_cast<float*>(smem + C::OFF_VEC);   // per stage: x[128], y[128]
    const int warp = threadIdx.x >> 5;
    const int lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(fix_full, 1);
        mbar_init(fix_empty, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(stage_full + s, 1);
            mbar_init(stage_empty + s, 8);     // the element-wise warps, after the dQ part left
        }
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        for (int part = 0; part < 2; ++part) {
            mbar_init(mid + part, 8);
            mbar_init(ready + part, 8);
        }
        mbar_init(dv_done, 1);
        mbar_init(dq_full, 1);
        mbar_init(drained, 8);
        mbar_init(acc_final, 1);
        mbar_init(acc_empty, 8);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
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
    sch.rows_per_item = 128;
    sch.order = schedule_order(p.g, 0);     // key blocks: fewer queries see later keys
    sch.bprefix = prefix;
    sch.uprefix = prefix + kMaxVarlenSeqs + 1;
    sch.total_units = build_schedule_prefix(p.g, 128, prefix, prefix + kMaxVarlenSeqs + 1,
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
        if (warp == 0) {
            // ---------------------------------- producer (whole warp) --
            uint32_t cnt = 0, item_it = 0, fix_issued = 0;
            bool ok = true;
            ItemIter<true> it;
            int s, h, blk;
            for (; ok && it.next(sch, s, h, blk); ++item_it) {
                const SeqSpan sp = sch.span(s);
                const int n = sp.len;
                const int k0 = blk * 128;
                int ib, ie;
                query_tile_range(k0, min(n, k0 + 128), n, p.g.causal, p.g.window, 128, ib, ie);
                if (lane == 0) {
                    ok = mbar_wait(fix_empty, (item_it & 1) ^ 1, wc);
                    if (ok) {
                        mbar_arrive_expect_tx(fix_full, 2 * C::TILE_BYTES);
                        for (int b = 0; b < 2; ++b) {
                            tma_load_3d(smem + C::OFF_FA + b * C::BOX, &tm_k, fix_full, b * 64, h,
                                        sp.start + k0);
                            tma_load_3d(smem + C::OFF_FB + b * C::BOX, &tm_v, fix_full, b * 64, h,
                                        sp.start + k0);
                        }
                        ++fix_issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                const int blocks_before = sch.blocks_before(s);
                for (int i = ib; i < ie && ok; ++i, ++cnt) {
                    const int slot = cnt % C::NSTAGE;
                    if (lane == 0) {
                        ok = mbar_wait(stage_empty + slot, ((cnt / C::NSTAGE) & 1) ^ 1, wc);
                        if (ok) {
                            mbar_arrive_expect_tx(stage_full + slot, 2 * C::TILE_BYTES + C::VEC_BYTES);
                            uint8_t* st = smem + C::OFF_ST + slot * 2 * C::TILE_BYTES;
                            for (int b = 0; b < 2; ++b) {
                                tma_load_3d(st + b * C::BOX, &tm_q, stage_full + slot, b * 64, h,
                                            sp.start + i * 128);
                                tma_load_3d(st + C::TILE_BYTES + b * C::BOX, &tm_do, stage_full + slot,
                                            b * 64, h, sp.start + i * 128);
                            }
                            bulk_load(vec + slot * 256,
                                      p.stats + stats_index(p.g, p.stats_stride, s, h, blocks_before,
                                                            i * 128),
                                      C::VEC_BYTES, stage_full + slot);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                }
            }
            if (!ok && lane == 0) {
                for (uint32_t x = cnt > C::NSTAGE ? cnt - C::NSTAGE : 0; x < cnt; ++x)
                    drain_wait(stage_full + x % C::NSTAGE, (x / C::NSTAGE) & 1, p.error_word);
                if (fix_issued) drain_wait(fix_full, (fix_issued - 1) & 1, p.error_word);
            }
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------- MMA --
            // per step i:  [P^T_i] dV += P^T_i dO_i, S^T_{i+1}  ->  [dS^T_i]
            //              dK += dS^T_i Q_i, dQ_i = dS_i K  ->  [dQ_i read out] dP^T_{i+1}
            constexpr uint32_t IDESC_DQ = idesc_bf16(128, D, true, true);
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
                const int k0 = blk * 128;
                int ib, ie;
                query_tile_range(k0, min(n, k0 + 128), n, p.g.causal, p.g.window, 128, ib, ie);
                if (!mbar_wait(fix_full, item_it & 1, wc)) { ok = false; break; }
                if (!mbar_wait(acc_empty, (item_it & 1) ^ 1, wc)) { ok = false; break; }
                if (!mbar_wait(stage_full + cnt % C::NSTAGE, (cnt / C::NSTAGE) & 1, wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                {
                    const uint32_t x = st_addr + (cnt % C::NSTAGE) * 2 * C::TILE_BYTES;
                    issue_scores_ss<D>(tmem + C::COL_S, fa_addr, x);                  // K Q^T
                    umma_commit(s_full);
                    issue_scores_ss<D>(tmem + C::COL_DP, fb_addr, x + C::TILE_BYTES);  // V dO^T
                    umma_commit(dp_full);
                }
                for (int i = ib; i < ie; ++i, ++cnt) {
                    const bool last = (i + 1 == ie);
                    const uint32_t x = st_addr + (cnt % C::NSTAGE) * 2 * C::TILE_BYTES;
                    const uint32_t xn = st_addr + ((cnt + 1) % C::NSTAGE) * 2 * C::TILE_BYTES;
                    bool mok = true;
                    for (int part = 0; part < 2 && mok; ++part) {
                        if (!mbar_wait(mid + part, cnt & 1, wc)) { mok = false; break; }
                        tc_fence_after();
                        issue_acc_ts<D>(tmem + C::COL_ACC1, tmem + C::COL_S, x + C::TILE_BYTES,
                                        i > ib || part > 0, part);                      // dV
                    }
                    if (!mok) { ok = false; break; }
                    umma_commit(dv_done);
                    if (!last) {
                        if (!mbar_wait(stage_full + (cnt + 1) % C::NSTAGE, ((cnt + 1) / C::NSTAGE) & 1, wc)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_scores_ss<D>(tmem + C::COL_S, fa_addr, xn);             // next K Q^T
                        umma_commit(s_full);
                    }
                    for (int part = 0; part < 2 && mok; ++part) {
                        if (!mbar_wait(ready + part, cnt & 1, wc)) { mok = false; break; }
                        tc_fence_after();
                        issue_acc_ts<D>(tmem + C::COL_ACC0, tmem + C::COL_DP, x, i > ib || part > 0,
                                        part);                                          // dK
                    }
                    if (!mok) { ok = false; break; }
                    // dQ_i = dS_i K: A = dS (queries x keys) MN-major over the dO
                    // tile, B = K (keys x d) MN-major in the fixed tile
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ss(tmem + C::COL_DP,
                                sw128_desc(x + C::TILE_BYTES + kk * 2048, C::BOX, 1024),
                                sw128_desc(fa_addr + kk * 2048, C::BOX, 1024), IDESC_DQ, kk > 0);
                    umma_commit(dq_full);
                    if (last) {
                        umma_commit(acc_final);
                        umma_commit(fix_empty);
                    }
                    if (!mbar_wait(drained, cnt & 1, wc)) { ok = false; break; }
                    if (!last) {
                        tc_fence_after();
                        issue_scores_ss<D>(tmem + C::COL_DP, fb_addr, xn + C::TILE_BYTES);  // next V dO^T
                        umma_commit(dp_full);
                    }
                }
            }
            if (!ok) {
                umma_commit(drain);
                drain_wait(drain, 0, p.error_word);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------ element-wise warpgroups --
        regs_alloc<200>();
        const int g = (warp >> 2) - 1;             // 64-query half of each tile
        const int wq = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const int row = wq * 32 + lane;            // key row of S^T / query row of dQ
        const int ew = threadIdx.x - 128;          // 0 .. 255
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
            const int k0 = blk * 128;
            const int j = k0 + row;               // this thread's key
            int ib, ie;
            query_tile_range(k0, min(n, k0 + 128), n, p.g.causal, p.g.window, 128, ib, ie);
            // packed batches: the first row of the item's last query tile past the
            // batch's last sequence (128: none)
            const int dead_r0 = first_dead_row(p.g.cu_seqlens, p.g.B, sp.start + (ie - 1) * 128);
            // and of the item's own key block, whose K tile is the dQ GEMM's B operand
            const int dead_k0 = first_dead_row(p.g.cu_seqlens, p.g.B, sp.start + k0);
            for (int i = ib; i < ie; ++i, ++cnt) {
                const uint32_t slot = cnt % C::NSTAGE;
                uint8_t* stage = smem + C::OFF_ST + slot * 2 * C::TILE_BYTES;
                if (!mbar_wait(s_full, cnt & 1, wc)) { ok = false; break; }
                if (!mbar_wait(stage_full + slot, (cnt / C::NSTAGE) & 1, wc)) { ok = false; break; }
                if (i == ib && dead_k0 < 128) {
                    // K rows past the batch end meet dS = 0 in the dQ GEMM: zero them
                    // after the item's first K Q^T (no other reader is in flight)
                    zero_tile_rows(smem + C::OFF_FA, C::NBOX, dead_k0, ew, 256);
                }
                if (i + 1 == ie && dead_r0 < 128) {
                    // Q and dO rows past the batch end meet dS = 0 and P = 0 in the
                    // dK and dV GEMMs: zero them once both score GEMMs have read
                    // them, before either accumulation is released
                    if (!mbar_wait(dp_full, cnt & 1, wc)) { ok = false; break; }
                    zero_tile_rows(stage, C::NBOX, dead_r0, ew, 256);
                    zero_tile_rows(stage + C::TILE_BYTES, C::NBOX, dead_r0, ew, 256);
                }
                tc_fence_after();
                const float* xs = vec + slot * 256 + 64 * g;   // -L log2e
                const float* ys = xs + 128;                    // -D
                const int q0 = i * 128 + 64 * g;       // this half's first query
                const bool need_mask = (k0 + 128 > n) || (q0 + 64 > n) ||
                                       (p.g.causal && k0 + 127 > q0) ||
                                       (p.g.window > 0 && q0 + 63 - k0 >= p.g.window);
                uint32_t r[64];
                tmem_ld64(tS, r);
                tmem_wait_ld();
                float pf[64];
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    if (!need_mask) {
#pragma unroll
                        for (int c = 32 * part; c < 32 * part + 32; ++c)
                            pf[c] = ex2(fmaf(__uint_as_float(r[c]), sl2, xs[c]));
                    } else {
                        int c_lo, c_hi;      // this key's allowed queries of the half
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
                    tmem_st16(tS + 16 * part, pk);
                    arrive_warp(mid + part);
                }
                if (!mbar_wait(dp_full, cnt & 1, wc)) { ok = false; break; }
                tc_fence_after();
                tmem_ld64(tP, r);
                tmem_wait_ld();
                // dS goes over the dO tile once the dV GEMM has read it
                if (!mbar_wait(dv_done, cnt & 1, wc)) { ok = false; break; }
                uint8_t* sds = stage + C::TILE_BYTES + g * C::BOX;   // this half's 64 queries
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int k = 32 * part + 2 * c;
                        const float d0 = pf[k] * (__uint_as_float(r[k]) + ys[k]);
                        const float d1 = pf[k + 1] * (__uint_as_float(r[k + 1]) + ys[k + 1]);
                        pk[c] = pack_bf16(pf[k] != 0.f ? d0 : 0.f, pf[k + 1] != 0.f ? d1 : 0.f);
                    }
                    tmem_st16(tP + 16 * part, pk);   // dS^T for the dK GEMM
                    // dS for the dQ GEMM: key row `row`, queries 32 part .. +31 of
                    // this half = 16-byte chunks 4 part .. 4 part + 3 of the row,
                    // at the 128-byte-swizzled position of an MN-major operand
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int chunk = 4 * part + c;
                        uint4* dst = reinterpret_cast<uint4*>(
                            sds + (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
                        *dst = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                    }
                    fence_proxy_async_smem();
                    arrive_warp(ready + part);
                }
                // the dQ part: rows of TMEM are queries here; this half's 64 of
                // the 128 d columns, staged over the stage (both tiles are done)
                if (!mbar_wait(dq_full, cnt & 1, wc)) { ok = false; break; }
                tc_fence_after();
                tmem_ld64(tmem + lane_base + C::COL_DP + 64 * g, r);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(drained);
                float* stg = reinterpret_cast<float*>(stage) + ew * 64;
#pragma unroll
                for (int v = 0; v < 16; ++v)
                    reinterpret_cast<float4*>(stg)[v] =
                        make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                    __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
                fence_proxy_async_smem();
                const int q = i * 128 + row;
                if (q < n)
                    bulk_reduce_add_f32(fp.dq_acc + ((static_cast<size_t>(sp.start) + q) * H + h) * D + 64 * g,
                                        stg, 256);
                bulk_commit_group();
                bulk_wait_group_read0();
                __syncwarp();
                if (lane == 0) mbar_arrive(stage_empty + slot);
            }
            if (!ok) break;
            // ------------------------------------------------ epilogue --
            if (!mbar_wait(acc_final, item_it & 1, wc)) { ok = false; break; }
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
            if (lane == 0) mbar_arrive(acc_empty);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dQ = scale * dq_acc as bf16, eight elements per thread and step.
__global__ void __launch_bounds__(256)
dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, int64_t n8,
                  float scale) {
    for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < n8;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 a = reinterpret_cast<const float4*>(acc)[2 * v];
        const float4 b = reinterpret_cast<const float4*>(acc)[2 * v + 1];
        reinterpret_cast<uint4*>(dq)[v] =
            make_uint4(pack_bf16(a.x * scale, a.y * scale), pack_bf16(a.z * scale, a.w * scale),
                       pack_bf16(b.x * scale, b.y * scale), pack_bf16(b.z * scale, b.w * scale));
    }
}

// Workspace of the fused backward: the statistics array, then the fp32 dQ
// accumulator [rows, H, 128], 256-byte aligned.
inline size_t fused_stats_bytes(int B, int H, int64_t stride, bool packed) {
    return bwd_workspace_bytes(B, H, stride, packed);
}
inline size_t fused_workspace_bytes(int B, int H, int64_t stride, bool packed, int64_t rows) {
    return fused_stats_bytes(B, H, stride, packed) +
           static_cast<size_t>((rows * H * 128 * 4 + 255) / 256 * 256);
}

inline cudaError_t fused_set_smem_limit() {
    return cudaFuncSetAttribute(dkdvq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                FusedCfg::SMEM_BYTES);
}

// Pre-pass (statistics + zeroed accumulator), the fused kernel, the dQ
// conversion; hooks time kinds 1 (pre-pass), 2 (fused kernel), 3 (conversion).
inline cudaError_t bwd_fused_launch(const BwdArgs& a, const BwdMaps& m, float* dq_acc,
                                    cudaStream_t stream, const BwdHooks& hk) {
    constexpr int D = 128;
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
            a.stats, a.stats_stride, a.g, dq_acc);
        hk.stop(1, slot, stream);
    }
    FusedParams fp;
    BwdParams& p = fp.b;
    p.g = a.g;
    p.stats = a.stats;
    p.stats_stride = a.stats_stride;
    p.qrows = static_cast<const __nv_bfloat16*>(a.q);
    p.dorows = static_cast<const __nv_bfloat16*>(a.dO);
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    p.error_word = a.error_word;
    p.timeout_ns = a.timeout_ns;
    p.out0 = static_cast<__nv_bfloat16*>(a.dk);
    p.out1 = static_cast<__nv_bfloat16*>(a.dv);
    fp.dq_acc = dq_acc;
    int grid = a.num_sms;
    if (!a.g.cu_seqlens) {
        const int64_t items = static_cast<int64_t>(a.g.B) * a.g.H * ((a.g.N + 127) / 128);
        if (items < grid) grid = static_cast<int>(items);
    }
    int slot = hk.start(2, stream);
    dkdvq_kernel<<<grid, FusedCfg::THREADS, FusedCfg::SMEM_BYTES, stream>>>(m.k, m.v, m.q, m.dO, fp);
    hk.stop(2, slot, stream);
    const int64_t n8 = static_cast<int64_t>(a.g.T) * a.g.H * D / 8;
    int64_t cblocks = (n8 + 255) / 256;
    if (cblocks > static_cast<int64_t>(a.num_sms) * 16) cblocks = static_cast<int64_t>(a.num_sms) * 16;
    if (cblocks < 1) cblocks = 1;
    slot = hk.start(3, stream);
    dq_convert_kernel<<<static_cast<int>(cblocks), 256, 0, stream>>>(
        dq_acc, static_cast<__nv_bfloat16*>(a.dq), n8, a.scale);
    hk.stop(3, slot, stream);
    return cudaGetLastError();
}

}  // namespace fa
