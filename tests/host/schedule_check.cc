// Host build of the kernels' tile schedule and mask classification
// (io_aware_exact_21_b200/csrc/schedule.cuh), checked for the invariants the
// kernels rely on:
//   1. every (sequence, head, row block) is visited by exactly one CTA, for
//      the pair walk and the pair + snake-tail walk, for fixed-length and
//      packed batches and for several grid sizes;
//   2. the key-tile range of a block holds every key any of its rows may see,
//      and the tiles outside it hold none;
//   3. a tile classified as needing no mask has every (row, key) pair of the
//      block allowed;
//   4. the column ranges the kernels mask with (tile_key_bounds for a row
//      against a key tile, tile_query_bounds for a key against a query tile)
//      hold exactly the pairs key_allowed allows;
//   5. first_dead_row finds the first tile row past a packed batch's end;
//   6. the singles walk visits every block exactly once.
// The CUDA built-ins the header reads (blockIdx, gridDim, threadIdx,
// blockDim, __syncthreads) are host variables here; the packed-batch prefix
// is built by one emulated thread.  Prints "ok" and exits 0, or names the
// first violation and exits 1.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <random>
#include <tuple>
#include <vector>

#define __device__
#define __forceinline__ inline
using std::max;
using std::min;
struct Dim3 {
    unsigned x = 0, y = 1, z = 1;
};
static Dim3 blockIdx, gridDim, threadIdx, blockDim;
static inline void __syncthreads() {}

#include "schedule.cuh"

namespace {

int failures = 0;

void fail(const char* what, int a, int b, int c, int d) {
    if (failures++ < 10) std::printf("FAIL %s (%d %d %d %d)\n", what, a, b, c, d);
}

// Visit every CTA's walk and count the (s, h, blk) it yields.  Packed batches
// of up to kMaxSortedSeqs sequences are dealt longest first (the schedule
// derives that from the geometry).  Returns the largest per-CTA cost over the
// mean per-CTA cost, a block's cost taken as the keys it sees under a causal
// mask (or all of them).
template <bool kTail>
double check_cover(const fa::Geometry& g, const std::vector<int>& lens, int rows_per_item, int order,
                   int G) {
    // the unit prefix is followed by the rank order (kMaxSortedSeqs shorts)
    std::vector<int> bpre(fa::kMaxVarlenSeqs + 1), upre(fa::kMaxVarlenSeqs + 1 + fa::kMaxSortedSeqs);
    std::vector<int> scratch(2);
    fa::Schedule sch;
    sch.g = g;
    sch.rows_per_item = rows_per_item;
    sch.order = order;
    sch.bprefix = bpre.data();
    sch.uprefix = upre.data();
    blockDim.x = 1;
    threadIdx.x = 0;
    gridDim.x = G;
    sch.total_units = fa::build_schedule_prefix(g, rows_per_item, bpre.data(), upre.data(),
                                                scratch.data());
    if (sch.ranked()) {
        // the ranks are a permutation, longest first
        const short* rank_seq = sch.ranked_seqs();
        std::vector<int> hit(g.B, 0);
        for (int r = 0; r < g.B; ++r) {
            const int sr = rank_seq[r];
            if (sr < 0 || sr >= g.B || hit[sr]++) fail("rank order is not a permutation", r, sr, g.B, 0);
            else if (r > 0 && lens[rank_seq[r - 1]] < lens[sr]) fail("rank order not longest first", r, sr, 0, 0);
        }
    }
    fa::schedule_split_tail(sch);
    std::map<std::tuple<int, int, int>, int> seen;
    std::vector<double> cost(G, 0.0);
    for (int c = 0; c < G; ++c) {
        blockIdx.x = c;
        fa::ItemIter<kTail> it;
        int s, h, blk, guard = 0;
        while (it.next(sch, s, h, blk)) {
            if (++guard > 1000000) {
                fail("walk does not end", c, G, rows_per_item, order);
                return 0.0;
            }
            ++seen[std::make_tuple(s, h, blk)];
            const int hi = min(lens[s], (blk + 1) * rows_per_item);
            cost[c] += g.causal ? hi : lens[s];
        }
    }
    size_t expected = 0;
    for (int s = 0; s < g.B; ++s) {
        const int n = lens[s];
        const int nb = (n + rows_per_item - 1) / rows_per_item;
        for (int h = 0; h < g.H; ++h)
            for (int b = 0; b < nb; ++b) {
                ++expected;
                auto f = seen.find(std::make_tuple(s, h, b));
                const int cnt = f == seen.end() ? 0 : f->second;
                if (cnt != 1) fail("block visited != once", s, h, b, cnt);
            }
    }
    if (seen.size() != expected) fail("walk yields blocks outside the batch", (int)seen.size(),
                                      (int)expected, G, order);
    double mx = 0.0, tot = 0.0;
    for (double v : cost) {
        mx = std::max(mx, v);
        tot += v;
    }
    return tot > 0.0 ? mx / (tot / G) : 1.0;
}

void check_masks(std::mt19937& rng) {
    const int BN = 128;
    for (int trial = 0; trial < 400; ++trial) {
        const int nk = 1 + rng() % 1500;
        const int nq = 1 + rng() % nk;              // queries: the last nq key positions
        const int off = nk - nq;
        const int causal = rng() % 4 != 0;
        const int window = causal && rng() % 2 ? 1 + rng() % 300 : 0;
        const int rows = rng() % 2 ? 128 : 256;
        for (int r_lo = 0; r_lo < nq; r_lo += rows) {
            const int r_hi = min(nq, r_lo + rows);
            int jb, je;
            fa::key_tile_range(r_lo + off, r_hi + off, nk, causal, window, BN, jb, je);
            if (jb < 0 || je <= jb) fail("empty or negative tile range", jb, je, nk, nq);
            const int ntiles = (nk + BN - 1) / BN;
            for (int t = 0; t < max(ntiles, je); ++t) {
                bool any = false, all = true;
                for (int i = r_lo; i < r_hi; ++i)
                    for (int k = t * BN; k < (t + 1) * BN; ++k) {
                        const bool a = fa::key_allowed(i + off, k, nk, causal, window);
                        any = any || a;
                        all = all && a;
                    }
                const bool inside = t >= jb && t < je;
                if (any && !inside) fail("allowed key outside the tile range", t, jb, je, nk);
                if (inside && !fa::tile_needs_mask_pos(r_lo + off, r_hi + off, t * BN, BN, nk,
                                                       causal, window) && !all)
                    fail("unmasked tile holds a disallowed pair", t, r_lo, nk, window);
            }
        }
    }
}

void check_bounds(std::mt19937& rng) {
    for (int trial = 0; trial < 3000; ++trial) {
        const int n = 1 + rng() % 700;
        const int causal = rng() % 3 != 0;
        const int window = rng() % 2 ? 1 + rng() % 400 : 0;
        const int BN = rng() % 2 ? 128 : 64;
        const int nk = n + (rng() % 2 ? 0 : static_cast<int>(rng() % 300));   // cached keys before the queries
        const int off = nk - n;
        // a row against key tiles (query positions shifted by off, keys of nk)
        const int i = rng() % n;
        for (int k0 = 0; k0 < nk + BN; k0 += BN) {
            int lo, hi;
            fa::tile_key_bounds(i + off, k0, nk, causal, window, BN, lo, hi);
            if (lo < 0 || hi < lo || hi > BN) fail("key bounds out of range", lo, hi, BN, k0);
            for (int c = 0; c < BN; ++c)
                if ((c >= lo && c < hi) != fa::key_allowed(i + off, k0 + c, nk, causal, window))
                    fail("tile_key_bounds disagrees with key_allowed", i, k0, c, window);
        }
        // a key against query tiles (self-attention, n rows, queries past n
        // allowed nothing)
        const int j = rng() % (n + 3);
        for (int q0 = 0; q0 < n + BN; q0 += 64) {
            int lo, hi;
            fa::tile_query_bounds(j, q0, n, causal, window, BN, lo, hi);
            if (lo < 0 || hi < lo || hi > BN) fail("query bounds out of range", lo, hi, BN, q0);
            for (int c = 0; c < BN; ++c) {
                const bool want = q0 + c < n && fa::key_allowed(q0 + c, j, n, causal, window);
                if ((c >= lo && c < hi) != want) fail("tile_query_bounds disagrees with key_allowed", j, q0, c, window);
            }
        }
    }
}

}  // namespace

// The singles walk (fixed length; every block its own unit, dealt in snake
// rounds): every (sequence, head, block) exactly once, for several grids.
void check_singles() {
    for (int B : {1, 3, 4})
        for (int H : {1, 5, 16})
            for (int N : {1, 255, 256, 257, 2048, 3000})
                for (int G : {1, 7, 148, 1000}) {
                    fa::Geometry g{};
                    g.B = B;
                    g.H = H;
                    g.N = N;
                    g.T = B * N;
                    fa::Schedule sch{};
                    sch.g = g;
                    sch.rows_per_item = 256;
                    const int nb = (N + 255) / 256;
                    sch.total_units = B * H * nb;
                    gridDim.x = G;
                    std::map<std::tuple<int, int, int>, int> seen;
                    for (int c = 0; c < G; ++c) {
                        blockIdx.x = c;
                        fa::ItemIter<true, true> it;
                        int s, h, blk, guard = 0;
                        while (it.next(sch, s, h, blk)) {
                            if (++guard > 100000) {
                                fail("singles walk does not end", c, G, N, 0);
                                break;
                            }
                            if (s < 0 || s >= B || h < 0 || h >= H || blk < 0 || blk >= nb)
                                fail("singles walk leaves the batch", s, h, blk, G);
                            ++seen[std::make_tuple(s, h, blk)];
                        }
                    }
                    if (static_cast<int>(seen.size()) != B * H * nb)
                        fail("singles walk misses blocks", (int)seen.size(), B * H * nb, G, N);
                    for (auto& kv : seen)
                        if (kv.second != 1) fail("singles block visited != once", std::get<0>(kv.first),
                                                 std::get<1>(kv.first), std::get<2>(kv.first), kv.second);
                }
}

// The singles walk over packed batches (unit prefix in blocks, ranked
// longest first up to kMaxSortedSeqs sequences, in index order above):
// every (sequence, head, block) exactly once.
void check_singles_packed(std::mt19937& rng) {
    for (int trial = 0; trial < 40; ++trial) {
        const int B = trial < 30 ? 1 + static_cast<int>(rng() % 20) : 250 + static_cast<int>(rng() % 20);
        const int H = 1 + static_cast<int>(rng() % 4);
        std::vector<int> lens(B), cu(B + 1, 0);
        for (int s = 0; s < B; ++s) {
            lens[s] = (rng() % 5 == 0) ? 0 : static_cast<int>(rng() % 1500);
            cu[s + 1] = cu[s] + lens[s];
        }
        fa::Geometry g{};
        g.B = B;
        g.H = H;
        g.N = 0;
        g.T = cu[B];
        g.cu_seqlens = cu.data();
        std::vector<int> bpre(fa::kMaxVarlenSeqs + 1), upre(fa::kMaxVarlenSeqs + 1 + fa::kMaxSortedSeqs);
        std::vector<int> scratch(2);
        blockDim.x = 1;
        threadIdx.x = 0;
        fa::Schedule sch{};
        sch.g = g;
        sch.rows_per_item = 256;
        sch.bprefix = bpre.data();
        sch.uprefix = upre.data();
        sch.total_units = fa::build_schedule_prefix(g, 256, bpre.data(), upre.data(), scratch.data(), true, true);
        for (int G : {1, 13, 148}) {
            gridDim.x = G;
            std::map<std::tuple<int, int, int>, int> seen;
            for (int c = 0; c < G; ++c) {
                blockIdx.x = c;
                fa::ItemIter<true, true> it;
                int s, h, blk, guard = 0;
                while (it.next(sch, s, h, blk)) {
                    if (++guard > 1000000) {
                        fail("packed singles walk does not end", c, G, B, 0);
                        break;
                    }
                    ++seen[std::make_tuple(s, h, blk)];
                }
            }
            size_t expected = 0;
            for (int s = 0; s < B; ++s)
                for (int h = 0; h < H; ++h)
                    for (int b = 0; b < (lens[s] + 255) / 256; ++b) {
                        ++expected;
                        auto f = seen.find(std::make_tuple(s, h, b));
                        if (f == seen.end() || f->second != 1)
                            fail("packed singles block visited != once", s, h, b, f == seen.end() ? 0 : f->second);
                    }
            if (seen.size() != expected) fail("packed singles walk leaves the batch", (int)seen.size(), (int)expected, G, B);
        }
    }
}

// first_dead_row against a row-by-row count: the first row of a 128-row tile
// at global row row0 that lies at or past cu[B] (128 if none); no rows are
// dead without a packed batch.
void check_dead_rows(std::mt19937& rng) {
    for (int trial = 0; trial < 2000; ++trial) {
        const int B = 1 + static_cast<int>(rng() % 6);
        std::vector<int> cu(B + 1, 0);
        for (int s = 0; s < B; ++s) cu[s + 1] = cu[s] + static_cast<int>(rng() % 400);
        const int row0 = static_cast<int>(rng() % (cu[B] + 1));
        int want = 128;
        for (int r = 0; r < 128; ++r)
            if (row0 + r >= cu[B]) {
                want = r;
                break;
            }
        const int got = fa::first_dead_row(cu.data(), B, row0);
        if (got != want) fail("first_dead_row", row0, cu[B], got, want);
        if (fa::first_dead_row(nullptr, B, row0) != 128) fail("first_dead_row without cu", row0, 0, 0, 0);
    }
}

int main() {
    std::mt19937 rng(12345);
    // fixed length: pairs, and pairs + snake tail in both cost directions
    const int grids[] = {1, 7, 148, 300};
    const int shapes[][3] = {{4, 16, 8192}, {4, 16, 2048}, {2, 16, 4096}, {1, 1, 128},
                             {3, 5, 1000}, {1, 2, 65536}, {64, 32, 128}, {2, 3, 257}};
    for (auto& sh : shapes) {
        for (int causal = 0; causal < 2; ++causal) {
            fa::Geometry g{};
            g.B = sh[0];
            g.H = sh[1];
            g.N = sh[2];
            g.T = sh[0] * sh[2];
            g.causal = causal;
            g.Nk = sh[2];
            g.Tk = g.T;
            std::vector<int> lens(g.B, g.N);
            for (int G : grids)
                for (int rows : {128, 256}) {
                    check_cover<false>(g, lens, rows, 0, G);
                    const int order = fa::schedule_order(g, 1);
                    check_cover<true>(g, lens, rows, order, G);
                    check_cover<true>(g, lens, rows, -order, G);
                }
        }
    }
    // packed batches (pairs only): random lengths, including empty sequences
    for (int trial = 0; trial < 30; ++trial) {
        const int B = 1 + rng() % 40;
        std::vector<int> lens(B), cu(B + 1, 0);
        for (int s = 0; s < B; ++s) {
            lens[s] = rng() % 5 == 0 ? 0 : 1 + rng() % 3000;
            cu[s + 1] = cu[s] + lens[s];
        }
        fa::Geometry g{};
        g.B = B;
        g.H = 1 + rng() % 8;
        g.N = 0;
        g.T = cu[B];
        g.cu_seqlens = cu.data();
        g.causal = rng() % 2;
        g.Nk = 0;
        g.Tk = g.T;
        g.cu_seqlens_k = cu.data();
        for (int G : grids) check_cover<false>(g, lens, 256, 0, G);
        for (int G : grids) check_cover<true>(g, lens, 128, fa::schedule_order(g, 1), G);
    }
    // the packed workload shape (16 sequences of 128..4096 tokens, 32 heads,
    // causal, 148 CTAs): longest-first snake dealing balances the CTAs at
    // least as well as dealing in sequence order, across many draws
    {
        double worst_plain = 0.0, worst_ranked = 0.0;
        for (int trial = 0; trial < 50; ++trial) {
            const int B = 16;
            std::vector<int> lens(B), cu(B + 1, 0);
            for (int s = 0; s < B; ++s) {
                lens[s] = 128 + rng() % 3969;
                cu[s + 1] = cu[s] + lens[s];
            }
            fa::Geometry g{};
            g.B = B;
            g.H = 32;
            g.T = cu[B];
            g.cu_seqlens = cu.data();
            g.causal = 1;
            g.Tk = g.T;
            g.cu_seqlens_k = cu.data();
            for (int rows : {128, 256}) {
                const double ranked = check_cover<false>(g, lens, rows, 0, 148);
                // the same units dealt round robin in sequence order
                std::vector<double> cost(148, 0.0);
                int w = 0;
                for (int sq = 0; sq < B; ++sq) {
                    const int nb = (lens[sq] + rows - 1) / rows;
                    for (int h = 0; h < g.H; ++h)
                        for (int p = 0; p < (nb + 1) / 2; ++p, ++w) {
                            cost[w % 148] += min(lens[sq], (p + 1) * rows);
                            if (nb - 1 - p != p) cost[w % 148] += min(lens[sq], (nb - p) * rows);
                        }
                }
                double mx = 0.0, tot = 0.0;
                for (double v : cost) {
                    mx = std::max(mx, v);
                    tot += v;
                }
                worst_plain = std::max(worst_plain, mx / (tot / 148));
                worst_ranked = std::max(worst_ranked, ranked);
            }
        }
        if (worst_ranked > worst_plain || worst_ranked > 1.12)
            fail("longest-first dealing does not balance the packed workload",
                 (int)(1000 * worst_ranked), (int)(1000 * worst_plain), 0, 0);
        std::fprintf(stderr, "packed workload, worst max/mean CTA cost: in order %.3f, longest first %.3f\n",
                     worst_plain, worst_ranked);
    }
    check_masks(rng);
    check_bounds(rng);
    check_dead_rows(rng);
    check_singles();
    check_singles_packed(rng);
    if (failures) {
        std::printf("%d violations\n", failures);
        return 1;
    }
    std::printf("ok\n");
    return 0;
}
