// schedule.cuh -- sequence geometry, mask classification and the static
// persistent tile schedule shared by the forward and backward kernels.
//
// Masks (FlashAttention encyclopedia page, "attention and the memory
// bottleneck": a mask restricts which query/key pairs interact; "software
// integration": causal, sliding-window and variable-length inputs).  Row i and
// key j are positions inside one sequence of length n:
//   key j exists            iff j < n
//   causal                  iff j <= i
//   sliding window of W > 0 iff i - W < j   (W keys including the query itself)
#pragma once

#include <stdint.h>

namespace fa {

constexpr int kMaxVarlenSeqs = 2048;   // sequences a packed batch may hold
constexpr int kMaxSortedSeqs = 256;    // packed batches up to this size are dealt longest first

struct Geometry {
    int B;                  // sequences
    int H;                  // heads
    int N;                  // fixed length of the query sequences; 0 for packed batches
    int T;                  // token rows of the query buffers [T, H, d]
    const int* cu_seqlens;  // device, B + 1 entries, or nullptr
    int causal;
    int window;             // <= 0: none
    // Key/value sequences (equal to the query ones for self-attention).  The
    // queries of a sequence are the last ones of its key sequence, so query
    // row i sits at key position i + (nk - nq).
    int Nk;                 // fixed key length (the rows of each sequence's slice)
    int Tk;                 // token rows of the key/value buffers
    const int* cu_seqlens_k;
};

// Rows of a packed batch's buffers past cu_seqlens[B] hold no sequence (a
// buffer may be larger than the batch) and may hold anything, NaN included.
// A 128-row tile that reaches past that end is loaded whole by TMA; where its
// rows would meet the tensor core in a product whose other factor is a masked
// zero (P = 0 times a V row, dS = 0 times a K, Q or dO row), 0 * NaN would
// still be NaN, so the kernels zero those rows in shared memory first
// (zero_tile_rows in dead_rows.cuh).  first_dead_row gives the first such
// row of a tile that starts at global row `row0`, or 128 when it has none
// (fixed-length batches never have any: their buffers end with the batch).
__device__ __forceinline__ int first_dead_row(const int* cu, int B, int row0) {
    if (!cu) return 128;
    const int end = cu[B];
    return row0 + 128 <= end ? 128 : max(0, end - row0);
}

struct SeqSpan {
    int start;
    int len;
};

// Allowed-key test for one (row, key) pair inside a sequence.
__device__ __forceinline__ bool key_allowed(int i, int j, int n, int causal, int window) {
    return j < n && (!causal || j <= i) && (window <= 0 || j > i - window);
}

// The same test for one row against a tile, as a column range: key k0 + c is
// allowed for row position ip iff c_lo <= c < c_hi (0 <= c_lo <= c_hi <= BN),
// so a masked tile costs two compares per element.
__device__ __forceinline__ void tile_key_bounds(int ip, int k0, int nk, int causal, int window, int BN,
                                                int& c_lo, int& c_hi) {
    int hi = nk - k0;                                    // k0 + c < nk
    if (causal) hi = min(hi, ip - k0 + 1);               // k0 + c <= ip
    const int lo = window > 0 ? max(0, ip - window + 1 - k0) : 0;   // k0 + c > ip - window
    c_lo = min(lo, BN);
    c_hi = max(c_lo, min(hi, BN));
}

// And for one key against a tile of queries (self-attention, n rows): query
// q0 + c may attend key j iff c_lo <= c < c_hi (0 <= c_lo <= c_hi <= BM);
// queries past n get none.
__device__ __forceinline__ void tile_query_bounds(int j, int q0, int n, int causal, int window, int BM,
                                                  int& c_lo, int& c_hi) {
    int hi = n - q0;                                     // q0 + c < n
    if (j >= n) hi = 0;                                  // the key itself exists
    if (window > 0) hi = min(hi, j + window - q0);       // j > q0 + c - window
    const int lo = causal ? max(0, j - q0) : 0;          // j <= q0 + c
    c_lo = min(lo, BM);
    c_hi = max(c_lo, min(hi, BM));
}

// Key-tile range [jb, je) that queries at key positions [p_lo, p_hi) need in
// a key sequence of length nk, for key tiles of BN keys; tiles outside it are
// fully masked and never loaded.  An empty range becomes one (fully masked)
// tile, so every block runs the same protocol and its queries without any
// allowed key come out as O = 0, LSE = -inf.
__device__ __forceinline__ void key_tile_range(int p_lo, int p_hi, int nk, int causal, int window,
                                               int BN, int& jb, int& je) {
    int k_lo = 0;
    if (window > 0) k_lo = max(0, p_lo - window + 1);
    int k_hi = causal ? min(nk, p_hi) : nk;
    jb = k_lo / BN;
    je = (k_hi + BN - 1) / BN;
    if (je <= jb) je = jb + 1;
}

// True when some pair of (queries at key positions [p0, p_end), keys
// [k0, k0+BN)) is masked out, so the tile needs the element-wise mask.
// p_end excludes rows past the query sequence end: their results are never
// stored, and ignoring them makes the decision depend only on the mask's
// meaning (a window of n or more keys classifies every tile like causal).
__device__ __forceinline__ bool tile_needs_mask_pos(int p0, int p_end, int k0, int BN, int nk,
                                                    int causal, int window) {
    if (k0 + BN > nk) return true;
    if (p0 < 0) return true;
    if (causal && k0 + BN - 1 > p0) return true;
    if (window > 0 && k0 <= p_end - 1 - window) return true;
    return false;
}

// Self-attention form: rows [r0, r0+BM) of a sequence of n tokens.
__device__ __forceinline__ bool tile_needs_mask(int r0, int BM, int k0, int BN, int n, int causal,
                                                int window) {
    return tile_needs_mask_pos(r0, min(r0 + BM, n), k0, BN, n, causal, window);
}

// Static persistent schedule.  The rows of a (sequence, head) are cut into
// blocks of `rows_per_item` rows, and each CTA walks its own list of blocks;
// every role of a CTA walks the same list independently.
//
// Pairs: a work unit is the pair of blocks p and nb-1-p of one (sequence,
// head) (the middle block alone when nb is odd), so that under a causal mask
// -- where a block's cost grows or shrinks linearly with its index -- every
// unit of a sequence costs the same.  Units are ordered sequence-major, then
// head, then p, so the CTAs running at the same time share K/V of few heads
// in L2; unit w goes to CTA w % gridDim.x.  This is the whole schedule for
// fixed length without a causal or window mask.
//
// Packed batches, longest first: a unit's cost grows with its sequence's
// length, so with up to kMaxSortedSeqs sequences the sequences are ranked by
// length (longest first, ties by index) and the units follow that order;
// they are dealt in rounds of gridDim.x, forwards in even rounds and
// backwards in odd ones (a "snake"), so that every CTA's list runs from
// costly units to cheap ones and the costs even out across CTAs (a greedy
// longest-first assignment in the usual sense).
//
// Pairs + snake tail (every kernel but the cached-KV forward, for fixed length
// with a causal or window mask, where a block's cost is monotone in its
// index): when the units per CTA are few, the last round of units leaves up
// to a unit's worth of imbalance.  So only the whole heads that fit in all
// rounds but the last go out as units; the blocks of the remaining heads are
// sorted heaviest first (block index major, then head) and dealt one by one
// in rounds of gridDim.x CTAs, forwards in even rounds and backwards in odd
// ones, starting at the CTA after the last unit.
// `order` is +1 when cost grows with the block index (query blocks), -1 when
// it shrinks (key blocks), 0 for pairs alone.
struct Schedule {
    Geometry g;
    int rows_per_item;
    int order;              // 0: pairs; +1 / -1: snake tail, heaviest block last / first
    int bulk_units;         // snake tail: units dealt as pairs
    int tail_sh0;           // snake tail: first (sequence, head) of the tail
    int tail_heads;         //   (sequence, head)s in the tail
    int tail_c0;            //   CTA that takes the tail's first block
    const int* bprefix;     // shared memory: blocks of the sequences before s (packed only)
    const int* uprefix;     // shared memory: units of the sequences ranked before r (packed
                            // only), followed by the sequence of each rank (ranked_seqs)
    int total_units;

    // Packed batches of up to kMaxSortedSeqs sequences are dealt longest first
    // (build_schedule_prefix ranks them).  Derived from the geometry rather
    // than stored: a field more stays live in a register across every role's
    // loop, which measurably slows the kernels.
    __device__ __forceinline__ bool ranked() const {
        return g.cu_seqlens != nullptr && g.B <= kMaxSortedSeqs;
    }
    __device__ __forceinline__ const short* ranked_seqs() const {
        return reinterpret_cast<const short*>(uprefix + kMaxVarlenSeqs + 1);
    }

    __device__ __forceinline__ int blocks_of(int len) const {
        return (len + rows_per_item - 1) / rows_per_item;
    }

    __device__ __forceinline__ SeqSpan span(int s) const {
        if (g.cu_seqlens) {
            int a = g.cu_seqlens[s];
            return SeqSpan{a, g.cu_seqlens[s + 1] - a};
        }
        return SeqSpan{s * g.N, g.N};
    }

    // Key/value span of sequence s.
    __device__ __forceinline__ SeqSpan kspan(int s) const {
        if (g.cu_seqlens_k) {
            int a = g.cu_seqlens_k[s];
            return SeqSpan{a, g.cu_seqlens_k[s + 1] - a};
        }
        return SeqSpan{s * g.Nk, g.Nk};
    }

    // Key/value span of sequence s in a padded cache (fixed length): the
    // first seqused_k[s] rows of its Nk-row slice (all Nk when seqused_k is null).
    __device__ __forceinline__ SeqSpan kspan_used(int s, const int* seqused_k) const {
        const int used = seqused_k ? min(max(seqused_k[s], 0), g.Nk) : g.Nk;
        return SeqSpan{s * g.Nk, used};
    }

    // Blocks of the sequences before s (packed batches; 0 for fixed length).
    __device__ __forceinline__ int blocks_before(int s) const {
        return g.cu_seqlens ? bprefix[s] : 0;
    }

    // Decode unit w into (sequence, head, first block p, blocks of the sequence nb).
    __device__ __forceinline__ void unit(int w, int& s, int& h, int& p, int& nb) const {
        int nu, local;
        if (!g.cu_seqlens) {
            nb = blocks_of(g.N);
            nu = (nb + 1) >> 1;
            s = w / (g.H * nu);
            local = w - s * g.H * nu;
        } else {
            // binary search: largest rank r with uprefix[r] * H <= w
            int lo = 0, hi = g.B - 1;
            while (lo < hi) {
                int mid = (lo + hi + 1) >> 1;
                if (uprefix[mid] * g.H <= w) lo = mid; else hi = mid - 1;
            }
            s = ranked() ? ranked_seqs()[lo] : lo;
            nu = uprefix[lo + 1] - uprefix[lo];
            nb = bprefix[s + 1] - bprefix[s];
            local = w - uprefix[lo] * g.H;
        }
        h = local / nu;
        p = local - h * nu;
    }
};

// Walks the blocks one CTA processes: its units in order, both blocks of each
// (pairs), then, with kTail and a non-zero order, its blocks of the snake
// tail round by round.  Without kTail the walk is pairs alone.
//
// kSingles: every block is a unit of its own, in sequence-major (packed:
// rank-major, longest first), head, block order, dealt in rounds of
// gridDim.x CTAs, forwards in even rounds and backwards in odd ones.  For blocks of similar
// cost (a chunk of queries after a long cached prefix) this balances as well
// as pairs do, and the CTAs that run at the same time then share the K/V of
// about gridDim.x / (blocks per head) heads -- half as many as with pairs,
// whose two blocks of a head run one after the other on one CTA -- so the
// heads in flight fit in L2.  total_units is then the number of blocks times
// H (build_schedule_prefix with singles = true).  kMayPack = false leaves
// out the packed decoding for callers that are fixed-length by construction.
template <bool kTail, bool kSingles = false, bool kMayPack = true>
struct ItemIter {
    int w;        // pairs: next unit
    int half;
    int round;    // snake tail (and singles): next round
    __device__ __forceinline__ ItemIter() : w(blockIdx.x), half(0), round(0) {}
    __device__ __forceinline__ bool next(const Schedule& sch, int& s, int& h, int& blk) {
        if constexpr (kSingles) {
            const int G = gridDim.x;
            const int x = static_cast<int>(blockIdx.x);
            const int u = round * G + ((round & 1) ? G - 1 - x : x);
            if (u >= sch.total_units) return false;
            ++round;
            if (kMayPack && sch.g.cu_seqlens) {
                // packed (build_schedule_prefix with singles): the unit prefix
                // counts blocks, in rank order
                int lo = 0, hi = sch.g.B - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (sch.uprefix[mid] * sch.g.H <= u) lo = mid; else hi = mid - 1;
                }
                s = sch.ranked() ? sch.ranked_seqs()[lo] : lo;
                const int nb = sch.uprefix[lo + 1] - sch.uprefix[lo];
                const int local = u - sch.uprefix[lo] * sch.g.H;
                h = local / nb;
                blk = local - h * nb;
                return true;
            }
            const int nb = sch.blocks_of(sch.g.N);
            const int per_seq = sch.g.H * nb;
            s = u / per_seq;
            const int local = u - s * per_seq;
            h = local / nb;
            blk = local - h * nb;
            return true;
        }
        const int limit = (kTail && sch.order != 0) ? sch.bulk_units : sch.total_units;
        while (w < limit) {
            int p, nb;
            sch.unit(w, s, h, p, nb);
            if (half == 0) {
                half = 1;
                blk = p;
                return true;
            }
            half = 0;
            // the next round's unit: forwards in even rounds, backwards in odd
            // ones when the units run longest first, else w + gridDim.x
            if (sch.ranked()) {
                const int G = gridDim.x;
                const int r = w / G + 1;
                w = r * G + ((r & 1) ? G - 1 - static_cast<int>(blockIdx.x)
                                     : static_cast<int>(blockIdx.x));
            } else {
                w += gridDim.x;
            }
            if (nb - 1 - p != p) {
                blk = nb - 1 - p;
                return true;
            }
        }
        if (!kTail || sch.order == 0) return false;
        const int G = gridDim.x;
        const int x0 = (static_cast<int>(blockIdx.x) - sch.tail_c0 + G) % G;
        const int r = round * G + ((round & 1) ? G - 1 - x0 : x0);
        const int nb = sch.blocks_of(sch.g.N);
        if (r >= sch.tail_heads * nb) return false;
        ++round;
        const int q = r / sch.tail_heads;              // rank of the block index, heaviest first
        const int sh = sch.tail_sh0 + (r - q * sch.tail_heads);
        blk = sch.order > 0 ? nb - 1 - q : q;
        s = sh / sch.g.H;
        h = sh - s * sch.g.H;
        return true;
    }
};

// Fill in the snake-tail split (see Schedule) once total_units is known.
__device__ __forceinline__ void schedule_split_tail(Schedule& sch) {
    sch.bulk_units = sch.total_units;
    sch.tail_sh0 = 0;
    sch.tail_heads = 0;
    sch.tail_c0 = 0;
    if (sch.order == 0) return;
    const int G = gridDim.x;
    const int nu = (sch.blocks_of(sch.g.N) + 1) >> 1;
    if (nu == 0) return;
    const int rounds = max(0, sch.total_units / G - 1);
    sch.bulk_units = (rounds * G / nu) * nu;
    sch.tail_sh0 = sch.bulk_units / nu;
    sch.tail_heads = sch.g.B * sch.g.H - sch.tail_sh0;
    sch.tail_c0 = sch.bulk_units % G;
}

// The order a kernel uses: snake for fixed length under a causal or window
// mask, with the direction in which its blocks' cost grows; pairs otherwise.
__device__ __forceinline__ int schedule_order(const Geometry& g, int cost_grows_with_index) {
    if (g.cu_seqlens || (!g.causal && g.window <= 0)) return 0;
    return cost_grows_with_index ? 1 : -1;
}

// Build the per-sequence block prefix (in sequence order) and the unit prefix
// (in rank order) in shared memory (packed batches only) and return the number
// of work units.  `uprefix` must have room for kMaxVarlenSeqs + 1 ints and,
// right after them, kMaxSortedSeqs shorts: with at most kMaxSortedSeqs
// sequences (Schedule::ranked) the ranks are by length, longest first (ties
// by index), and the sequence of each rank is stored there
// (Schedule::ranked_seqs); otherwise the rank is the index.  With
// `with_rank` false only the block prefix is needed (the unit prefix is then
// in sequence order).  All threads of the CTA call it.
__device__ __forceinline__ int build_schedule_prefix(const Geometry& g, int rows_per_item,
                                                     int* bprefix, int* uprefix,
                                                     int* scratch /* 2 * blockDim */,
                                                     bool with_rank = true, bool singles = false) {
    if (!g.cu_seqlens) {
        const int nb = (g.N + rows_per_item - 1) / rows_per_item;
        return g.B * g.H * (singles ? nb : ((nb + 1) >> 1));
    }
    const bool sort = with_rank && g.B <= kMaxSortedSeqs;
    short* rank_seq = reinterpret_cast<short*>(uprefix + kMaxVarlenSeqs + 1);
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (g.B + nt - 1) / nt;
    const int s0 = min(g.B, tid * per), s1 = min(g.B, s0 + per);
    // raw per-sequence counts: blocks at the sequence's index, units at its rank
    for (int s = s0; s < s1; ++s) {
        const int len = g.cu_seqlens[s + 1] - g.cu_seqlens[s];
        const int nb = (len + rows_per_item - 1) / rows_per_item;
        bprefix[s + 1] = nb;
        int r = s;
        if (sort) {
            r = 0;
            for (int o = 0; o < g.B; ++o) {
                const int lo = g.cu_seqlens[o + 1] - g.cu_seqlens[o];
                r += (lo > len) || (lo == len && o < s);
            }
            rank_seq[r] = static_cast<short>(s);
        }
        uprefix[r + 1] = singles ? nb : (nb + 1) >> 1;
    }
    __syncthreads();
    // inclusive prefix sums over [1, B]: per-thread chunks, then chunk offsets
    int runb = 0, runu = 0;
    for (int x = s0; x < s1; ++x) {
        runb += bprefix[x + 1];
        bprefix[x + 1] = runb;
        runu += uprefix[x + 1];
        uprefix[x + 1] = runu;
    }
    scratch[tid] = runb;
    scratch[nt + tid] = runu;
    __syncthreads();
    if (tid == 0) {
        int ab = 0, au = 0;
        for (int t = 0; t < nt; ++t) {
            const int vb = scratch[t], vu = scratch[nt + t];
            scratch[t] = ab;
            scratch[nt + t] = au;
            ab += vb;
            au += vu;
        }
        bprefix[0] = 0;
        uprefix[0] = 0;
    }
    __syncthreads();
    const int ob = scratch[tid], ou = scratch[nt + tid];
    for (int x = s0; x < s1; ++x) {
        bprefix[x + 1] += ob;
        uprefix[x + 1] += ou;
    }
    __syncthreads();
    return uprefix[g.B] * g.H;
}

}  // namespace fa
