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
    int Nk;                 // fixed key length
    int Tk;                 // token rows of the key/value buffers
    const int* cu_seqlens_k;
};

struct SeqSpan {
    int start;
    int len;
};

// Allowed-key test for one (row, key) pair inside a sequence.
__device__ __forceinline__ bool key_allowed(int i, int j, int n, int causal, int window) {
    return j < n && (!causal || j <= i) && (window <= 0 || j > i - window);
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
// blocks of `rows_per_item` rows; a work unit is the pair of blocks p and
// nb-1-p of one (sequence, head) (the middle block alone when nb is odd), so
// that under a causal mask -- where a block's cost grows or shrinks linearly
// with its index -- every unit costs the same.  Units are ordered sequence-
// major, then head, then p, so the CTAs running at the same time share K/V of
// few heads in L2; unit w goes to CTA w % gridDim.x.
struct Schedule {
    Geometry g;
    int rows_per_item;
    const int* bprefix;     // shared memory: blocks of the sequences before s (packed only)
    const int* uprefix;     // shared memory: units of the sequences before s (packed only)
    int total_units;

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
            // binary search: largest s with uprefix[s] * H <= w
            int lo = 0, hi = g.B - 1;
            while (lo < hi) {
                int mid = (lo + hi + 1) >> 1;
                if (uprefix[mid] * g.H <= w) lo = mid; else hi = mid - 1;
            }
            s = lo;
            nu = uprefix[s + 1] - uprefix[s];
            nb = bprefix[s + 1] - bprefix[s];
            local = w - uprefix[s] * g.H;
        }
        h = local / nu;
        p = local - h * nu;
    }
};

// Walks the blocks one CTA processes: its units in order, both blocks of each.
struct ItemIter {
    int w;
    int half;
    __device__ __forceinline__ ItemIter() : w(blockIdx.x), half(0) {}
    __device__ __forceinline__ bool next(const Schedule& sch, int& s, int& h, int& blk) {
        while (w < sch.total_units) {
            int p, nb;
            sch.unit(w, s, h, p, nb);
            if (half == 0) {
                half = 1;
                blk = p;
                return true;
            }
            half = 0;
            w += gridDim.x;
            if (nb - 1 - p != p) {
                blk = nb - 1 - p;
                return true;
            }
        }
        return false;
    }
};

// Build the per-sequence block and unit prefixes in shared memory (packed
// batches only) and return the number of work units.  All threads of the CTA
// call it.
__device__ __forceinline__ int build_schedule_prefix(const Geometry& g, int rows_per_item,
                                                     int* bprefix, int* uprefix,
                                                     int* scratch /* 2 * blockDim */) {
    if (!g.cu_seqlens) {
        const int nb = (g.N + rows_per_item - 1) / rows_per_item;
        return g.B * g.H * ((nb + 1) >> 1);
    }
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (g.B + nt - 1) / nt;
    const int s0 = min(g.B, tid * per), s1 = min(g.B, s0 + per);
    int runb = 0, runu = 0;
    for (int s = s0; s < s1; ++s) {
        const int len = g.cu_seqlens[s + 1] - g.cu_seqlens[s];
        const int nb = (len + rows_per_item - 1) / rows_per_item;
        runb += nb;
        runu += (nb + 1) >> 1;
        bprefix[s + 1] = runb;          // local inclusive prefixes for now
        uprefix[s + 1] = runu;
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
    for (int s = s0; s < s1; ++s) {
        bprefix[s + 1] += ob;
        uprefix[s + 1] += ou;
    }
    __syncthreads();
    return uprefix[g.B] * g.H;
}

}  // namespace fa
