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

constexpr int kMaxVarlenSeqs = 4096;   // sequences a packed batch may hold

struct Geometry {
    int B;                  // sequences
    int H;                  // heads
    int N;                  // fixed length; 0 for packed batches
    int T;                  // token rows of the [T, H, d] buffers
    const int* cu_seqlens;  // device, B + 1 entries, or nullptr
    int causal;
    int window;             // <= 0: none
};

struct SeqSpan {
    int start;
    int len;
};

// Allowed-key test for one (row, key) pair inside a sequence.
__device__ __forceinline__ bool key_allowed(int i, int j, int n, int causal, int window) {
    return j < n && (!causal || j <= i) && (window <= 0 || j > i - window);
}

// Key-tile range [jb, je) that query rows [r_lo, r_hi) of a sequence of
// length n need, for key tiles of BN keys; tiles outside it are fully masked
// and never loaded.
__device__ __forceinline__ void key_tile_range(int r_lo, int r_hi, int n, int causal, int window,
                                               int BN, int& jb, int& je) {
    int k_lo = 0;
    if (window > 0) k_lo = max(0, r_lo - window + 1);
    int k_hi = causal ? min(n, r_hi) : n;
    jb = k_lo / BN;
    je = (k_hi + BN - 1) / BN;
    if (je < jb) je = jb;
}

// True when some pair of (rows [r0, r0+BM), keys [k0, k0+BN)) is masked out,
// so the tile needs the element-wise mask.
__device__ __forceinline__ bool tile_needs_mask(int r0, int BM, int k0, int BN, int n, int causal,
                                                int window) {
    if (k0 + BN > n) return true;
    if (causal && k0 + BN - 1 > r0) return true;
    if (window > 0 && k0 <= r0 + BM - 1 - window) return true;
    return false;
}

// Static persistent schedule.  Work items are (sequence, head, block of
// `rows_per_item` rows); item w goes to CTA w % gridDim.x.  Items are ordered
// sequence-major, then head, then block, so the CTAs running at the same time
// share K/V of few heads in L2; with `heavy_first` the blocks of a head are
// visited from the last (most keys under a causal mask) to the first.
struct Schedule {
    Geometry g;
    int rows_per_item;
    int heavy_first;
    const int* prefix;      // shared memory: prefix[s] = sum of blocks of sequences < s
    int total_items;

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

    // Decode item w into (sequence, head, block).
    __device__ __forceinline__ void item(int w, int& s, int& h, int& blk) const {
        int nb;
        int local;
        if (!g.cu_seqlens) {
            nb = blocks_of(g.N);
            s = w / (g.H * nb);
            local = w - s * g.H * nb;
        } else {
            // binary search: largest s with prefix[s] * H <= w
            int lo = 0, hi = g.B - 1;
            while (lo < hi) {
                int mid = (lo + hi + 1) >> 1;
                if (prefix[mid] * g.H <= w) lo = mid; else hi = mid - 1;
            }
            s = lo;
            nb = prefix[s + 1] - prefix[s];
            local = w - prefix[s] * g.H;
        }
        h = local / nb;
        blk = local - h * nb;
        if (heavy_first) blk = nb - 1 - blk;
    }
};

// Build the per-sequence block prefix in shared memory (packed batches only)
// and return the number of work items.  All threads of the CTA call it.
__device__ __forceinline__ int build_schedule_prefix(const Geometry& g, int rows_per_item,
                                                     int* prefix, int* scratch /* blockDim */) {
    if (!g.cu_seqlens) {
        int nb = (g.N + rows_per_item - 1) / rows_per_item;
        return g.B * g.H * nb;
    }
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (g.B + nt - 1) / nt;
    const int s0 = min(g.B, tid * per), s1 = min(g.B, s0 + per);
    int run = 0;
    for (int s = s0; s < s1; ++s) {
        int len = g.cu_seqlens[s + 1] - g.cu_seqlens[s];
        run += (len + rows_per_item - 1) / rows_per_item;
        prefix[s + 1] = run;          // local inclusive prefix for now
    }
    scratch[tid] = run;
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int t = 0; t < nt; ++t) { int v = scratch[t]; scratch[t] = acc; acc += v; }
        prefix[0] = 0;
    }
    __syncthreads();
    const int off = scratch[tid];
    for (int s = s0; s < s1; ++s) prefix[s + 1] += off;
    __syncthreads();
    return prefix[g.B] * g.H;
}

}  // namespace fa
