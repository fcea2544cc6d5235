/*
 * fa.h -- C ABI of the B200 (sm_100a) exact IO-aware attention library.
 *
 * Operation (FlashAttention encyclopedia page, section "attention and the
 * memory bottleneck"): for every sequence and head,
 *     O = softmax(scale * Q K^T) V,
 * the softmax taken row by row over the keys the mask allows.  The forward
 * pass is one fused, tiled kernel that streams K/V tiles past an on-chip Q
 * tile and keeps the online-softmax state of each row on chip (same page,
 * "tiled computation and online normalisation"); it writes only O and the
 * per-row log-sum-exp, never the N x N score or probability matrix.  The
 * backward pass recomputes score tiles from that log-sum-exp instead of
 * storing probabilities (same page, "training and complexity": compact
 * normalisation statistics plus recomputation).
 *
 * Data layout (all tensors are caller-owned device memory; the library never
 * allocates, frees or keeps a reference past the call):
 *   q, k, v, o, dO, dq, dk, dv : bf16, token-major [tokens, H, d], contiguous,
 *       i.e. element (token t, head h, channel c) at ((t * H) + h) * d + c.
 *       Fixed length: tokens = B * N, sequence b at rows b*N .. b*N+N-1
 *       (the usual [B, N, H, d] tensor).  Packed variable length: tokens = T,
 *       sequence b at rows cu_seqlens[b] .. cu_seqlens[b+1]-1; rows past
 *       cu_seqlens[B] (a buffer larger than its batch) belong to no sequence,
 *       may hold anything (NaN included), and reach no result.
 *   lse : fp32 natural-log log-sum-exp of the scaled scores of each row,
 *       LSE_i = ln sum_j exp(scale * q_i . k_j) over allowed keys.
 *       Fixed length: [B, H, N].  Packed: [H, T].
 *   cu_seqlens : device int32, B + 1 non-decreasing offsets, cu_seqlens[0] = 0,
 *       cu_seqlens[B] <= T; NULL selects fixed length.
 *
 * Shape arguments: B sequences, H heads, d in {64, 128} channels per head.
 *   N is the sequence length for fixed-length inputs; for packed inputs N is
 *   the number of token rows T the buffers hold (the per-sequence lengths are
 *   read from cu_seqlens on the device, so no host synchronisation is needed).
 *   Packed batches hold at most 2048 sequences.
 *
 * Masks (row i, key j local to a sequence of n tokens; query and key sequences
 * have the same length except in fa_fwd_kv, below):
 *   causal != 0 : key j allowed only if j <= i (top-left aligned).
 *   window  > 0 : sliding window of exactly `window` keys ending at the
 *                 query's own position: allowed only if i - window < j <= i.
 *                 Requires causal != 0.  window >= n equals plain causal.
 *   window <= 0 : no window.
 *
 * scale: must be finite and > 0 (1/sqrt(d) for standard attention).
 *
 * Errors: every entry point returns FA_OK (0) or a negative fa_status.
 *   Argument errors are detected on the host before anything is launched.
 *   FA_ERR_CUDA means a launch or runtime call failed (cudaGetLastError is
 *   left set).  Kernels never trap: every wait inside them is bounded, and a
 *   wait that runs out records FA_ERR_DEVICE_TIMEOUT in a device error word
 *   that fa_get_device_error() reports.
 *
 * Asynchrony: the forward and backward entry points enqueue kernels on
 *   `stream` and return without synchronising; outputs are valid once the
 *   stream reaches them.
 *
 * Threads and devices: calls run on the calling thread's current CUDA
 *   device.  The first call on a device does a one-time set-up (SM count,
 *   the tensor-map encoder, the kernels' shared-memory limits) under a
 *   mutex; after it, calls from several host threads and on several streams
 *   are independent, except fa_bwd_noalloc (see there) and the per-thread
 *   profiling counters of fa_profile_begin/end.  The device error word is
 *   shared by all calls on a device.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_NULLPTR = -1,        /* a required pointer is NULL */
    FA_ERR_UNSUPPORTED_D = -2,  /* d not in {64, 128} */
    FA_ERR_BAD_SHAPE = -3,      /* negative sizes, too many packed sequences, size overflow */
    FA_ERR_MISALIGNED = -4,     /* a tensor base pointer is not 16-byte aligned */
    FA_ERR_BAD_MASK = -5,       /* window > 0 without causal */
    FA_ERR_WORKSPACE = -6,      /* workspace NULL or smaller than fa_bwd_workspace_size */
    FA_ERR_CUDA = -7,           /* CUDA runtime / launch failure */
    FA_ERR_DEVICE_TIMEOUT = -8, /* a bounded device-side wait gave up */
    FA_ERR_BAD_SCALE = -9,      /* scale not finite or not > 0 */
    FA_ERR_SCRATCH_LIMIT = -10  /* problem larger than fa_bwd_noalloc's built-in scratch */
} fa_status;

/*
 * Forward pass.  Writes o (bf16, layout of q) and lse (fp32, see above).
 * q, k, v are read only.  Rows of o/lse outside every sequence (packed
 * buffers with cu_seqlens[B] < T) are left untouched.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, float scale, int causal, int window,
           const int* cu_seqlens, cudaStream_t stream);

/*
 * Forward pass of queries against a longer cached key/value sequence
 * (prefill of a chunk of new tokens after earlier ones whose keys and values
 * are already computed).  Same operation as fa_fwd, with key/value sequences
 * that may differ in length from the query sequences; fa_fwd(..., N, ...) is
 * fa_fwd_kv(..., N, N, ..., cu_seqlens, cu_seqlens, ...).  The pages define
 * attention for any number of keys per query and name cached keys and values
 * as an interface (FlashAttention encyclopedia page, "software integration");
 * where the queries sit inside the key sequence they leave open, and this
 * library takes the reading that follows from prefill: the nq queries of a
 * sequence are its LAST nq positions, so query row i is at key position
 * i + nk - nq (bottom-right alignment) and the causal and window rules apply
 * to that position:
 *   causal : key j allowed only if j <= i + nk - nq,
 *   window : also only if j > i + nk - nq - window.
 * A query without any allowed key (nk = 0, or causal with i + nk - nq < 0)
 * gets O = 0 and LSE = -inf.
 *
 * q, o : [tokens_q, H, d]; k, v : [tokens_k, H, d]; lse as fa_fwd over the
 *   query rows ([B, H, Nq] fixed, [H, Tq] packed).
 * Fixed length (both cu_seqlens NULL): Nq queries and Nk keys per sequence,
 *   tokens_q = B * Nq, tokens_k = B * Nk.
 * Packed (both non-NULL; one NULL and one not is FA_ERR_BAD_SHAPE):
 *   cu_seqlens_q / cu_seqlens_k are device int32 arrays of B + 1 offsets into
 *   the query and key buffers; Nq and Nk are the token rows those buffers
 *   hold.  Per-sequence lengths may differ in either direction.
 * k and v may be NULL when the key buffers hold no rows (tokens_k = 0).
 * Errors as fa_fwd.  The backward entry points take equal query and key
 * lengths only.
 */
int fa_fwd_kv(const void* q, const void* k, const void* v, void* o, float* lse,
              int B, int H, int Nq, int Nk, int d, float scale, int causal, int window,
              const int* cu_seqlens_q, const int* cu_seqlens_k, cudaStream_t stream);

/*
 * Decode against a key/value cache, split along the keys.  A few new queries
 * per sequence (one per generated token; several for speculative decoding or
 * a short chunk) attend to the sequence's cached keys and values.  The pages
 * single out this shape: each step reads the whole accumulated K/V cache, so
 * it is bound by the cache's bandwidth rather than by matrix throughput
 * (IO-aware essay, section on training, prefill and per-token decode, and its
 * scenario table), and they list inference with cached keys and values among
 * the interfaces (FlashAttention encyclopedia page, "software integration").
 *
 * q, o    : [B, Nq, H, d] bf16 (Nq = 0 is a no-op).  Up to 16 queries per
 *           sequence run on a CUDA-core kernel built for the cache read;
 *           longer chunks (prefill of new tokens after cached ones) run on the
 *           tensor-core forward kernel, split along the keys the same way.
 * k_cache, v_cache : [B, Nk, H, d] bf16; sequence b uses rows 0 .. nk_b - 1
 *           of its slice, nk_b = seqlens_k[b] (device int32 [B], clamped to
 *           [0, Nk]) or Nk when seqlens_k is NULL.  Rows past nk_b are
 *           never read and may hold anything, NaN included (with Nq > 16 a
 *           key tile that would reach past nk_b is read as the 128 rows that
 *           end at nk_b, zeros before row 0, and its rows already covered by
 *           the tile before are masked out).  k_cache and v_cache may be NULL
 *           when B * Nk = 0.
 * lse     : [B, H, Nq] fp32, natural log.
 * Masks   : as fa_fwd_kv with the queries at the last Nq positions of the
 *           nk_b keys: query i is at position nk_b - Nq + i.
 * Splits  : the keys of each (sequence, head) are cut into num_splits
 *           contiguous ranges that run as separate CTAs (so that few
 *           sequences still fill the GPU); each writes a partial output and
 *           log-sum-exp to `workspace`, and a second kernel merges them.
 *           num_splits = 0 lets the library choose
 *           (fa_fwd_kvcache_num_splits returns that choice); 1 writes o and
 *           lse directly and needs no workspace; at most 32.
 * workspace : device memory of at least fa_fwd_kvcache_workspace_size(B, H,
 *           Nq, d, splits) bytes, 16-byte aligned, for splits > 1 (NULL
 *           otherwise); contents on entry do not matter.
 * Errors as fa_fwd; num_splits outside [0, 32] is FA_ERR_BAD_SHAPE, a
 * missing or short workspace FA_ERR_WORKSPACE.
 */
int fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, void* o,
                   float* lse, int B, int H, int Nq, int Nk, int d, float scale, int causal,
                   int window, const int* seqlens_k, int num_splits, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream);

/* The split count fa_fwd_kvcache uses for num_splits = 0 on the current
 * device (1 for empty problems). */
int fa_fwd_kvcache_num_splits(int B, int H, int Nq, int Nk, int d);

/* Workspace bytes fa_fwd_kvcache needs for `num_splits` splits:
 * num_splits * B * Nq * H * (d + 1) * 4 rounded up to 256, or 0 when
 * num_splits <= 1 or the problem is empty. */
size_t fa_fwd_kvcache_workspace_size(int B, int H, int Nq, int d, int num_splits);

/*
 * FP8 forward (block-quantised e4m3; NOT exact attention -- a separate,
 * lower-precision path).  The FlashAttention encyclopedia page (FlashAttention-3
 * paragraph) names an FP8 path with block quantisation and a processing step
 * that reduces quantisation error, to be kept apart from exact dense attention;
 * it prints no formulas, and this library reads it as follows (d = 128 and
 * fixed-length sequences only):
 *
 * fa_quantize_fp8: x bf16 [B, N, H, 128] -> e4m3 codes and one float scale per
 *   block of 128 rows of a head, scales [B, H, ceil(N/128)]: s = amax / 448
 *   (1 for an all-zero block), code = e4m3(x / s): the real quotient rounded
 *   once to the nearest e4m3 value, ties to even, saturating.  signs (128 floats of +-1, or NULL) selects the
 *   error-reducing rotation of each row before quantising: multiply by the
 *   signs, then the orthonormal Walsh-Hadamard transform (q.k is unchanged;
 *   use the same signs for Q and K).  transpose = 0 writes codes as
 *   [B, N, H, 128] (use for Q and K); transpose = 1 writes [B, H, 128, Np],
 *   Np = N rounded up to 16, zeros past N (use for V; signs must be NULL,
 *   else FA_ERR_BAD_SHAPE).  fa_fp8_vt_bytes gives that buffer's size.
 * fa_fwd_fp8: O (bf16 [B, N, H, 128]) and LSE ([B, H, N]) from the codes and
 *   scales: the softmax of the quantised scores (codes times block scales),
 *   with the probabilities rounded to e4m3 before they multiply the quantised
 *   V and the row sums taken from the unrounded ones.  Which reference the
 *   probabilities are rounded against is the kernel's: a running maximum
 *   raised only when it grows by more than 2^3 (base 2), with the V block
 *   scale folded in relative to the head's largest; the result lies within
 *   one e4m3 step of P per key of rounding against the row's final maximum.
 *   Masks as fa_fwd.
 * Errors as fa_fwd; d != 128 is FA_ERR_UNSUPPORTED_D.
 */
size_t fa_fp8_vt_bytes(int B, int H, int N, int d);
int fa_quantize_fp8(const void* x, void* out, float* scales, int B, int N, int H, int d,
                    int transpose, const float* signs, cudaStream_t stream);
int fa_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* sq,
               const float* sk, const float* sv, void* o, float* lse, int B, int H, int N,
               int d, float scale, int causal, int window, cudaStream_t stream);

/*
 * Bytes of device workspace fa_bwd needs: 8 bytes per (head, row) for the
 * per-row statistics {-LSE_i * log2(e), D_i = rowsum(dO_i * O_i)}, stored with
 * every sequence padded to a multiple of 128 rows.  Fixed length:
 * B * H * roundup(N, 128) * 8.  Packed: pass varlen_total = T and the number of
 * sequences B (N is ignored): H * roundup(T + 127 * B, 128) * 8.  Rounded up
 * to 256 bytes.  Returns 0 for H <= 0 or B <= 0.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d, int varlen_total);

/*
 * Backward pass (gradients of O = softmax(scale Q K^T) V).  Inputs: q, k, v,
 * the forward's o and lse, and dO (layout of o).  Outputs dq, dk, dv (bf16,
 * layout of q).  `workspace` is caller-owned device memory of at least
 * fa_bwd_workspace_size(...) bytes, 16-byte aligned; its contents on entry do
 * not matter and on exit are unspecified.  Shape and mask arguments as fa_fwd.
 *
 * The gradients follow from the definition (the pages print no formulas):
 *   P_ij = exp(scale s_ij - LSE_i),  D_i = dO_i . O_i,
 *   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . v_j - D_i),
 *   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv,
           int B, int H, int N, int d, float scale, int causal, int window,
           const int* cu_seqlens, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Single-kernel backward (d = 128 only): the same gradients as fa_bwd, with
 * dK, dV and the dQ contributions computed in one kernel that recomputes each
 * score and gradient tile once (five GEMMs per key tile x query tile pair
 * instead of fa_bwd's seven).  The pages say only that the backward pass
 * recomputes attention blocks from compact normalisation statistics
 * (FlashAttention encyclopedia page, "training and complexity"); this entry
 * point is the variant that trades fa_bwd's second recomputation for an fp32
 * reduction of every tile's dQ part into an accumulator in the workspace
 * (through the L2's reduction units), then a scaling kernel writes bf16 dQ.
 * Results equal fa_bwd's up to the order of the fp32 additions into dQ, which
 * is not fixed (the reductions of different key tiles land in any order), so
 * dQ is not bit-reproducible from run to run; dK and dV are.
 *
 * Arguments as fa_bwd; `workspace` must hold fa_bwd_fused_workspace_size(...)
 * bytes (the statistics array plus rows x H x 128 floats) and be 256-byte
 * aligned; its contents on entry do not matter.  d != 128 returns
 * FA_ERR_UNSUPPORTED_D; fa_bwd_fused_workspace_size returns 0 for it.
 */
size_t fa_bwd_fused_workspace_size(int B, int H, int N, int d, int varlen_total);
int fa_bwd_fused(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv,
                 int B, int H, int N, int d, float scale, int causal, int window,
                 const int* cu_seqlens, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream);

/*
 * fa_bwd_noalloc: the backward pass for callers that cannot allocate device
 * memory -- for example a plugin inside a framework or runtime that owns every
 * device allocation and has no way to hand this library a workspace, or a
 * serving loop that must not allocate once it is running.  It computes exactly
 * what fa_bwd computes, with the same arguments minus the workspace: the
 * per-row statistics live in a fixed device array built into the library
 * instead (FA_NOALLOC_MAX_ROWS entries of 8 bytes, 8 MiB, held on every GPU
 * that loads the library until the process exits).  The pages have no
 * counterpart of this entry point; it only changes where the scratch lives.
 *
 * - The limit is on the workspace, not on H * N alone: a call fits when
 *   fa_bwd_workspace_size(B, H, N, d, packed ? N : 0) <= 8 * FA_NOALLOC_MAX_ROWS,
 *   where each sequence counts its length rounded up to a multiple of 128
 *   rows, once per head (fixed length: B * H * ceil(N / 128) * 128 entries;
 *   packed: H * (N + 127 * B) rounded up to 128).  So H = 16, N = 65536
 *   fits, H = 16, N = 65537 does not.  Larger problems return
 *   FA_ERR_SCRATCH_LIMIT and launch nothing; use fa_bwd for them.
 * - It calls no cudaMalloc / cudaFree and no allocating library routine.
 * - The first call on a device looks up the array's device address (a
 *   one-time set-up with that device current).
 * - All calls share the one array per device and leave their per-row
 *   statistics in it; every call rewrites the part it uses before reading
 *   it.  Calls whose kernels overlap on the GPU (different streams, or
 *   different host threads) race on the array: serialise them.
 */
#define FA_NOALLOC_MAX_ROWS (1 << 20)
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, float scale, int causal, int window,
                   const int* cu_seqlens, cudaStream_t stream);

/* Static, human-readable text for a status code. */
const char* fa_status_string(int status);

/*
 * Synchronises `stream`, then returns FA_ERR_DEVICE_TIMEOUT if any kernel of
 * this library on the current device recorded a bounded-wait timeout since the
 * last call (and clears the record), FA_ERR_CUDA if the synchronisation
 * failed, else FA_OK.
 */
int fa_get_device_error(cudaStream_t stream);

/*
 * Per-kernel device timing.  fa_profile_begin() resets the counters and makes
 * the following calls of the entry points above on the calling thread's current device
 * record a CUDA event pair on the launch stream around each kernel they launch
 * (up to 1024 launches per kernel kind; later ones are not recorded).
 * fa_profile_end() waits for the recorded events, stops recording, and writes
 * for each kind k (0 forward, 1 D pre-pass, 2 dK/dV, 3 dQ, 4 decode, 5 decode
 * split merge, 6 FP8 quantisation, 7 FP8 forward, 8 single-kernel backward,
 * 9 its dQ conversion) the summed device
 * milliseconds ms[k] and the number of recorded launches counts[k] (arrays of
 * FA_PROFILE_KINDS entries).
 * Either output pointer may be NULL.  The events are created once per device
 * on the first fa_profile_begin() call.
 */
#define FA_PROFILE_KINDS 10
int fa_profile_begin(void);
int fa_profile_end(double* ms, int* counts);

/*
 * While profiling is on, each forward launch (fa_fwd, fa_fwd_kv and the
 * prefill path of fa_fwd_kvcache) also records the start and end time of
 * every CTA of its persistent grid.  fa_profile_cta_balance() synchronises
 * the device and reports, for the last such launch, the mean CTA busy time
 * over the largest one (1 = every SM busy until the last one finishes) and
 * the grid size.  The first fa_profile_begin() on a device allocates the
 * small timing buffer this needs (profiling only; no other entry point
 * allocates).
 */
int fa_profile_cta_balance(double* balance, int* ctas);

/*
 * Test hook for the failure path.  mode 0: normal operation.  mode 1: the
 * next fa_fwd launches make their load warp skip the first V tile, so the
 * consumer's bounded wait runs out after timeout_ns nanoseconds (0 keeps the
 * default of 2 s) and the kernel returns with FA_ERR_DEVICE_TIMEOUT recorded.
 * mode 2: the same for the decode kernel of fa_fwd_kvcache (queries <= 16):
 * each CTA's load thread leaves its first K/V stage unloaded.
 * Host-side setting, not thread safe; returns the previous mode.
 */
int fa_debug_set_fault(int mode, unsigned long long timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
