/*
 * fp8_oracle.c -- CPU oracle for the FP8 forward pass (block-quantised e4m3
 * attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Like attn_oracle.c it is loaded by the tests,
 * the smoke check and the benchmark's CPU leg, never by the product path, and
 * shares no code, header or table with the CUDA sources.
 *
 * The FlashAttention encyclopedia page (section on the versions, the
 * FlashAttention-3 paragraph) says that the FP8 path adds block quantisation
 * and a processing step that reduces quantisation error, and that such
 * low-precision execution is to be kept apart from exact dense attention at
 * higher precision.  It prints no formulas.  This file writes out, step by
 * step, the reading the CUDA path implements:
 *
 *  1. Error-reducing rotation (optional) of every q and k row, d = 128:
 *     multiply element-wise by a random sign vector, then apply the
 *     orthonormal Walsh-Hadamard transform -- butterflies (a, b) ->
 *     (a + b, a - b) on element pairs (j, j + h) for h = 1, 2, 4, ..., 64 in
 *     that order, then a factor 1/sqrt(128).  The rotation is orthogonal, so
 *     every q.k is unchanged while outliers are spread over all channels.
 *  2. Block scales: for every block of 128 rows of one head (rows past the
 *     sequence end excluded), s = amax / 448 (448 is the largest finite
 *     e4m3 value; s = 1 for an all-zero block), and codes c = e4m3(x * inv)
 *     with inv = 1 / s rounded to float32 once per block (one multiply per
 *     element instead of a division; the two readings of "x over s" differ
 *     only where x / s and x * inv fall on opposite sides of an e4m3
 *     rounding boundary).
 *     Steps 1-2 decide integer codes, so they are taken in float32, the
 *     precision the CUDA kernel takes them in; every float operation here is
 *     a single IEEE-754 float32 operation (no fused multiply-add).
 *  3. Forward, in float64 from the codes: for each query row the 128-key
 *     blocks are visited in order with the online normalisation of the
 *     encyclopedia page, section "tiled computation and online
 *     normalisation", in base 2 and with the reference maximum raised only
 *     when a block's maximum exceeds it by more than 8 (the exponentials
 *     then stay <= 2^8, inside e4m3's range):
 *        x_j = (c_q . c_k_j) * scale * log2(e) * s_q * s_k(block of j)
 *        p_j = 2^(x_j - m),  l += p_j
 *        P_j = e4m3(p_j * r_b),  r_b = min(1, s_v(b) / max_b' s_v(b'))
 *        acc += P_j * c_v_j
 *     and O = acc * max_b s_v(b) / l, LSE = ln 2 * (m + log2 l).  The V
 *     block scales are folded into P relative to the head's largest one so
 *     that a single fp32 accumulator serves all blocks.
 *
 * Return value 0 = ok, -3 = bad shape, -5 = window without causal.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define BLK 128

/* The e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities) value nearest to x, ties to even, saturating at +-448; NaN
 * stays NaN.  Below 2^-6 the spacing is that of the 2^-6 binade (2^-9,
 * subnormals). */
static double e4m3_round_d(double x)
{
    if (x != x) return x;
    const double a = fabs(x);
    if (a >= 448.0) return copysign(448.0, x);
    int e;
    frexp(a, &e);                       /* a = f * 2^e, f in [0.5, 1) */
    int E = e - 1;                      /* floor(log2 a) */
    if (E < -6) E = -6;
    const double q = ldexp(1.0, E - 3); /* spacing of 3 mantissa bits */
    const double n = nearbyint(a / q);  /* round half to even (default mode) */
    return copysign(n * q, x);
}

float oracle_e4m3_round(float x) { return (float)e4m3_round_d((double)x); }

static void fwht128(float *y)
{
    for (int h = 1; h < BLK; h <<= 1)
        for (int i = 0; i < BLK; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                const float a = y[j], b = y[j + h];
                y[j] = a + b;
                y[j + h] = a - b;
            }
    const float c = 0.08838834764831845f;   /* 1/sqrt(128), rounded to float */
    for (int j = 0; j < BLK; ++j) y[j] = y[j] * c;
}

/* Step 1 on its own: rows [rows, d] (d = 128) rotated in place. */
int oracle_rotate_rows(float *x, int rows, int d, const float *signs)
{
    if (d != BLK || rows < 0 || !signs) return -3;
    for (int r = 0; r < rows; ++r) {
        float *y = x + (size_t)r * d;
        for (int c = 0; c < d; ++c) y[c] = y[c] * signs[c];
        fwht128(y);
    }
    return 0;
}

/* Steps 1-2.  x: [B * N, H, d] float32 (exact bf16 values), fixed length N.
 * signs: d entries of +-1 or NULL (no rotation).  codes: same layout as x
 * (the e4m3 values); scales: [B, H, nb], nb = ceil(N / 128). */
int oracle_quantize_fp8(const float *x, int B, int N, int H, int d, const float *signs,
                        float *codes, float *scales)
{
    if (B < 0 || N < 0 || H <= 0 || d != BLK) return -3;
    const int nb = (N + BLK - 1) / BLK;
    float *y = (float *)malloc(sizeof(float) * BLK * BLK);
    if (!y) return -3;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int blk = 0; blk < nb; ++blk) {
                const int r0 = blk * BLK, r1 = (r0 + BLK < N) ? r0 + BLK : N;
                float amax = 0.0f;
                for (int r = r0; r < r1; ++r) {
                    float *yr = y + (size_t)(r - r0) * d;
                    const float *xr = x + (((size_t)b * N + r) * H + h) * d;
                    memcpy(yr, xr, sizeof(float) * d);
                    if (signs) {
                        for (int c = 0; c < d; ++c) yr[c] = yr[c] * signs[c];
                        fwht128(yr);
                    }
                    for (int c = 0; c < d; ++c) {
                        const float v = fabsf(yr[c]);
                        if (v > amax) amax = v;
                    }
                }
                const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
                const float inv = 1.0f / s;
                scales[((size_t)b * H + h) * nb + blk] = s;
                for (int r = r0; r < r1; ++r) {
                    const float *yr = y + (size_t)(r - r0) * d;
                    float *cr = codes + (((size_t)b * N + r) * H + h) * d;
                    for (int c = 0; c < d; ++c) cr[c] = oracle_e4m3_round(yr[c] * inv);
                }
            }
    free(y);
    return 0;
}

static int allowed(int i, int j, int causal, int window)
{
    if (causal && j > i) return 0;
    if (window > 0 && j <= i - window) return 0;
    return 1;
}

/* Step 3.  qc, kc, vc: [B * N, H, d] code values; sq, sk, sv: [B, H, nb].
 * quantize_p = 0 skips the e4m3 rounding of P (with unit scales and exact
 * values this is then the exact forward).  o: [B * N, H, d]; lse: [B, H, N]. */
int oracle_fwd_fp8(const float *qc, const float *kc, const float *vc, const float *sq,
                   const float *sk, const float *sv, int B, int N, int H, int d, double scale,
                   int causal, int window, int quantize_p, double *o, double *lse)
{
    if (B < 0 || N < 0 || H <= 0 || d <= 0) return -3;
    if (window > 0 && !causal) return -5;
    const int nb = (N + BLK - 1) / BLK;
    const double log2e = 1.4426950408889634;
    #pragma omp parallel for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < N; ++i) {
                const float *sv_bh = sv + ((size_t)b * H + h) * nb;
                double svmax = 0.0;
                for (int j = 0; j < nb; ++j)
                    if (sv_bh[j] > svmax) svmax = sv_bh[j];
                const float *qr = qc + (((size_t)b * N + i) * H + h) * d;
                const double sqi = sq[((size_t)b * H + h) * nb + i / BLK];
                double *acc = o + (((size_t)b * N + i) * H + h) * d;
                for (int c = 0; c < d; ++c) acc[c] = 0.0;
                double m = -INFINITY, l = 0.0;
                double xs[BLK];
                for (int kb = 0; kb < nb; ++kb) {
                    const double skb = sk[((size_t)b * H + h) * nb + kb];
                    const int j0 = kb * BLK, j1 = (j0 + BLK < N) ? j0 + BLK : N;
                    double mx = -INFINITY;
                    for (int j = j0; j < j1; ++j) {
                        xs[j - j0] = -INFINITY;
                        if (!allowed(i, j, causal, window)) continue;
                        const float *kr = kc + (((size_t)b * N + j) * H + h) * d;
                        double s = 0.0;
                        for (int c = 0; c < d; ++c) s += (double)qr[c] * (double)kr[c];
                        xs[j - j0] = s * scale * log2e * sqi * skb;
                        if (xs[j - j0] > mx) mx = xs[j - j0];
                    }
                    if (mx == -INFINITY) continue;          /* nothing allowed in this block */
                    const double m_new = mx > m ? mx : m;
                    if (m_new > m + 8.0) {
                        const double alpha = exp2(m - m_new);   /* 0 on the first block */
                        l *= alpha;
                        for (int c = 0; c < d; ++c) acc[c] *= alpha;
                        m = m_new;
                    }
                    double r = svmax > 0.0 ? sv_bh[kb] / svmax : 1.0;
                    if (r > 1.0) r = 1.0;
                    for (int j = j0; j < j1; ++j) {
                        if (xs[j - j0] == -INFINITY) continue;
                        const double p = exp2(xs[j - j0] - m);
                        l += p;
                        const double pq = quantize_p ? e4m3_round_d(p * r) : p * r;
                        const float *vr = vc + (((size_t)b * N + j) * H + h) * d;
                        for (int c = 0; c < d; ++c) acc[c] += pq * (double)vr[c];
                    }
                }
                const double f = l > 0.0 ? svmax / l : 0.0;
                for (int c = 0; c < d; ++c) acc[c] *= f;
                lse[((size_t)b * H + h) * N + i] = l > 0.0 ? log(2.0) * (m + log2(l)) : -INFINITY;
            }
    return 0;
}
