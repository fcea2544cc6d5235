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
 * higher precision.  It prints no formulas.  This file writes out the plain
 * reading of block-quantised attention, step by step:
 *
 *  1. Error-reducing rotation (optional) of every q and k row, d = 128:
 *     multiply element-wise by a random sign vector, then apply the
 *     orthonormal Walsh-Hadamard transform -- butterflies (a, b) ->
 *     (a + b, a - b) on element pairs (j, j + h) for h = 1, 2, 4, ..., 64 in
 *     that order, then a factor 1/sqrt(128).  The rotation is orthogonal, so
 *     every q.k is unchanged while outliers are spread over all channels.
 *     Its values are the inputs of integer decisions (the codes), so they are
 *     taken in float32, one IEEE-754 operation at a time (no fused
 *     multiply-add).
 *  2. Block scales: for every block of 128 rows of one head (rows past the
 *     sequence end excluded), s = amax / 448 in float32 (448 is the largest
 *     finite e4m3 value; s = 1 for an all-zero block), and codes
 *     c = e4m3(x / s): the real quotient rounded once to the nearest e4m3
 *     value, ties to even, saturating at +-448.  (The quotient of two float32
 *     numbers is taken in float64; no float64 quotient lies on an e4m3
 *     rounding boundary unless the real one does, so this is the exactly
 *     rounded code.)
 *  3. Forward from the codes, in float64: the codes times their block scales
 *     are the quantised operands q^, k^, v^; per query row the scores
 *     x_j = scale q^.k^_j over the allowed keys, the row maximum m, the
 *     exponentials p_j = exp(x_j - m) and their sum l (the softmax statistics
 *     are not matmul operands and keep full precision), and the output
 *        O = sum_j e4m3(p_j) v^_j / l,     LSE = m + ln l,
 *     i.e. the probabilities are quantised to e4m3 against the row maximum
 *     (p <= 1) before they multiply V.  This is the exact softmax of the
 *     quantised scores, with no tiling: how a kernel walks the keys is not
 *     part of what the method computes.
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
                scales[((size_t)b * H + h) * nb + blk] = s;
                for (int r = r0; r < r1; ++r) {
                    const float *yr = y + (size_t)(r - r0) * d;
                    float *cr = codes + (((size_t)b * N + r) * H + h) * d;
                    for (int c = 0; c < d; ++c)
                        cr[c] = (float)e4m3_round_d((double)yr[c] / (double)s);
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
 * quantize_p = 0 skips the e4m3 rounding of p (with unit scales and exact
 * values this is then the exact forward).  o: [B * N, H, d]; lse: [B, H, N].
 *
 * Optional outputs (NULL to skip), [B * N, H, d] like o, the sums an error
 * bound on the rounding of p needs, per output element (row i, channel c):
 *   wa  = sum_j p_j |v^_jc| / l        wa2 = sum_j (p_j v^_jc)^2 / l^2
 *   wz  = sum_j |cv_jc| / l            wz2 = sum_j cv_jc^2 / l^2
 * (cv: the V codes, p_j = exp(x_j - m) as above, j over the allowed keys). */
int oracle_fwd_fp8(const float *qc, const float *kc, const float *vc, const float *sq,
                   const float *sk, const float *sv, int B, int N, int H, int d, double scale,
                   int causal, int window, int quantize_p, double *o, double *lse,
                   double *wa, double *wa2, double *wz, double *wz2)
{
    if (B < 0 || N < 0 || H <= 0 || d <= 0) return -3;
    if (window > 0 && !causal) return -5;
    const int nb = (N + BLK - 1) / BLK;
    int bad = 0;
    #pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (N > 0 ? N : 1));
        double *qh = (double *)malloc(sizeof(double) * d);
        if (!x || !qh) {
            #pragma omp atomic write
            bad = 1;
        }
        #pragma omp for collapse(3) schedule(dynamic, 16)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h)
                for (int i = 0; i < N; ++i) {
                    if (!x || !qh) continue;
                    const size_t sb = ((size_t)b * H + h) * nb;
                    const size_t oi = (((size_t)b * N + i) * H + h) * d;
                    const float *qr = qc + oi;
                    for (int c = 0; c < d; ++c) qh[c] = (double)qr[c] * sq[sb + i / BLK];
                    /* scores of the quantised operands and their maximum */
                    double m = -INFINITY;
                    for (int j = 0; j < N; ++j) {
                        x[j] = -INFINITY;
                        if (!allowed(i, j, causal, window)) continue;
                        const float *kr = kc + (((size_t)b * N + j) * H + h) * d;
                        const double skj = sk[sb + j / BLK];
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) acc += qh[c] * ((double)kr[c] * skj);
                        x[j] = scale * acc;
                        if (x[j] > m) m = x[j];
                    }
                    double *orow = o + oi;
                    for (int c = 0; c < d; ++c) orow[c] = 0.0;
                    if (wa) for (int c = 0; c < d; ++c) wa[oi + c] = 0.0;
                    if (wa2) for (int c = 0; c < d; ++c) wa2[oi + c] = 0.0;
                    if (wz) for (int c = 0; c < d; ++c) wz[oi + c] = 0.0;
                    if (wz2) for (int c = 0; c < d; ++c) wz2[oi + c] = 0.0;
                    if (m == -INFINITY) {               /* no allowed key */
                        lse[sb / nb * N + i] = -INFINITY;
                        continue;
                    }
                    /* exponentials and their sum */
                    double l = 0.0;
                    for (int j = 0; j < N; ++j)
                        if (x[j] != -INFINITY) l += exp(x[j] - m);
                    /* output: quantised p times the quantised V rows */
                    for (int j = 0; j < N; ++j) {
                        if (x[j] == -INFINITY) continue;
                        const double p = exp(x[j] - m);
                        const double pq = quantize_p ? e4m3_round_d(p) : p;
                        const float *vr = vc + (((size_t)b * N + j) * H + h) * d;
                        const double svj = sv[sb + j / BLK];
                        for (int c = 0; c < d; ++c) {
                            const double vh = (double)vr[c] * svj;
                            orow[c] += pq * vh;
                            if (wa) wa[oi + c] += p * fabs(vh);
                            if (wa2) wa2[oi + c] += (p * vh) * (p * vh);
                            if (wz) wz[oi + c] += fabs((double)vr[c]);
                            if (wz2) wz2[oi + c] += (double)vr[c] * (double)vr[c];
                        }
                    }
                    for (int c = 0; c < d; ++c) {
                        orow[c] /= l;
                        if (wa) wa[oi + c] /= l;
                        if (wa2) wa2[oi + c] /= l * l;
                        if (wz) wz[oi + c] /= l;
                        if (wz2) wz2[oi + c] /= l * l;
                    }
                    lse[sb / nb * N + i] = m + log(l);
                }
        free(x);
        free(qh);
    }
    return bad ? -3 : 0;
}
