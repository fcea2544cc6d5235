/*
 * attn_oracle.c -- float64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * tests, the smoke check and the benchmark's CPU-baseline leg compare the CUDA
 * library against.  The product path never loads it, and it shares no code,
 * header, table or helper with the CUDA sources.
 *
 * What it computes (FlashAttention encyclopedia page, section "attention and
 * the memory bottleneck", the SDPA definition): for one head,
 *     O = softmax(scale * Q K^T) V,  softmax taken row by row over the keys a
 * mask allows.  The method reaches exactly this result (same page, paragraph
 * on the meaning of "exact"), so the oracle is that definition written out,
 * using the three-pass safe softmax of the blog article "From Online Softmax
 * to FlashAttention", section 2.1-2.2 (pass 1: row max, pass 2: sum of
 * exponentials, pass 3: normalise and accumulate).
 *
 * The backward formulas are not printed on the pages (the encyclopedia page,
 * section "training and complexity", only says the blocks are recomputed from
 * compact normalisation statistics).  They follow from the definition by the
 * softmax Jacobian and are written out in oracle_bwd below.
 *
 * Data layout (shared with the callers, not with the CUDA code):
 *   q, k, v, dout, o, dq, dk, dv : float64 [T, H, d] row-major, T = total
 *       tokens; sequence s occupies token rows starts[s] .. starts[s]+lens[s]-1.
 *   lse, D : float64 [H, T].
 * Masks (row i and key j are indices local to their sequence, 0 <= i,j < n):
 *   causal:  key j allowed iff j <= i
 *   window W > 0 (needs causal): allowed iff i - W < j <= i  (exactly W keys
 *       including the query's own position)
 * A row with no allowed key gets O = 0 and LSE = -inf (cannot happen with
 * the masks above, because j = i is always allowed).
 *
 * All arithmetic is float64 with libm exp/log.  Return value 0 = ok,
 * -5 = window without causal, -3 = bad shape.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static int key_allowed(int i, int j, int causal, int window)
{
    if (causal && j > i) return 0;
    if (window > 0 && j <= i - window) return 0;
    return 1;
}

static int check_args(int T, int H, int d, int nseq, const int *starts, const int *lens,
                      int causal, int window)
{
    if (window > 0 && !causal) return -5;
    if (T < 0 || H <= 0 || d <= 0 || nseq < 0) return -3;
    for (int s = 0; s < nseq; ++s)
        if (lens[s] < 0 || starts[s] < 0 || starts[s] + lens[s] > T) return -3;
    return 0;
}

static double dot(const double *a, const double *b, int d)
{
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += a[c] * b[c];
    return acc;
}

/* One query row, three passes.  The query row is qstart + i of q; its keys
 * and values are rows kstart .. kstart + nk - 1 of k and v, and the mask sees
 * the query at position i + off of the key sequence (off = 0 for
 * self-attention).  Writes o_row[d] and returns the LSE. */
static double three_pass_row_kv(const double *q, const double *k, const double *v,
                                int H, int d, int qstart, int kstart, int nk, int off,
                                int h, int i, double scale, int causal, int window,
                                double *o_row)
{
    const size_t rs = (size_t)H * d;               /* token row stride */
    const double *qi = q + (size_t)(qstart + i) * rs + (size_t)h * d;
    const int pos = i + off;

    /* pass 1: row maximum of the scaled scores over allowed keys */
    double m = -INFINITY;
    for (int j = 0; j < nk; ++j) {
        if (!key_allowed(pos, j, causal, window)) continue;
        double s = scale * dot(qi, k + (size_t)(kstart + j) * rs + (size_t)h * d, d);
        if (s > m) m = s;
    }
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    if (m == -INFINITY) return -INFINITY;

    /* pass 2: normaliser l = sum_j exp(s_j - m) */
    double l = 0.0;
    for (int j = 0; j < nk; ++j) {
        if (!key_allowed(pos, j, causal, window)) continue;
        double s = scale * dot(qi, k + (size_t)(kstart + j) * rs + (size_t)h * d, d);
        l += exp(s - m);
    }

    /* pass 3: o = sum_j (exp(s_j - m) / l) v_j */
    for (int j = 0; j < nk; ++j) {
        if (!key_allowed(pos, j, causal, window)) continue;
        const double *vj = v + (size_t)(kstart + j) * rs + (size_t)h * d;
        double s = scale * dot(qi, k + (size_t)(kstart + j) * rs + (size_t)h * d, d);
        double p = exp(s - m) / l;
        for (int c = 0; c < d; ++c) o_row[c] += p * vj[c];
    }
    return m + log(l);
}

/* Self-attention row: queries and keys are the same sequence. */
static double three_pass_row(const double *q, const double *k, const double *v,
                             int H, int d, int start, int n, int h, int i,
                             double scale, int causal, int window, double *o_row)
{
    return three_pass_row_kv(q, k, v, H, d, start, start, n, 0, h, i, scale, causal, window,
                             o_row);
}

/* Full forward over every (sequence, head, row). */
int oracle_fwd(const double *q, const double *k, const double *v,
               int T, int H, int d, int nseq, const int *starts, const int *lens,
               double scale, int causal, int window, double *o, double *lse)
{
    int rc = check_args(T, H, d, nseq, starts, lens, causal, window);
    if (rc) return rc;
    const size_t rs = (size_t)H * d;
    for (int s = 0; s < nseq; ++s) {
        const int start = starts[s], n = lens[s];
        #pragma omp parallel for collapse(2) schedule(dynamic, 8)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < n; ++i) {
                double *orow = o + (size_t)(start + i) * rs + (size_t)h * d;
                lse[(size_t)h * T + start + i] =
                    three_pass_row(q, k, v, H, d, start, n, h, i, scale, causal, window, orow);
            }
    }
    return 0;
}

/* Forward for a list of rows only: rows[3*r .. 3*r+2] = (sequence, head, row).
 * o_rows is [nrows, d], lse_rows is [nrows].  Rows are independent, so this is
 * exactly the full forward restricted to those rows. */
int oracle_fwd_rows(const double *q, const double *k, const double *v,
                    int T, int H, int d, int nseq, const int *starts, const int *lens,
                    double scale, int causal, int window,
                    int nrows, const int *rows, double *o_rows, double *lse_rows)
{
    int rc = check_args(T, H, d, nseq, starts, lens, causal, window);
    if (rc) return rc;
    for (int r = 0; r < nrows; ++r) {
        int s = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (s < 0 || s >= nseq || h < 0 || h >= H || i < 0 || i >= lens[s]) return -3;
    }
    #pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < nrows; ++r) {
        int s = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        lse_rows[r] = three_pass_row(q, k, v, H, d, starts[s], lens[s], h, i,
                                     scale, causal, window, o_rows + (size_t)r * d);
    }
    return 0;
}

/*
 * Forward with a key/value sequence that may be longer than the query
 * sequence (prefill against cached keys and values): sequence s has nq =
 * qlens[s] query rows starting at qstarts[s] of q and nk = klens[s] key/value
 * rows starting at kstarts[s] of k and v.  The queries are the LAST nq
 * positions of the key sequence, so query row i sits at position
 * i + (nk - nq): under the causal mask it sees keys j <= i + nk - nq
 * (bottom-right alignment), under a window W also only j > i + nk - nq - W.
 * With nq = nk this is oracle_fwd.  A query that sees no key gets O = 0 and
 * LSE = -inf.  o is [Tq, H, d]; lse is [H, Tq].
 */
int oracle_fwd_kv(const double *q, const double *k, const double *v,
                  int Tq, int Tk, int H, int d, int nseq,
                  const int *qstarts, const int *qlens, const int *kstarts, const int *klens,
                  double scale, int causal, int window, double *o, double *lse)
{
    if (window > 0 && !causal) return -5;
    if (Tq < 0 || Tk < 0 || H <= 0 || d <= 0 || nseq < 0) return -3;
    for (int s = 0; s < nseq; ++s)
        if (qlens[s] < 0 || klens[s] < 0 || qstarts[s] < 0 || kstarts[s] < 0 ||
            qstarts[s] + qlens[s] > Tq || kstarts[s] + klens[s] > Tk) return -3;
    const size_t rs = (size_t)H * d;
    for (int s = 0; s < nseq; ++s) {
        const int nq = qlens[s], nk = klens[s];
        #pragma omp parallel for collapse(2) schedule(dynamic, 8)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < nq; ++i) {
                double *orow = o + (size_t)(qstarts[s] + i) * rs + (size_t)h * d;
                lse[(size_t)h * Tq + qstarts[s] + i] =
                    three_pass_row_kv(q, k, v, H, d, qstarts[s], kstarts[s], nk, nk - nq, h, i,
                                      scale, causal, window, orow);
            }
    }
    return 0;
}

/* Online (one-pass, blocked) forward, used only to check that the blocked
 * update reaches the three-pass result.  It follows the update of the
 * encyclopedia page, section "tiled computation and online normalisation":
 * for each new block of scores s_b,
 *     m' = max(m, max s_b)
 *     l' = e^{m-m'} l + sum_j e^{s_bj - m'}
 *     u' = e^{m-m'} u + sum_j e^{s_bj - m'} v_bj
 * and the output is u / l after the last block.  The blog article's section 4
 * takes the block maximum first and then merges it with the running maximum,
 * which is what the first line does.  `block` is the number of keys per block
 * (the blog's b); masked keys inside a block are simply left out. */
int oracle_fwd_online(const double *q, const double *k, const double *v,
                      int T, int H, int d, int nseq, const int *starts, const int *lens,
                      double scale, int causal, int window, int block,
                      double *o, double *lse)
{
    int rc = check_args(T, H, d, nseq, starts, lens, causal, window);
    if (rc) return rc;
    if (block <= 0) return -3;
    const size_t rs = (size_t)H * d;
    for (int s = 0; s < nseq; ++s) {
        const int start = starts[s], n = lens[s];
        #pragma omp parallel for collapse(2) schedule(dynamic, 8)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < n; ++i) {
                const double *qi = q + (size_t)(start + i) * rs + (size_t)h * d;
                double *u = o + (size_t)(start + i) * rs + (size_t)h * d;
                double m = -INFINITY, l = 0.0;
                for (int c = 0; c < d; ++c) u[c] = 0.0;
                for (int j0 = 0; j0 < n; j0 += block) {
                    int j1 = j0 + block < n ? j0 + block : n;
                    /* block maximum, then merge with the running maximum */
                    double mb = -INFINITY;
                    for (int j = j0; j < j1; ++j) {
                        if (!key_allowed(i, j, causal, window)) continue;
                        double sc = scale * dot(qi, k + (size_t)(start + j) * rs + (size_t)h * d, d);
                        if (sc > mb) mb = sc;
                    }
                    if (mb == -INFINITY) continue;            /* block fully masked */
                    double mnew = m > mb ? m : mb;
                    double alpha = exp(m - mnew);              /* e^{m-m'}; 0 when m = -inf */
                    l *= alpha;
                    for (int c = 0; c < d; ++c) u[c] *= alpha;
                    for (int j = j0; j < j1; ++j) {
                        if (!key_allowed(i, j, causal, window)) continue;
                        const double *vj = v + (size_t)(start + j) * rs + (size_t)h * d;
                        double sc = scale * dot(qi, k + (size_t)(start + j) * rs + (size_t)h * d, d);
                        double p = exp(sc - mnew);
                        l += p;
                        for (int c = 0; c < d; ++c) u[c] += p * vj[c];
                    }
                    m = mnew;
                }
                if (m == -INFINITY) {
                    lse[(size_t)h * T + start + i] = -INFINITY;
                } else {
                    for (int c = 0; c < d; ++c) u[c] /= l;
                    lse[(size_t)h * T + start + i] = m + log(l);
                }
            }
    }
    return 0;
}

/*
 * Backward for selected (sequence, head) pairs: pairs[2*p], pairs[2*p+1];
 * pairs == NULL means all of them.  Given dO, it returns dQ, dK, dV for those
 * heads (other entries of dq/dk/dv are left untouched).  The oracle recomputes
 * its own O and LSE with the three-pass forward; it never sees the GPU's.
 *
 * With P_ij = exp(s_ij - LSE_i) on allowed pairs (0 elsewhere):
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . v_j
 *   D_i   = sum_j P_ij dP_ij = dO_i . O_i
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 * o_out, lse_out, D_out may be NULL; otherwise they receive the oracle's own
 * O [T,H,d], LSE [H,T] and D [H,T] for the selected heads.
 */
int oracle_bwd(const double *q, const double *k, const double *v, const double *dout,
               int T, int H, int d, int nseq, const int *starts, const int *lens,
               double scale, int causal, int window, int npairs, const int *pairs,
               double *dq, double *dk, double *dv,
               double *o_out, double *lse_out, double *D_out)
{
    int rc = check_args(T, H, d, nseq, starts, lens, causal, window);
    if (rc) return rc;
    const size_t rs = (size_t)H * d;
    int total_pairs = pairs ? npairs : nseq * H;
    for (int p = 0; p < total_pairs; ++p) {
        int s = pairs ? pairs[2 * p] : p / H;
        int h = pairs ? pairs[2 * p + 1] : p % H;
        if (s < 0 || s >= nseq || h < 0 || h >= H) return -3;
    }
    for (int p = 0; p < total_pairs; ++p) {
        const int s = pairs ? pairs[2 * p] : p / H;
        const int h = pairs ? pairs[2 * p + 1] : p % H;
        const int start = starts[s], n = lens[s];
        if (n == 0) continue;
        double *o_h = (double *)malloc(sizeof(double) * (size_t)n * d);
        double *lse_h = (double *)malloc(sizeof(double) * (size_t)n);
        double *D_h = (double *)malloc(sizeof(double) * (size_t)n);
        if (!o_h || !lse_h || !D_h) { free(o_h); free(lse_h); free(D_h); return -3; }

        /* forward (three passes) and D_i = dO_i . O_i */
        #pragma omp parallel for schedule(dynamic, 8)
        for (int i = 0; i < n; ++i) {
            lse_h[i] = three_pass_row(q, k, v, H, d, start, n, h, i, scale, causal, window,
                                      o_h + (size_t)i * d);
            D_h[i] = dot(dout + (size_t)(start + i) * rs + (size_t)h * d, o_h + (size_t)i * d, d);
        }

        /* dQ_i = scale * sum_j P_ij (dP_ij - D_i) k_j */
        #pragma omp parallel for schedule(dynamic, 8)
        for (int i = 0; i < n; ++i) {
            const double *qi = q + (size_t)(start + i) * rs + (size_t)h * d;
            const double *doi = dout + (size_t)(start + i) * rs + (size_t)h * d;
            double *dqi = dq + (size_t)(start + i) * rs + (size_t)h * d;
            for (int c = 0; c < d; ++c) dqi[c] = 0.0;
            if (lse_h[i] == -INFINITY) continue;
            for (int j = 0; j < n; ++j) {
                if (!key_allowed(i, j, causal, window)) continue;
                const double *kj = k + (size_t)(start + j) * rs + (size_t)h * d;
                const double *vj = v + (size_t)(start + j) * rs + (size_t)h * d;
                double P = exp(scale * dot(qi, kj, d) - lse_h[i]);
                double dS = P * (dot(doi, vj, d) - D_h[i]);
                for (int c = 0; c < d; ++c) dqi[c] += scale * dS * kj[c];
            }
        }

        /* dV_j = sum_i P_ij dO_i ;  dK_j = scale * sum_i P_ij (dP_ij - D_i) q_i */
        #pragma omp parallel for schedule(dynamic, 8)
        for (int j = 0; j < n; ++j) {
            const double *kj = k + (size_t)(start + j) * rs + (size_t)h * d;
            const double *vj = v + (size_t)(start + j) * rs + (size_t)h * d;
            double *dkj = dk + (size_t)(start + j) * rs + (size_t)h * d;
            double *dvj = dv + (size_t)(start + j) * rs + (size_t)h * d;
            for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            for (int i = 0; i < n; ++i) {
                if (!key_allowed(i, j, causal, window) || lse_h[i] == -INFINITY) continue;
                const double *qi = q + (size_t)(start + i) * rs + (size_t)h * d;
                const double *doi = dout + (size_t)(start + i) * rs + (size_t)h * d;
                double P = exp(scale * dot(qi, kj, d) - lse_h[i]);
                double dS = P * (dot(doi, vj, d) - D_h[i]);
                for (int c = 0; c < d; ++c) {
                    dvj[c] += P * doi[c];
                    dkj[c] += scale * dS * qi[c];
                }
            }
        }

        for (int i = 0; i < n; ++i) {
            if (o_out)
                memcpy(o_out + (size_t)(start + i) * rs + (size_t)h * d, o_h + (size_t)i * d,
                       sizeof(double) * d);
            if (lse_out) lse_out[(size_t)h * T + start + i] = lse_h[i];
            if (D_out) D_out[(size_t)h * T + start + i] = D_h[i];
        }
        free(o_h); free(lse_h); free(D_h);
    }
    return 0;
}

/*
 * The same gradients as oracle_bwd, for listed rows only (self-attention):
 * qrows[3*r .. 3*r+2] = (sequence, head, query row) gets dq_rows[r*d ..] =
 * dQ_i, and krows[3*r .. 3*r+2] = (sequence, head, key row) gets
 * dk_rows[r*d ..] = dK_j and dv_rows[r*d ..] = dV_j, with the formulas of
 * oracle_bwd.  dQ_i needs only row i's own LSE_i and D_i.  dK_j and dV_j
 * need LSE_i and D_i of every query row i that may attend key j; for each
 * (sequence, head) of the key list they are computed (three-pass forward)
 * for the query rows from the smallest listed key (causal: no earlier row
 * sees it) to the largest listed key + W - 1 (window W; else the sequence
 * end), which is every row that can contribute.  So a long causal sequence
 * with keys listed near its end costs little.
 */
int oracle_bwd_rows(const double *q, const double *k, const double *v, const double *dout,
                    int T, int H, int d, int nseq, const int *starts, const int *lens,
                    double scale, int causal, int window,
                    int nq, const int *qrows, double *dq_rows,
                    int nk, const int *krows, double *dk_rows, double *dv_rows)
{
    int rc = check_args(T, H, d, nseq, starts, lens, causal, window);
    if (rc) return rc;
    const size_t rs = (size_t)H * d;
    for (int r = 0; r < nq; ++r) {
        int s = qrows[3 * r], h = qrows[3 * r + 1], i = qrows[3 * r + 2];
        if (s < 0 || s >= nseq || h < 0 || h >= H || i < 0 || i >= lens[s]) return -3;
    }
    for (int r = 0; r < nk; ++r) {
        int s = krows[3 * r], h = krows[3 * r + 1], j = krows[3 * r + 2];
        if (s < 0 || s >= nseq || h < 0 || h >= H || j < 0 || j >= lens[s]) return -3;
    }

    /* dQ_i = scale * sum_j P_ij (dP_ij - D_i) k_j, from row i's own statistics */
    int fail = 0;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nq; ++r) {
        const int s = qrows[3 * r], h = qrows[3 * r + 1], i = qrows[3 * r + 2];
        const int start = starts[s], n = lens[s];
        double *o_i = (double *)malloc(sizeof(double) * (size_t)d);
        if (!o_i) { fail = 1; continue; }
        const double lse_i = three_pass_row(q, k, v, H, d, start, n, h, i, scale, causal, window, o_i);
        const double *qi = q + (size_t)(start + i) * rs + (size_t)h * d;
        const double *doi = dout + (size_t)(start + i) * rs + (size_t)h * d;
        const double D_i = dot(doi, o_i, d);
        double *dqi = dq_rows + (size_t)r * d;
        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
        if (lse_i != -INFINITY)
            for (int j = 0; j < n; ++j) {
                if (!key_allowed(i, j, causal, window)) continue;
                const double *kj = k + (size_t)(start + j) * rs + (size_t)h * d;
                const double *vj = v + (size_t)(start + j) * rs + (size_t)h * d;
                const double P = exp(scale * dot(qi, kj, d) - lse_i);
                const double dS = P * (dot(doi, vj, d) - D_i);
                for (int c = 0; c < d; ++c) dqi[c] += scale * dS * kj[c];
            }
        free(o_i);
    }
    if (fail) return -3;

    /* dV_j = sum_i P_ij dO_i ;  dK_j = scale * sum_i P_ij (dP_ij - D_i) q_i,
       one (sequence, head) of the key list at a time */
    char *done = (char *)calloc(nk > 0 ? (size_t)nk : 1, 1);
    if (!done) return -3;
    for (int r0 = 0; r0 < nk; ++r0) {
        if (done[r0]) continue;
        const int s = krows[3 * r0], h = krows[3 * r0 + 1];
        const int start = starts[s], n = lens[s];
        int jmin = n, jmax = -1;
        for (int r = r0; r < nk; ++r)
            if (krows[3 * r] == s && krows[3 * r + 1] == h) {
                if (krows[3 * r + 2] < jmin) jmin = krows[3 * r + 2];
                if (krows[3 * r + 2] > jmax) jmax = krows[3 * r + 2];
            }
        const int i_lo = causal ? jmin : 0;
        const int i_hi = window > 0 ? (jmax + window < n ? jmax + window : n) : n;
        const int m = i_hi - i_lo;
        double *lse_h = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
        double *D_h = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
        if (!lse_h || !D_h) { free(lse_h); free(D_h); free(done); return -3; }
        #pragma omp parallel for schedule(dynamic, 8)
        for (int x = 0; x < m; ++x) {
            double *o_i = (double *)malloc(sizeof(double) * (size_t)d);
            if (!o_i) { lse_h[x] = NAN; D_h[x] = NAN; continue; }
            const int i = i_lo + x;
            lse_h[x] = three_pass_row(q, k, v, H, d, start, n, h, i, scale, causal, window, o_i);
            D_h[x] = dot(dout + (size_t)(start + i) * rs + (size_t)h * d, o_i, d);
            free(o_i);
        }
        #pragma omp parallel for schedule(dynamic, 1)
        for (int r = r0; r < nk; ++r) {
            if (krows[3 * r] != s || krows[3 * r + 1] != h) continue;
            const int j = krows[3 * r + 2];
            const double *kj = k + (size_t)(start + j) * rs + (size_t)h * d;
            const double *vj = v + (size_t)(start + j) * rs + (size_t)h * d;
            double *dkj = dk_rows + (size_t)r * d;
            double *dvj = dv_rows + (size_t)r * d;
            for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            for (int i = i_lo; i < i_hi; ++i) {
                const double lse_i = lse_h[i - i_lo];
                if (!key_allowed(i, j, causal, window) || lse_i == -INFINITY) continue;
                const double *qi = q + (size_t)(start + i) * rs + (size_t)h * d;
                const double *doi = dout + (size_t)(start + i) * rs + (size_t)h * d;
                const double P = exp(scale * dot(qi, kj, d) - lse_i);
                const double dS = P * (dot(doi, vj, d) - D_h[i - i_lo]);
                for (int c = 0; c < d; ++c) {
                    dvj[c] += P * doi[c];
                    dkj[c] += scale * dS * qi[c];
                }
            }
        }
        for (int r = r0; r < nk; ++r)
            if (krows[3 * r] == s && krows[3 * r + 1] == h) done[r] = 1;
        free(lse_h); free(D_h);
    }
    free(done);
    return 0;
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
