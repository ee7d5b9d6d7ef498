/*
 * RRAttention prefill path -- CPU ORACLE (test infrastructure only).
 *
 * A plain, slow, obviously-correct restatement in double precision of what the
 * method computes.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg load this library; the product path never does.  It shares no code
 * with the CUDA kernels.
 *
 * Source: "RRAttention: Dynamic Block Sparse Attention via Per-Head Round-Robin
 * Shifts for Long-Context Inference" (paperpeel.com/paper/2602.05853):
 *   - Sec. 2.1: blocks of size B, stride S, Nb = L/B, causal block selection.
 *   - Sec. 1 contribution (i) and Sec. 3.1 heading: one sampled query per stride,
 *     the sampled position rotated across heads (round-robin).  The body of 3.1 is
 *     missing from the page; the offset rule is the reading documented below.
 *   - Sec. 3.2 "where" clause: score of sampled query Q_{P(i,h)} against the sum of
 *     all key vectors in stride j, scaled by 1/(S*sqrt(d)); stride-level softmax
 *     (Sec. 2.2, softmax granularity), cost O(L^2/S^2).
 *   - Sec. 1 contribution (iii), Sec. 3.3 heading: adaptive Top-tau block selection
 *     (the XAttention card, elamur.ai "Key points": the minimal set of blocks whose
 *     cumulative score reaches tau).
 *   - Sec. 4.3 "Last Query Block Protection": the last query block is kept whole.
 *
 * Readings where the pages are silent:
 *   o1 offset(h) = h mod S on the query-head index (head-RR); other strategies of
 *      Sec. 4.3 Table 6: none -> S-1, layer-RR -> layer mod S, hybrid -> (h+layer) mod S.
 *   o2 causality at stride granularity (key stride j <= query stride i).
 *   o3 pooled key = sum of the S keys, logit scale 1/(S*sqrt(d)).
 *   o4 block score A[I][J] = (S/B) * sum of stride probabilities over the
 *      (B/S)x(B/S) sub-grid (row I of A then sums to 1).
 *   o5 per (head, query block) row, ordered by (score desc, J asc), the smallest
 *      prefix whose cumulative sum is >= tau * T, T = the row total; tau >= 1 keeps all.
 *   o9 GQA: query head h reads KV head h / (H/Hkv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define RRO_OK 0
#define RRO_EINVAL 1
#define RRO_ECAP 4

enum { RRO_HEAD_RR = 0, RRO_NO_RR = 1, RRO_LAYER_RR = 2, RRO_HYBRID_RR = 3 };

/* bf16 bit pattern -> double, exact. */
static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int rro_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Offset of the sampled query inside each stride for head h (reading o1). */
int rro_offset(int h, int S, int mode, int layer) {
    switch (mode) {
    case RRO_HEAD_RR: return h % S;
    case RRO_NO_RR: return S - 1;
    case RRO_LAYER_RR: return layer % S;
    case RRO_HYBRID_RR: return (h + layer) % S;
    default: return -1;
    }
}

/* P(i,h): position of the query sampled from stride i for head h. */
long rro_sample_position(long i, int h, int S, int mode, int layer) {
    return i * (long)S + rro_offset(h, S, mode, layer);
}

/* Kbar[g][j][:] = sum over the S keys of stride j of K[g][t][:]  (Sec. 3.2). */
void rro_pool_keys(const uint16_t *K, int Hkv, int L, int d, int S, double *Kbar) {
    const long Ns = L / S;
    for (int g = 0; g < Hkv; ++g)
        for (long j = 0; j < Ns; ++j) {
            double *out = Kbar + ((long)g * Ns + j) * d;
            for (int e = 0; e < d; ++e) out[e] = 0.0;
            for (int u = 0; u < S; ++u) {
                const uint16_t *k = K + ((long)g * L + j * S + u) * d;
                for (int e = 0; e < d; ++e) out[e] += bf16_to_double(k[e]);
            }
        }
}

/* Stride-level probabilities of one sampled query row:
 * z_j = q . Kbar_j / (S sqrt d) for j = 0..i, p = softmax(z).  Writes p[0..i]. */
static void stride_softmax_row(const double *q, const double *Kbar_g, long i, int d, int S,
                               double *p) {
    const double scale = 1.0 / ((double)S * sqrt((double)d));
    double m = -INFINITY;
    for (long j = 0; j <= i; ++j) {
        const double *kb = Kbar_g + j * d;
        double z = 0.0;
        for (int e = 0; e < d; ++e) z += q[e] * kb[e];
        p[j] = z * scale;
        if (p[j] > m) m = p[j];
    }
    double l = 0.0;
    for (long j = 0; j <= i; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    for (long j = 0; j <= i; ++j) p[j] /= l;
}

/* Block importance A[h][I][J] for heads h in [h_begin, h_end)  (Sec. 3.2-3.3, reading o4).
 * A is [H][Nb][Nb]; entries with J > I are set to 0.  Returns RRO_OK or RRO_EINVAL. */
int rro_estimate(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d, int S,
                 int B, int mode, int layer, int h_begin, int h_end, double *A) {
    if (H <= 0 || Hkv <= 0 || H % Hkv || d <= 0 || S <= 0 || B <= 0 || B % S || L % B)
        return RRO_EINVAL;
    if (h_begin < 0 || h_end > H || h_begin > h_end) return RRO_EINVAL;
    const long Ns = L / S, Nb = L / B, r = B / S;
    const int G = H / Hkv;
    double *Kbar = (double *)malloc(sizeof(double) * (size_t)Hkv * Ns * d + 1);
    if (!Kbar) return RRO_EINVAL;
    rro_pool_keys(K, Hkv, L, d, S, Kbar);
    const double w = (double)S / (double)B;
    const long nrows = (long)(h_end - h_begin) * Nb;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)Ns + 1);
        double *q = (double *)malloc(sizeof(double) * (size_t)d + 1);
#pragma omp for schedule(dynamic, 1)
        for (long row = 0; row < nrows; ++row) {
            const int h = h_begin + (int)(row / Nb);
            const long I = Nb - 1 - row % Nb; /* long rows first */
            const int g = h / G;
            double *Arow = A + ((long)h * Nb + I) * Nb;
            for (long J = 0; J < Nb; ++J) Arow[J] = 0.0;
            for (long i = I * r; i < (I + 1) * r; ++i) {
                const long pos = rro_sample_position(i, h, S, mode, layer);
                const uint16_t *qs = Q + ((long)h * L + pos) * d;
                for (int e = 0; e < d; ++e) q[e] = bf16_to_double(qs[e]);
                stride_softmax_row(q, Kbar + (long)g * Ns * d, i, d, S, p);
                for (long j = 0; j <= i; ++j) Arow[j / r] += w * p[j];
            }
        }
        free(p);
        free(q);
    }
    free(Kbar);
    return RRO_OK;
}

/* ---------------------------------------------------------------- XAttention estimate
 * The comparison estimator of the pattern-discovery timing (RRAttention Sec. 4.2 "Runtime
 * Efficiency", Fig. 3(b); RRAttention Sec. 2.2 and the XAttention card, "Summary" and "Key
 * points"): inside every S x S sub-block of the attention logits (query stride i, key stride
 * j) the entries on the antidiagonal, from lower-left (query iS+S-1, key jS) to upper-right
 * (query iS, key jS+S-1), are summed; the sums are softmax-normalised over the key strides and
 * aggregated into blocks, then the same Top-tau selection keeps the blocks.
 * Readings where the pages are silent (the same as for the round-robin estimate):
 *   x1 score a(i,j) = (1/(S sqrt d)) sum_{u<S} Q[iS+S-1-u] . K[jS+u], the mean of the S
 *      antidiagonal logits q.k/sqrt(d) (the card's "sums", scaled like Sec. 3.2's 1/(S sqrt d));
 *   x2 causality at stride granularity (j <= i), softmax over j in [0, i] (stride-level
 *      softmax granularity, RRAttention Sec. 2.2);
 *   x3 block score (S/B) * sum over the (B/S) x (B/S) sub-grid, as reading o4.
 * A is [H][Nb][Nb]; rows of heads outside [h_begin, h_end) are not touched; J > I entries 0. */
int rro_xattn_estimate(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d, int S,
                       int B, int h_begin, int h_end, double *A) {
    if (H <= 0 || Hkv <= 0 || H % Hkv || d <= 0 || S <= 0 || B <= 0 || B % S || L % B)
        return RRO_EINVAL;
    if (h_begin < 0 || h_end > H || h_begin > h_end) return RRO_EINVAL;
    const long Ns = L / S, Nb = L / B, r = B / S;
    const int G = H / Hkv;
    const double scale = 1.0 / ((double)S * sqrt((double)d));
    const double w = (double)S / (double)B;
    const long nrows = (long)(h_end - h_begin) * Nb;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)Ns + 1);
#pragma omp for schedule(dynamic, 1)
        for (long row = 0; row < nrows; ++row) {
            const int h = h_begin + (int)(row / Nb);
            const long I = Nb - 1 - row % Nb; /* long rows first */
            const int g = h / G;
            double *Arow = A + ((long)h * Nb + I) * Nb;
            for (long J = 0; J < Nb; ++J) Arow[J] = 0.0;
            for (long i = I * r; i < (I + 1) * r; ++i) {
                double m = -INFINITY;
                for (long j = 0; j <= i; ++j) {
                    double a = 0.0;
                    for (int u = 0; u < S; ++u) {
                        const uint16_t *q = Q + ((long)h * L + i * S + (S - 1 - u)) * d;
                        const uint16_t *k = K + ((long)g * L + j * S + u) * d;
                        for (int e = 0; e < d; ++e) a += bf16_to_double(q[e]) * bf16_to_double(k[e]);
                    }
                    p[j] = a * scale;
                    if (p[j] > m) m = p[j];
                }
                double l = 0.0;
                for (long j = 0; j <= i; ++j) {
                    p[j] = exp(p[j] - m);
                    l += p[j];
                }
                for (long j = 0; j <= i; ++j) Arow[j / r] += w * p[j] / l;
            }
        }
        free(p);
    }
    return RRO_OK;
}

typedef struct {
    double a;
    int J;
} scored_block;

/* Order: score descending, then block index ascending (reading o6). */
static int by_score_desc(const void *x, const void *y) {
    const scored_block *u = (const scored_block *)x, *v = (const scored_block *)y;
    if (u->a > v->a) return -1;
    if (u->a < v->a) return 1;
    return (u->J > v->J) - (u->J < v->J);
}

/* Top-tau selection for one row of n = I+1 causal blocks.  Writes the chosen block
 * indices (ascending) to out, returns their count.  diag (5 doubles, may be NULL):
 * k*, cum_{k*-1}, cum_{k*}, tau*T, a_(k*) - a_(k*+1) (+inf when k* = n). */
static int select_row(const double *Arow, int n, double tau, int keep_all, int *out,
                      scored_block *buf, char *mark, double *diag) {
    for (int J = 0; J < n; ++J) {
        buf[J].a = Arow[J];
        buf[J].J = J;
    }
    qsort(buf, (size_t)n, sizeof *buf, by_score_desc);
    double T = 0.0;
    for (int k = 0; k < n; ++k) T += buf[k].a;
    const double thr = tau * T;
    int kstar = n;
    double cum = 0.0, cum_before = 0.0;
    if (!keep_all) {
        for (int k = 0; k < n; ++k) {
            cum_before = cum;
            cum += buf[k].a;
            if (cum >= thr) {
                kstar = k + 1;
                break;
            }
        }
    } else {
        for (int k = 0; k < n; ++k) {
            cum_before = cum;
            cum += buf[k].a;
        }
    }
    if (diag) {
        diag[0] = kstar;
        diag[1] = cum_before;
        diag[2] = cum;
        diag[3] = thr;
        diag[4] = (kstar < n) ? buf[kstar - 1].a - buf[kstar].a : INFINITY;
    }
    memset(mark, 0, (size_t)n);
    for (int k = 0; k < kstar; ++k) mark[buf[k].J] = 1;
    int c = 0;
    for (int J = 0; J < n; ++J)
        if (mark[J]) out[c++] = J;
    return c;
}

/* Per-head CSR block lists from A[H][Nb][Nb]  (Sec. 3.3 heading, XAttention card, Sec. 4.3
 * last-block protection).  Row r = h*Nb + I lists its blocks J <= I in ascending order.
 * col_capacity bounds col_idx; returns RRO_ECAP when it would be exceeded.
 * diag: NULL or [H*Nb][5] (see select_row). */
int rro_select(const double *A, int H, int Nb, double tau, int protect_last, int32_t *row_ptr,
               int32_t *col_idx, int64_t col_capacity, double *diag) {
    if (H < 0 || Nb < 0 || !(tau > 0.0)) return RRO_EINVAL;
    const long nrows = (long)H * Nb;
    int *counts = (int *)malloc(sizeof(int) * (size_t)nrows + 1);
    int *lists = (int *)malloc(sizeof(int) * ((size_t)nrows * (Nb > 0 ? Nb : 1)) + 1);
    if (!counts || !lists) return RRO_EINVAL;
#pragma omp parallel
    {
        scored_block *buf = (scored_block *)malloc(sizeof(scored_block) * (size_t)Nb + 1);
        char *mark = (char *)malloc((size_t)Nb + 1);
#pragma omp for schedule(dynamic, 16)
        for (long row = 0; row < nrows; ++row) {
            const int I = (int)(row % Nb);
            const int keep_all = (tau >= 1.0) || (protect_last && I == Nb - 1);
            counts[row] = select_row(A + row * Nb, I + 1, tau, keep_all, lists + row * Nb, buf,
                                     mark, diag ? diag + row * 5 : NULL);
        }
        free(buf);
        free(mark);
    }
    int64_t nnz = 0;
    for (long row = 0; row < nrows; ++row) nnz += counts[row];
    if (nnz > col_capacity || nnz > INT32_MAX) {
        free(counts);
        free(lists);
        return RRO_ECAP;
    }
    int64_t at = 0;
    for (long row = 0; row < nrows; ++row) {
        row_ptr[row] = (int32_t)at;
        for (int c = 0; c < counts[row]; ++c) col_idx[at++] = lists[row * Nb + c];
    }
    row_ptr[nrows] = (int32_t)at;
    free(counts);
    free(lists);
    return RRO_OK;
}

/* Causal block-sparse attention for the requested query rows (Sec. 2.1 with the
 * selected blocks as the block selection matrix).  rows = nrows pairs (h, q).
 * Key k of KV head h/(H/Hkv) is attended iff k <= q and k/B is listed in row
 * h*Nb + q/B of the CSR.  O is [nrows][d].  scale <= 0 means 1/sqrt(d). */
int rro_prefill_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv,
                     int L, int d, int B, const int32_t *row_ptr, const int32_t *col_idx,
                     double scale, const int64_t *rows, int64_t nrows, double *O) {
    if (H <= 0 || Hkv <= 0 || H % Hkv || d <= 0 || B <= 0 || L % B) return RRO_EINVAL;
    if (!(scale > 0.0)) scale = 1.0 / sqrt((double)d);
    const int Nb = L / B, G = H / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)L + 1);
        double *q = (double *)malloc(sizeof(double) * (size_t)d + 1);
#pragma omp for schedule(dynamic, 4) reduction(| : bad)
        for (int64_t n = 0; n < nrows; ++n) {
            const int h = (int)rows[2 * n];
            const long t = (long)rows[2 * n + 1];
            double *o = O + n * d;
            if (h < 0 || h >= H || t < 0 || t >= L) {
                bad = 1;
                continue;
            }
            const int g = h / G;
            const long r = (long)h * Nb + t / B;
            for (int e = 0; e < d; ++e) q[e] = bf16_to_double(Q[((long)h * L + t) * d + e]);
            double m = -INFINITY;
            long cnt = 0;
            for (int32_t c = row_ptr[r]; c < row_ptr[r + 1]; ++c) {
                const long J = col_idx[c];
                for (long k = J * B; k < (J + 1) * B && k <= t; ++k) {
                    const uint16_t *kr = K + ((long)g * L + k) * d;
                    double z = 0.0;
                    for (int e = 0; e < d; ++e) z += q[e] * bf16_to_double(kr[e]);
                    z *= scale;
                    s[cnt++] = z;
                    if (z > m) m = z;
                }
            }
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            double l = 0.0;
            cnt = 0;
            for (int32_t c = row_ptr[r]; c < row_ptr[r + 1]; ++c) {
                const long J = col_idx[c];
                for (long k = J * B; k < (J + 1) * B && k <= t; ++k) {
                    const double p = exp(s[cnt++] - m);
                    l += p;
                    const uint16_t *vr = V + ((long)g * L + k) * d;
                    for (int e = 0; e < d; ++e) o[e] += p * bf16_to_double(vr[e]);
                }
            }
            for (int e = 0; e < d; ++e) o[e] = (l > 0.0) ? o[e] / l : NAN;
        }
        free(s);
        free(q);
    }
    return bad ? RRO_EINVAL : RRO_OK;
}
