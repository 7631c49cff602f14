/*
 * rfb_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of attention with an additive
 * rank-factorised bias.  Only tests/, the smoke check and the CPU-baseline
 * leg of the bench may build, load or call this file.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * What it computes, per (batch b, head h), with s the softmax scale:
 *
 *   Bm   = U W^T                      (N x N bias, every element formed explicitly)
 *   S    = s Q K^T + Bm               (the bias is added to the query-key scores)
 *   P    = softmax over each row of S
 *   O    = P V,   LSE_i = log sum_j exp(S_ij)   (natural log)
 *
 * Sources:
 *   - "FlashBias: Fast Computation of Attention with Bias", Abstract: attention
 *     with bias adds a bias matrix to the query-key scores before the softmax.
 *   - "Rank-Factorized Implicit Neural Bias: Scaling Super-Resolution Transformer
 *     with FlashAttention", Abstract: the positional bias is approximated by
 *     low-rank factors, concatenated with the content tokens along channels, so
 *     the element-wise bias addition becomes part of one dot product.  The oracle
 *     deliberately does NOT use that concatenation: it forms the bias matrix
 *     explicitly and adds it, which is the definition the concatenation must
 *     reproduce.
 *   - The scale convention (s multiplies Q K^T only, not the bias) is the
 *     plainest reading of "an additive bias to the scores"; the pages do not
 *     place s explicitly.
 *
 * Backward, for an upstream gradient dO (plain chain rule through the above):
 *   dP_ij = dO_i . V_j
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = s sum_j dS_ij K_j        dU_i = sum_j dS_ij W_j
 *   dK_j  = s sum_i dS_ij Q_i        dW_j = sum_i dS_ij U_i
 *   dV_j  =   sum_i P_ij dO_i
 * Each output element is computed as its own plain sum (a gather over the
 * other index); P is recomputed from the inputs, never taken from a stored
 * forward result.
 *
 * Layout: every tensor is contiguous [BH, N, c] with c = d (Q, K, V, O, dO and
 * their gradients) or c = r (U, W, dU, dW); LSE and D are [BH, N].
 * r == 0 is allowed (U, W may then be NULL); the bias is then zero.
 *
 * Threads: OpenMP over independent output rows; nthreads <= 0 means the
 * OpenMP default.  No BLAS, no blocking beyond one row at a time.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double dot(const double* a, const double* b, long n) {
    double acc = 0.0;
    for (long c = 0; c < n; ++c) acc += a[c] * b[c];
    return acc;
}

/* Row i of S for one head: S_ij = s * (q_i . k_j) + bias_ij, with the bias row
 * bias_ij = u_i . w_j formed explicitly first. */
static void score_row(const double* q, const double* k, const double* u, const double* w,
                      long N, long d, long r, double s, long i, double* bias_row,
                      double* s_row) {
    for (long j = 0; j < N; ++j)
        bias_row[j] = (r > 0) ? dot(u + i * r, w + j * r, r) : 0.0;
    for (long j = 0; j < N; ++j)
        s_row[j] = s * dot(q + i * d, k + j * d, d) + bias_row[j];
}

/* Softmax of one row in place; returns LSE = m + log(sum_j exp(S_j - m)). */
static double softmax_row(double* row, long N) {
    double m = -INFINITY;
    for (long j = 0; j < N; ++j)
        if (row[j] > m) m = row[j];
    double sum = 0.0;
    for (long j = 0; j < N; ++j) {
        row[j] = exp(row[j] - m);
        sum += row[j];
    }
    for (long j = 0; j < N; ++j) row[j] /= sum;
    return m + log(sum);
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int rfb_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Forward for the query rows rows[0..nrows) of every head in [bh0, bh1).
 * o: [bh1-bh0, nrows, d], lse: [bh1-bh0, nrows].  rows == NULL means all N
 * rows in order (then nrows must equal N). */
int rfb_oracle_fwd(const double* q, const double* k, const double* v, const double* u,
                   const double* w, double* o, double* lse, long BH, long N, long d, long r,
                   double s, long bh0, long bh1, const long* rows, long nrows, int nthreads) {
    if (N < 1 || d < 1 || r < 0 || bh0 < 0 || bh1 > BH || bh0 > bh1 || nrows < 0) return 1;
    if (!rows && nrows != N) return 1;
    set_threads(nthreads);
    long nh = bh1 - bh0;
    int bad = 0;
#pragma omp parallel
    {
        double* bias_row = (double*)malloc(sizeof(double) * N);
        double* p = (double*)malloc(sizeof(double) * N);
        if (!bias_row || !p) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (long hh = 0; hh < nh; ++hh) {
            for (long t = 0; t < nrows; ++t) {
                if (!bias_row || !p) continue;
                long bh = bh0 + hh;
                long i = rows ? rows[t] : t;
                if (i < 0 || i >= N) {
#pragma omp atomic write
                    bad = 1;
                    continue;
                }
                const double* qh = q + bh * N * d;
                const double* kh = k + bh * N * d;
                const double* vh = v + bh * N * d;
                const double* uh = r ? u + bh * N * r : NULL;
                const double* wh = r ? w + bh * N * r : NULL;
                score_row(qh, kh, uh, wh, N, d, r, s, i, bias_row, p);
                double l = softmax_row(p, N);
                double* orow = o + (hh * nrows + t) * d;
                for (long c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < N; ++j) acc += p[j] * vh[j * d + c];
                    orow[c] = acc;
                }
                lse[hh * nrows + t] = l;
            }
        }
        free(bias_row);
        free(p);
    }
    return bad;
}

/* Row quantities of the backward for query row i of one head:
 * p[j] = P_ij, ds[j] = dS_ij.  Returns D_i. */
static double bwd_row(const double* qh, const double* kh, const double* vh, const double* uh,
                      const double* wh, const double* doh, long N, long d, long r, double s,
                      long i, double* bias_row, double* p, double* ds) {
    score_row(qh, kh, uh, wh, N, d, r, s, i, bias_row, p);
    softmax_row(p, N);
    double D = 0.0;
    for (long j = 0; j < N; ++j) {
        ds[j] = dot(doh + i * d, vh + j * d, d); /* dP_ij */
        D += p[j] * ds[j];
    }
    for (long j = 0; j < N; ++j) ds[j] = p[j] * (ds[j] - D);
    return D;
}

/* Full backward for every head in [bh0, bh1).  Gradient outputs are laid out
 * [bh1-bh0, N, c].  du / dw may be NULL when r == 0.  dcol_out (optional,
 * [bh1-bh0, N]) receives D_i. */
int rfb_oracle_bwd(const double* q, const double* k, const double* v, const double* u,
                   const double* w, const double* dout, double* dq, double* dk, double* dv,
                   double* du, double* dw, double* dcol_out, long BH, long N, long d, long r,
                   double s, long bh0, long bh1, int nthreads) {
    if (N < 1 || d < 1 || r < 0 || bh0 < 0 || bh1 > BH || bh0 > bh1) return 1;
    set_threads(nthreads);
    long nh = bh1 - bh0;
    double* lse_all = (double*)malloc(sizeof(double) * (nh * N > 0 ? nh * N : 1));
    double* D_all = (double*)malloc(sizeof(double) * (nh * N > 0 ? nh * N : 1));
    if (!lse_all || !D_all) {
        free(lse_all);
        free(D_all);
        return 2;
    }
    int bad = 0;
    /* Pass 1, over query rows i: LSE_i, D_i, dQ_i, dU_i. */
#pragma omp parallel
    {
        double* bias_row = (double*)malloc(sizeof(double) * N);
        double* p = (double*)malloc(sizeof(double) * N);
        double* ds = (double*)malloc(sizeof(double) * N);
        if (!bias_row || !p || !ds) {
#pragma omp atomic write
            bad = 2;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (long hh = 0; hh < nh; ++hh) {
            for (long i = 0; i < N; ++i) {
                if (!bias_row || !p || !ds) continue;
                long bh = bh0 + hh;
                const double* qh = q + bh * N * d;
                const double* kh = k + bh * N * d;
                const double* vh = v + bh * N * d;
                const double* uh = r ? u + bh * N * r : NULL;
                const double* wh = r ? w + bh * N * r : NULL;
                const double* doh = dout + bh * N * d;
                score_row(qh, kh, uh, wh, N, d, r, s, i, bias_row, p);
                lse_all[hh * N + i] = softmax_row(p, N);
                double D = 0.0;
                for (long j = 0; j < N; ++j) {
                    ds[j] = dot(doh + i * d, vh + j * d, d);
                    D += p[j] * ds[j];
                }
                for (long j = 0; j < N; ++j) ds[j] = p[j] * (ds[j] - D);
                D_all[hh * N + i] = D;
                for (long c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < N; ++j) acc += ds[j] * kh[j * d + c];
                    dq[(hh * N + i) * d + c] = s * acc;
                }
                for (long c = 0; c < r; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < N; ++j) acc += ds[j] * wh[j * r + c];
                    du[(hh * N + i) * r + c] = acc;
                }
            }
        }
        free(bias_row);
        free(p);
        free(ds);
    }
    /* Pass 2, over key rows j: dK_j, dW_j, dV_j, each a sum over all query rows i,
     * with P_ij = exp(S_ij - LSE_i) and dS_ij = P_ij (dP_ij - D_i). */
#pragma omp parallel
    {
        double* accK = (double*)malloc(sizeof(double) * (d + 1));
        double* accV = (double*)malloc(sizeof(double) * (d + 1));
        double* accW = (double*)malloc(sizeof(double) * (r + 1));
        if (!accK || !accV || !accW) {
#pragma omp atomic write
            bad = 2;
        }
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (long hh = 0; hh < nh; ++hh) {
            for (long j = 0; j < N; ++j) {
                if (!accK || !accV || !accW) continue;
                long bh = bh0 + hh;
                const double* qh = q + bh * N * d;
                const double* kh = k + bh * N * d;
                const double* vh = v + bh * N * d;
                const double* uh = r ? u + bh * N * r : NULL;
                const double* wh = r ? w + bh * N * r : NULL;
                const double* doh = dout + bh * N * d;
                for (long c = 0; c < d; ++c) accK[c] = accV[c] = 0.0;
                for (long c = 0; c < r; ++c) accW[c] = 0.0;
                for (long i = 0; i < N; ++i) {
                    double bias = (r > 0) ? dot(uh + i * r, wh + j * r, r) : 0.0;
                    double S = s * dot(qh + i * d, kh + j * d, d) + bias;
                    double P = exp(S - lse_all[hh * N + i]);
                    double dP = dot(doh + i * d, vh + j * d, d);
                    double dS = P * (dP - D_all[hh * N + i]);
                    for (long c = 0; c < d; ++c) {
                        accV[c] += P * doh[i * d + c];
                        accK[c] += dS * qh[i * d + c];
                    }
                    for (long c = 0; c < r; ++c) accW[c] += dS * uh[i * r + c];
                }
                for (long c = 0; c < d; ++c) {
                    dv[(hh * N + j) * d + c] = accV[c];
                    dk[(hh * N + j) * d + c] = s * accK[c];
                }
                for (long c = 0; c < r; ++c) dw[(hh * N + j) * r + c] = accW[c];
            }
        }
        free(accK);
        free(accV);
        free(accW);
    }
    if (dcol_out) memcpy(dcol_out, D_all, sizeof(double) * nh * N);
    free(lse_all);
    free(D_all);
    return bad;
}

/* Backward restricted to the query-side gradients dQ_i, dU_i (and D_i) of the
 * listed query rows of one head bh: each needs only row i of P and dS, so it
 * is cheap at any N.  dq: [nrows, d], du: [nrows, r], dcol: [nrows] or NULL. */
int rfb_oracle_bwd_query_rows(const double* q, const double* k, const double* v,
                              const double* u, const double* w, const double* dout, double* dq,
                              double* du, double* dcol, long BH, long N, long d, long r,
                              double s, long bh, const long* rows, long nrows, int nthreads) {
    if (N < 1 || d < 1 || r < 0 || bh < 0 || bh >= BH || nrows < 0 || !rows) return 1;
    set_threads(nthreads);
    int bad = 0;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    const double* uh = r ? u + bh * N * r : NULL;
    const double* wh = r ? w + bh * N * r : NULL;
    const double* doh = dout + bh * N * d;
#pragma omp parallel
    {
        double* bias_row = (double*)malloc(sizeof(double) * N);
        double* p = (double*)malloc(sizeof(double) * N);
        double* ds = (double*)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
        for (long t = 0; t < nrows; ++t) {
            long i = rows[t];
            if (!bias_row || !p || !ds || i < 0 || i >= N) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            double D = bwd_row(qh, kh, vh, uh, wh, doh, N, d, r, s, i, bias_row, p, ds);
            if (dcol) dcol[t] = D;
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long j = 0; j < N; ++j) acc += ds[j] * kh[j * d + c];
                dq[t * d + c] = s * acc;
            }
            for (long c = 0; c < r; ++c) {
                double acc = 0.0;
                for (long j = 0; j < N; ++j) acc += ds[j] * wh[j * r + c];
                du[t * r + c] = acc;
            }
        }
        free(bias_row);
        free(p);
        free(ds);
    }
    return bad;
}
