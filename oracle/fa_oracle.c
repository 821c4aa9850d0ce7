/*
 * fa_oracle.c -- plain fp64 CPU oracle for exact scaled dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's CPU-baseline leg load this
 * library; the CUDA library never includes, links or calls anything here, and this file includes nothing
 * from the CUDA library. It is deliberately slow: naive loops, a two-pass (non-online) softmax, no tiling,
 * no blocking, no fusion.
 *
 * Sources (page title, then section):
 *  - Standard attention, the definition this oracle writes out:
 *      "Flash Attention — 長い系列を扱う Transformer の学習と推論を速くする" (mlops-flash-attention skill),
 *      Workflow 1, Step 2: softmax(q @ k^T / sqrt(d_k)) @ v, with the causal flag of the quick-start call.
 *  - Default scale 1/sqrt(d) ("softmax_scale=None  # Auto-scale"): same page, Workflow 2, Step 2.
 *  - FlashAttention returns the same mathematical result as standard attention (it is exact):
 *      "FlashAttention（フラッシュアテンション）とは？…", section "よくある誤解", misconception 1.
 *  - Training (forward and backward) is supported; the pages give no backward formulas, so the backward
 *    here is the chain rule applied to the definition above.
 *
 * Readings where the pages are silent:
 *  - causal mask with Sq != Sk is bottom-right aligned: key j is visible to query i iff j <= i + (Sk - Sq);
 *  - LSE_i is the natural log of sum_{j visible} exp(s_ij), scale included;
 *  - a query row with no visible key has O_i = 0, LSE_i = -inf and zero gradients.
 *
 * Layouts: every matrix is one attention head, row-major, fp64.
 *   q, dout : [n_heads][Sq][D]      k, v : [n_heads][Sk][D]
 *   rows    : [n_heads][n_rows]     query-row indices (0 <= rows < Sq) evaluated for each head
 *   out, dq : [n_heads][n_rows][D]  lse  : [n_heads][n_rows]
 *   dk, dv  : [n_heads][Sk][D]      contributions of the listed rows only (the gradient of
 *                                   L = sum over listed rows i of dout_i . O_i)
 * Return value: 0 on success, -1 on an invalid argument (nothing written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* 1 if query row i may attend to key j. */
static int visible(int64_t i, int64_t j, int64_t Sq, int64_t Sk, int causal)
{
    if (!causal) return 1;
    return j <= i + (Sk - Sq);
}

/* Scores s_ij = scale * q_i . k_j for one row, all keys. */
static void row_scores(const double *qi, const double *k, int64_t Sk, int64_t D, double scale, double *s)
{
    for (int64_t j = 0; j < Sk; ++j) {
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qi[d] * k[j * D + d];
        s[j] = scale * acc;
    }
}

/*
 * Full (two-pass) softmax of one row over the visible keys. Writes p[j] = P_ij (0 where masked) and returns
 * LSE_i; returns -INFINITY and writes p = 0 when no key is visible.
 */
static double row_softmax(const double *s, int64_t i, int64_t Sq, int64_t Sk, int causal, double *p)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < Sk; ++j)
        if (visible(i, j, Sq, Sk, causal) && s[j] > m) m = s[j];
    if (m == -INFINITY) {
        for (int64_t j = 0; j < Sk; ++j) p[j] = 0.0;
        return -INFINITY;
    }
    double sum = 0.0;
    for (int64_t j = 0; j < Sk; ++j)
        if (visible(i, j, Sq, Sk, causal)) sum += exp(s[j] - m);
    double lse = m + log(sum);
    for (int64_t j = 0; j < Sk; ++j)
        p[j] = visible(i, j, Sq, Sk, causal) ? exp(s[j] - lse) : 0.0;
    return lse;
}

static int check_args(const void *q, const void *k, const void *v, int64_t n_heads, int64_t Sq, int64_t Sk,
                      int64_t D, const int64_t *rows, int64_t n_rows)
{
    if (!q || !k || !v || !rows) return -1;
    if (n_heads < 1 || Sq < 1 || Sk < 1 || D < 1 || n_rows < 0) return -1;
    for (int64_t t = 0; t < n_heads * n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= Sq) return -1;
    return 0;
}

int oracle_attn_fwd(const double *q, const double *k, const double *v, int64_t n_heads, int64_t Sq, int64_t Sk,
                    int64_t D, int causal, double scale, const int64_t *rows, int64_t n_rows, double *out,
                    double *lse)
{
    if (check_args(q, k, v, n_heads, Sq, Sk, D, rows, n_rows) || !out || !lse) return -1;
    int64_t total = n_heads * n_rows;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Sk);
        double *p = (double *)malloc(sizeof(double) * (size_t)Sk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < total; ++t) {
            int64_t h = t / n_rows;
            int64_t i = rows[t];
            const double *kh = k + h * Sk * D;
            const double *vh = v + h * Sk * D;
            row_scores(q + (h * Sq + i) * D, kh, Sk, D, scale, s);
            lse[t] = row_softmax(s, i, Sq, Sk, causal, p);
            double *o = out + t * D;
            for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t j = 0; j < Sk; ++j)
                for (int64_t d = 0; d < D; ++d) o[d] += p[j] * vh[j * D + d];
        }
        free(s);
        free(p);
    }
    return 0;
}

int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout, int64_t n_heads,
                    int64_t Sq, int64_t Sk, int64_t D, int causal, double scale, const int64_t *rows,
                    int64_t n_rows, double *dq, double *dk, double *dv)
{
    if (check_args(q, k, v, n_heads, Sq, Sk, D, rows, n_rows) || !dout || !dq || !dk || !dv) return -1;
    /* Per head: P and dS of the listed rows, kept whole so that dK and dV are plain sums over rows. */
    double *P = (double *)malloc(sizeof(double) * (size_t)(n_rows ? n_rows : 1) * (size_t)Sk);
    double *dS = (double *)malloc(sizeof(double) * (size_t)(n_rows ? n_rows : 1) * (size_t)Sk);
    if (!P || !dS) {
        free(P);
        free(dS);
        return -1;
    }
    for (int64_t h = 0; h < n_heads; ++h) {
        const double *qh = q + h * Sq * D;
        const double *kh = k + h * Sk * D;
        const double *vh = v + h * Sk * D;
        const double *doh = dout + h * Sq * D;
        const int64_t *rh = rows + h * n_rows;
#pragma omp parallel
        {
            double *s = (double *)malloc(sizeof(double) * (size_t)Sk);
            double *dP = (double *)malloc(sizeof(double) * (size_t)Sk);
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n_rows; ++r) {
                int64_t i = rh[r];
                double *Pi = P + r * Sk;
                double *dSi = dS + r * Sk;
                row_scores(qh + i * D, kh, Sk, D, scale, s);
                row_softmax(s, i, Sq, Sk, causal, Pi);
                /* dP_ij = dO_i . v_j */
                for (int64_t j = 0; j < Sk; ++j) {
                    double acc = 0.0;
                    for (int64_t d = 0; d < D; ++d) acc += doh[i * D + d] * vh[j * D + d];
                    dP[j] = acc;
                }
                /* D_i = sum_j P_ij dP_ij (taken from P and dP, not from dO . O) */
                double Di = 0.0;
                for (int64_t j = 0; j < Sk; ++j) Di += Pi[j] * dP[j];
                /* dS_ij = P_ij (dP_ij - D_i) */
                for (int64_t j = 0; j < Sk; ++j) dSi[j] = Pi[j] * (dP[j] - Di);
                /* dQ_i = scale sum_j dS_ij k_j */
                double *dqi = dq + (h * n_rows + r) * D;
                for (int64_t d = 0; d < D; ++d) dqi[d] = 0.0;
                for (int64_t j = 0; j < Sk; ++j)
                    for (int64_t d = 0; d < D; ++d) dqi[d] += dSi[j] * kh[j * D + d];
                for (int64_t d = 0; d < D; ++d) dqi[d] *= scale;
            }
            free(s);
            free(dP);
        }
        double *dkh = dk + h * Sk * D;
        double *dvh = dv + h * Sk * D;
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < Sk; ++j) {
            for (int64_t d = 0; d < D; ++d) {
                double gk = 0.0, gv = 0.0;
                for (int64_t r = 0; r < n_rows; ++r) {
                    int64_t i = rh[r];
                    /* dK_j = scale sum_i dS_ij q_i ;  dV_j = sum_i P_ij dO_i */
                    gk += dS[r * Sk + j] * qh[i * D + d];
                    gv += P[r * Sk + j] * doh[i * D + d];
                }
                dkh[j * D + d] = scale * gk;
                dvh[j * D + d] = gv;
            }
        }
    }
    free(P);
    free(dS);
    return 0;
}
