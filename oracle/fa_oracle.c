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
 *  - Multi-query / grouped-query attention ("K/V shared across heads", fewer KV heads) and sliding-window
 *    attention (window_size = (left, right), (-1, -1) = none): skill page, Workflow 2, Steps 2 and 3.
 *  - Attention dropout (the `dropout_p` argument of the skill page's flash_attn_func call, Workflow 2 Step 2):
 *    the pages name the argument only; the reading below is the usual one (inverted dropout on the
 *    attention probabilities).
 *  - The dropout mask comes from Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and Shaw,
 *    "Parallel random numbers: as easy as 1, 2, 3" (SC 2011), written here from that definition.
 *
 * Readings where the pages are silent:
 *  - causal mask with Sq != Sk is bottom-right aligned: key j is visible to query i iff j <= i + (Sk - Sq);
 *  - the window is aligned the same way: with c = i + (Sk - Sq), key j is visible iff
 *    (left < 0 or j >= c - left) and (right < 0 or j <= c + right), on top of the causal condition;
 *  - grouped heads: q head h reads K/V head h / (n_q_heads / n_kv_heads); dK and dV of a K/V head sum the
 *    contributions of its group of q heads;
 *  - LSE_i is the natural log of sum_{j visible} exp(s_ij), scale included;
 *  - a query row with no visible key has O_i = 0, LSE_i = -inf and zero gradients;
 *  - dropout: the drop probability is rounded to t / 256, t = floor(256 dropout_p + 1/2) (t <= 255); element
 *    (i, j) of head number bh (b * n_q_heads + h) is kept iff byte (j mod 4) of word (i mod 4) of
 *    Philox4x32-10(counter = (i / 4, j / 4, bh, offset), key = (seed mod 2^32, seed / 2^32)) is >= t (byte 0 =
 *    least significant); kept probabilities are multiplied by 1 / (1 - t / 256), so that O is unbiased;
 *    LSE is that of the undropped scores. With Z_ij = keep_ij / (1 - t/256):
 *      O_i = sum_j P_ij Z_ij v_j,   dV_j = sum_i P_ij Z_ij dO_i,   dP_ij = Z_ij (dO_i . v_j),
 *      D_i = sum_j P_ij dP_ij (= dO_i . O_i),   dS_ij = P_ij (dP_ij - D_i).
 *
 * Layouts: every matrix is one attention head, row-major, fp64.
 *   q, dout : [n_q_heads][Sq][D]      k, v : [n_kv_heads][Sk][D]   (n_q_heads a multiple of n_kv_heads)
 *   rows    : [n_q_heads][n_rows]     query-row indices (0 <= rows < Sq) evaluated for each q head
 *   out, dq : [n_q_heads][n_rows][D]  lse  : [n_q_heads][n_rows]
 *   dk, dv  : [n_kv_heads][Sk][D]     contributions of the listed rows only (the gradient of
 *                                     L = sum over listed rows i of dout_i . O_i), summed over each group
 * Return value: 0 on success, -1 on an invalid argument (nothing written).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Size of the OpenMP team that the parallel loops below use when called from this thread (n >= 1; n < 1 leaves
 * it unchanged); returns the team size now in effect. Lets a caller that times the oracle in different
 * processes use the same number of threads in each. */
int oracle_set_threads(int n)
{
    if (n >= 1) omp_set_num_threads(n);
    return omp_get_max_threads();
}

/* ---------------------------------------------------------------------------------------- Philox4x32-10 */

/* Round constants of Philox4x32 (the SC 2011 paper): two multipliers and the two Weyl key increments (golden
 * ratio and sqrt(3) - 1, as 32-bit fractions). */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

/* out = Philox4x32 with 10 rounds applied to counter ctr under key key. One round multiplies words 0 and 2 by
 * the two multipliers (64-bit products) and recombines: (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1,
 * lo(M0 c0)); the key advances by the Weyl increments before every round after the first. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        uint32_t n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        uint32_t n3 = (uint32_t)p0;
        c0 = n0;
        c1 = n1;
        c2 = n2;
        c3 = n3;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* The dropout rule of one call: threshold t (0 = no dropout), Philox key and counter word 3. */
struct dropout {
    int t;
    uint32_t key[2];
    uint32_t offset;
};

/* Threshold t = floor(256 p + 1/2); -1 if p is outside [0, 1) or rounds to 256. */
static int dropout_threshold(double p)
{
    if (!(p >= 0.0 && p < 1.0)) return -1;
    int t = (int)floor(256.0 * p + 0.5);
    return t <= 255 ? t : -1;
}

/* Z_ij for head number bh: 1 / (1 - t/256) if kept, 0 if dropped; 1 without dropout. */
static double dropout_z(const struct dropout *dr, int64_t bh, int64_t i, int64_t j)
{
    if (dr->t == 0) return 1.0;
    uint32_t ctr[4] = {(uint32_t)(i >> 2), (uint32_t)(j >> 2), (uint32_t)bh, dr->offset};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, dr->key, w);
    uint32_t byte = (w[i & 3] >> (8 * (j & 3))) & 0xffu;
    return byte >= (uint32_t)dr->t ? 1.0 / (1.0 - dr->t / 256.0) : 0.0;
}

/* Keep mask of one head (1 kept, 0 dropped), [Sq][Sk] bytes, exported for the tests' statistics. */
int oracle_dropout_mask(double dropout_p, uint64_t seed, uint32_t offset, int64_t bh, int64_t Sq, int64_t Sk,
                        uint8_t *keep)
{
    int t = dropout_threshold(dropout_p);
    if (t < 0 || !keep || Sq < 0 || Sk < 0) return -1;
    struct dropout dr = {t, {(uint32_t)seed, (uint32_t)(seed >> 32)}, offset};
    for (int64_t i = 0; i < Sq; ++i)
        for (int64_t j = 0; j < Sk; ++j) keep[i * Sk + j] = dropout_z(&dr, bh, i, j) != 0.0;
    return 0;
}

/* ------------------------------------------------------------------------------------------- attention */

/* The visibility rule of one problem: causal flag and window bounds (negative = unbounded). */
struct mask {
    int64_t Sq, Sk;
    int causal;
    int64_t left, right;
};

/* 1 if query row i may attend to key j. */
static int visible(int64_t i, int64_t j, const struct mask *m)
{
    int64_t c = i + (m->Sk - m->Sq); /* the key aligned with query i */
    if (m->causal && j > c) return 0;
    if (m->left >= 0 && j < c - m->left) return 0;
    if (m->right >= 0 && j > c + m->right) return 0;
    return 1;
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
static double row_softmax(const double *s, int64_t i, const struct mask *mk, double *p)
{
    int64_t Sk = mk->Sk;
    double m = -INFINITY;
    for (int64_t j = 0; j < Sk; ++j)
        if (visible(i, j, mk) && s[j] > m) m = s[j];
    if (m == -INFINITY) {
        for (int64_t j = 0; j < Sk; ++j) p[j] = 0.0;
        return -INFINITY;
    }
    double sum = 0.0;
    for (int64_t j = 0; j < Sk; ++j)
        if (visible(i, j, mk)) sum += exp(s[j] - m);
    double lse = m + log(sum);
    for (int64_t j = 0; j < Sk; ++j)
        p[j] = visible(i, j, mk) ? exp(s[j] - lse) : 0.0;
    return lse;
}

static int check_args(const void *q, const void *k, const void *v, int64_t n_heads, int64_t n_kv_heads, int64_t Sq,
                      int64_t Sk, int64_t D, const int64_t *rows, int64_t n_rows)
{
    if (!q || !k || !v || !rows) return -1;
    if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads || Sq < 1 || Sk < 1 || D < 1 || n_rows < 0) return -1;
    for (int64_t t = 0; t < n_heads * n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= Sq) return -1;
    return 0;
}

/* head_index[h] = the dropout head number bh of listed head h (NULL: h itself). */
static int64_t head_number(const int64_t *head_index, int64_t h)
{
    return head_index ? head_index[h] : h;
}

static int attn_fwd(const double *q, const double *k, const double *v, int64_t n_heads, int64_t n_kv_heads,
                    int64_t Sq, int64_t Sk, int64_t D, int causal, int64_t window_left, int64_t window_right,
                    double scale, const struct dropout *dr, const int64_t *head_index, const int64_t *rows,
                    int64_t n_rows, double *out, double *lse)
{
    if (check_args(q, k, v, n_heads, n_kv_heads, Sq, Sk, D, rows, n_rows) || !out || !lse) return -1;
    const struct mask mk = {Sq, Sk, causal, window_left, window_right};
    const int64_t group = n_heads / n_kv_heads;
    int64_t total = n_heads * n_rows;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Sk);
        double *p = (double *)malloc(sizeof(double) * (size_t)Sk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < total; ++t) {
            int64_t h = t / n_rows;
            int64_t i = rows[t];
            const double *kh = k + (h / group) * Sk * D;
            const double *vh = v + (h / group) * Sk * D;
            row_scores(q + (h * Sq + i) * D, kh, Sk, D, scale, s);
            lse[t] = row_softmax(s, i, &mk, p);
            double *o = out + t * D;
            for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t j = 0; j < Sk; ++j) {
                /* O_i = sum_j P_ij Z_ij v_j (Z = 1 without dropout) */
                double pz = p[j] * dropout_z(dr, head_number(head_index, h), i, j);
                for (int64_t d = 0; d < D; ++d) o[d] += pz * vh[j * D + d];
            }
        }
        free(s);
        free(p);
    }
    return 0;
}

int oracle_attn_fwd(const double *q, const double *k, const double *v, int64_t n_heads, int64_t n_kv_heads,
                    int64_t Sq, int64_t Sk, int64_t D, int causal, int64_t window_left, int64_t window_right,
                    double scale, const int64_t *rows, int64_t n_rows, double *out, double *lse)
{
    const struct dropout none = {0, {0, 0}, 0};
    return attn_fwd(q, k, v, n_heads, n_kv_heads, Sq, Sk, D, causal, window_left, window_right, scale, &none, NULL,
                    rows, n_rows, out, lse);
}

int oracle_attn_fwd_dropout(const double *q, const double *k, const double *v, int64_t n_heads, int64_t n_kv_heads,
                            int64_t Sq, int64_t Sk, int64_t D, int causal, int64_t window_left,
                            int64_t window_right, double scale, double dropout_p, uint64_t seed, uint32_t offset,
                            const int64_t *head_index, const int64_t *rows, int64_t n_rows, double *out,
                            double *lse)
{
    const struct dropout dr = {dropout_threshold(dropout_p), {(uint32_t)seed, (uint32_t)(seed >> 32)}, offset};
    if (dr.t < 0) return -1;
    return attn_fwd(q, k, v, n_heads, n_kv_heads, Sq, Sk, D, causal, window_left, window_right, scale, &dr,
                    head_index, rows, n_rows, out, lse);
}

static int attn_bwd(const double *q, const double *k, const double *v, const double *dout, int64_t n_heads,
                    int64_t n_kv_heads, int64_t Sq, int64_t Sk, int64_t D, int causal, int64_t window_left,
                    int64_t window_right, double scale, const struct dropout *dr, const int64_t *head_index,
                    const int64_t *rows, int64_t n_rows, double *dq, double *dk, double *dv)
{
    if (check_args(q, k, v, n_heads, n_kv_heads, Sq, Sk, D, rows, n_rows) || !dout || !dq || !dk || !dv) return -1;
    const struct mask mk = {Sq, Sk, causal, window_left, window_right};
    const int64_t group = n_heads / n_kv_heads;
    memset(dk, 0, sizeof(double) * (size_t)(n_kv_heads * Sk * D));
    memset(dv, 0, sizeof(double) * (size_t)(n_kv_heads * Sk * D));
    /* Per head: P and dS of the listed rows, kept whole so that dK and dV are plain sums over rows. */
    double *P = (double *)malloc(sizeof(double) * (size_t)(n_rows ? n_rows : 1) * (size_t)Sk);
    double *dS = (double *)malloc(sizeof(double) * (size_t)(n_rows ? n_rows : 1) * (size_t)Sk);
    /* G = P o Z, the dropped probabilities that multiply V (equal to P without dropout) */
    double *G = (double *)malloc(sizeof(double) * (size_t)(n_rows ? n_rows : 1) * (size_t)Sk);
    if (!P || !dS || !G) {
        free(P);
        free(dS);
        free(G);
        return -1;
    }
    for (int64_t h = 0; h < n_heads; ++h) {
        const double *qh = q + h * Sq * D;
        const double *kh = k + (h / group) * Sk * D;
        const double *vh = v + (h / group) * Sk * D;
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
                double *Gi = G + r * Sk;
                row_scores(qh + i * D, kh, Sk, D, scale, s);
                row_softmax(s, i, &mk, Pi);
                /* dP_ij = Z_ij (dO_i . v_j): the gradient reaching P through the dropped G = P o Z */
                for (int64_t j = 0; j < Sk; ++j) {
                    double z = dropout_z(dr, head_number(head_index, h), i, j);
                    double acc = 0.0;
                    for (int64_t d = 0; d < D; ++d) acc += doh[i * D + d] * vh[j * D + d];
                    dP[j] = z * acc;
                    Gi[j] = Pi[j] * z;
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
        /* this q head's contributions are added to its K/V head (a group shares one K/V head) */
        double *dkh = dk + (h / group) * Sk * D;
        double *dvh = dv + (h / group) * Sk * D;
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < Sk; ++j) {
            for (int64_t d = 0; d < D; ++d) {
                double gk = 0.0, gv = 0.0;
                for (int64_t r = 0; r < n_rows; ++r) {
                    int64_t i = rh[r];
                    /* dK_j = scale sum_i dS_ij q_i ;  dV_j = sum_i G_ij dO_i */
                    gk += dS[r * Sk + j] * qh[i * D + d];
                    gv += G[r * Sk + j] * doh[i * D + d];
                }
                dkh[j * D + d] += scale * gk;
                dvh[j * D + d] += gv;
            }
        }
    }
    free(P);
    free(dS);
    free(G);
    return 0;
}

int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout, int64_t n_heads,
                    int64_t n_kv_heads, int64_t Sq, int64_t Sk, int64_t D, int causal, int64_t window_left,
                    int64_t window_right, double scale, const int64_t *rows, int64_t n_rows, double *dq, double *dk,
                    double *dv)
{
    const struct dropout none = {0, {0, 0}, 0};
    return attn_bwd(q, k, v, dout, n_heads, n_kv_heads, Sq, Sk, D, causal, window_left, window_right, scale, &none,
                    NULL, rows, n_rows, dq, dk, dv);
}

int oracle_attn_bwd_dropout(const double *q, const double *k, const double *v, const double *dout, int64_t n_heads,
                            int64_t n_kv_heads, int64_t Sq, int64_t Sk, int64_t D, int causal, int64_t window_left,
                            int64_t window_right, double scale, double dropout_p, uint64_t seed, uint32_t offset,
                            const int64_t *head_index, const int64_t *rows, int64_t n_rows, double *dq, double *dk,
                            double *dv)
{
    const struct dropout dr = {dropout_threshold(dropout_p), {(uint32_t)seed, (uint32_t)(seed >> 32)}, offset};
    if (dr.t < 0) return -1;
    return attn_bwd(q, k, v, dout, n_heads, n_kv_heads, Sq, Sk, D, causal, window_left, window_right, scale, &dr,
                    head_index, rows, n_rows, dq, dk, dv);
}
