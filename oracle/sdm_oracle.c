/*
 * sdm_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.
 *
 * A plain, slow, single-threaded CPU restatement of the Sparse Delta Memory (SDM)
 * per-head memory pass.  Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this file's library.  It shares no code, header,
 * table or helper with the CUDA library: it is an independent statement of the
 * method, written from the descriptions of the method and in double precision.
 *
 * Sources (each function names the passage it follows):
 *   [P5]  "Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity"
 *         (paper.rainbus.top summary), method paragraph: step 1 (sparse key
 *         selection), step 2 (gated delta write), step 3 (sparse read),
 *         step 4 (normalisation, gating, head mixing).
 *   [P1]  "用稀疏内存把线性RNN的状态放大1000倍" (ai-paper-analysis.pages.dev),
 *         sections 步骤 1 .. 步骤 4 and the learned-initial-state section.
 *   [P3]  m.163.com article on SDM, section 二 (product keys: top candidates per
 *         half, then combination) and section 三 (learnable M0).
 *
 * Readings taken where the pages are silent (all listed with the design notes):
 *   - flat slot index of the pair (i1, i2) is i1*S2 + i2, i1 indexing the first half;
 *   - a score is the fp32 sum of the two fp32 half scores; the order used at every
 *     stage is (score descending, index ascending); -0 and +0 are the same score;
 *   - the slot weight k^(i) (write) and q^(i) (read) is the softmax, at temperature
 *     one, of the selected scores over the selected set only;
 *   - alpha_t and beta_t are per (token, head) scalars given as inputs;
 *   - the write of token t happens before its read (y_t reads M_t);
 *   - the delta prediction term is per slot (M~[i] of the slot being written); a second
 *     entry point takes the coupled reading (one prediction shared by the token's written
 *     rows), the one under which the method reduces to the gated delta rule;
 *   - RMSNorm is over d_v with epsilon eps and optional weight gamma; the output
 *     gate is act(g) with act in {silu, sigmoid, identity}.
 *
 * NaN scores are outside the supported input domain.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_UNTRACKED (-2)
#define ORACLE_ERR_NOMEM (-3)

typedef struct {
    float s;   /* score */
    int64_t i; /* index (per-half index, or flat slot index) */
} scored_t;

/* Does a come before b in (score descending, index ascending) order?  C compares
 * -0.0f == +0.0f as equal, so the two zeros fall through to the index tie-break. */
static int before(const scored_t *a, const scored_t *b) {
    if (a->s != b->s) return a->s > b->s;
    return a->i < b->i;
}

/* Keeps best[0 .. *n) as the first (at most K) items seen so far, in order: the new item
 * is inserted at its place and the item pushed past position K falls off. */
static void keep_top(scored_t *best, int *n, int K, scored_t c) {
    int pos = *n;
    if (pos == K) {
        if (!before(&c, &best[K - 1])) return;
        pos = K - 1;
    } else {
        (*n)++;
    }
    while (pos > 0 && before(&c, &best[pos - 1])) {
        best[pos] = best[pos - 1];
        --pos;
    }
    best[pos] = c;
}

/* Softmax of the selected scores over the selected set [P1 step 2: k_t^(i) is the
 * slot's write weight; P1 Fig. 6 / P3 section 七: weights are ranked "by softmax
 * score" and their top-m mass is measured over the selected set].  sel[0] holds the
 * largest score. */
static void softmax_selected(const scored_t *sel, int K, double *wt) {
    double s0 = (double)sel[0].s;
    double total = 0.0;
    for (int j = 0; j < K; ++j) {
        wt[j] = exp((double)sel[j].s - s0);
        total += wt[j];
    }
    for (int j = 0; j < K; ++j) wt[j] /= total;
}

/*
 * Step 1, sparse key selection, for n score rows.  Row r holds the two halves
 * k'_1 (S1 values) then k'_2 (S2 values) at halves + r*row_stride.
 *
 * mode 0 (product-key route) [P5 step 1; P1 步骤 1; P3 section 二]: top-K of each
 *   half, then top-K of the K1*K2 candidate outer sums (K1=min(K,S1), K2=min(K,S2)).
 * mode 1 (definition): top-K of all N = S1*S2 outer sums.
 *
 * Outputs, per row: idx[r*K + j] flat slot index, wt[r*K + j] softmax weight, in
 * selection order.  *n_scored (optional) receives the number of candidate sums
 * scored for the last row.
 */
int sdm_oracle_select(const float *halves, long n, long row_stride, int S1, int S2, int K,
                      int mode, int32_t *idx, double *wt, long *n_scored) {
    if (!halves || !idx || !wt || n < 0 || S1 < 1 || S2 < 1 || K < 1) return ORACLE_ERR_ARG;
    const long N = (long)S1 * (long)S2;
    if ((long)K > N || N > 2147483647L) return ORACLE_ERR_ARG;
    if (mode != 0 && mode != 1) return ORACLE_ERR_ARG;
    const int K1 = K < S1 ? K : S1;
    const int K2 = K < S2 ? K : S2;
    if ((long)K1 * (long)K2 < (long)K) return ORACLE_ERR_ARG;

    scored_t *h1 = (scored_t *)malloc(sizeof(scored_t) * (size_t)K1);
    scored_t *h2 = (scored_t *)malloc(sizeof(scored_t) * (size_t)K2);
    scored_t *top = (scored_t *)malloc(sizeof(scored_t) * (size_t)K);
    if (!h1 || !h2 || !top) {
        free(h1); free(h2); free(top);
        return ORACLE_ERR_NOMEM;
    }
    for (long r = 0; r < n; ++r) {
        const float *k1 = halves + r * row_stride; /* first half, length S1 */
        const float *k2 = k1 + S1;                 /* second half, length S2 */
        long nc = 0;
        int ntop = 0;
        if (mode == 0) {
            int n1 = 0, n2 = 0;
            for (int a = 0; a < S1; ++a) {
                scored_t c = {k1[a], a};
                keep_top(h1, &n1, K1, c);
            }
            for (int b = 0; b < S2; ++b) {
                scored_t c = {k2[b], b};
                keep_top(h2, &n2, K2, c);
            }
            for (int a = 0; a < K1; ++a) {
                for (int b = 0; b < K2; ++b) {
                    scored_t c;
                    c.s = h1[a].s + h2[b].s; /* one fp32 addition */
                    c.i = h1[a].i * (int64_t)S2 + h2[b].i;
                    keep_top(top, &ntop, K, c);
                    ++nc;
                }
            }
        } else {
            for (int a = 0; a < S1; ++a) {
                for (int b = 0; b < S2; ++b) {
                    scored_t c;
                    c.s = k1[a] + k2[b];
                    c.i = (int64_t)a * S2 + b;
                    keep_top(top, &ntop, K, c);
                    ++nc;
                }
            }
        }
        for (int j = 0; j < K; ++j) idx[r * K + j] = (int32_t)top[j].i;
        softmax_selected(top, K, wt + r * K);
        if (n_scored) *n_scored = nc;
    }
    free(h1); free(h2); free(top);
    return ORACLE_OK;
}

/*
 * Steps 2 and 3 for one (sequence, head) over tokens 0..T-1, on a tracked subset of
 * the N memory rows (rows == NULL tracks all N rows, in slot order).
 *
 * Step 2, gated delta write [P5 step 2; P1 步骤 2]: for every selected write slot i
 * of token t, M~[i] = alpha_t * M[i], then M[i] = M~[i] + beta_t * k^(i) * (v_t - M~[i]);
 * unselected slots keep their value.  Rows evolve independently of one another, so
 * restricting the pass to a subset of rows changes nothing for those rows.
 *
 * Step 3, sparse read [P5 step 3; P1 步骤 3]: y_t = sum over the R read slots of
 * q^(i) * M_t[i], taken after token t's write.  The read rows of every token with
 * want_y[t] != 0 (want_y == NULL: every token) must be tracked.
 *
 *   idx_w/wt_w [T, W], idx_r/wt_r [T, R]   selection of step 1
 *   v: v_t at v + t*v_stride (d_v floats)   alpha_t, beta_t at alpha/beta + t*ab_stride
 *   M_in  [n_rows, d_v] initial values of the tracked rows (fp32)
 *   y     [T, d_v] read result (double); rows of unwanted tokens are left untouched
 *   M_out [n_rows, d_v] final values of the tracked rows (rounded to fp32)
 */
static int pass_impl(int T, int N, int d_v, int W, int R, const int32_t *idx_w,
                     const double *wt_w, const int32_t *idx_r, const double *wt_r,
                     const float *v, long v_stride, const float *alpha, const float *beta,
                     long ab_stride, int n_rows, const int32_t *rows, const float *M_in,
                     const uint8_t *want_y, double *y, float *M_out, int coupled,
                     double *wlog) {
    if (T < 0 || N < 1 || d_v < 1 || W < 1 || R < 1 || n_rows < 0) return ORACLE_ERR_ARG;
    if (!idx_w || !wt_w || !idx_r || !wt_r || !v || !alpha || !beta || !M_in || !M_out)
        return ORACLE_ERR_ARG;
    if (!rows && n_rows != N) return ORACLE_ERR_ARG;

    int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    double *S = (double *)malloc(sizeof(double) * (size_t)n_rows * (size_t)d_v + 1);
    double *acc = (double *)malloc(sizeof(double) * (size_t)d_v);
    double *pred = (double *)malloc(sizeof(double) * (size_t)d_v);
    if (!pos || !S || !acc || !pred) {
        free(pos); free(S); free(acc); free(pred);
        return ORACLE_ERR_NOMEM;
    }
    for (int i = 0; i < N; ++i) pos[i] = rows ? -1 : i;
    if (rows) {
        for (int p = 0; p < n_rows; ++p) {
            if (rows[p] < 0 || rows[p] >= N) {
                free(pos); free(S); free(acc); free(pred);
                return ORACLE_ERR_ARG;
            }
            pos[rows[p]] = p;
        }
    }
    for (long e = 0; e < (long)n_rows * d_v; ++e) S[e] = (double)M_in[e];

    int rc = ORACLE_OK;
    for (int t = 0; t < T && rc == ORACLE_OK; ++t) {
        const double a_t = (double)alpha[(long)t * ab_stride];
        const double b_t = (double)beta[(long)t * ab_stride];
        const float *v_t = v + (long)t * v_stride;
        /* step 2, coupled reading: the token's written rows share one prediction,
         * pred = sum over the write set of k_j * alpha_t * M[j]; then each written row
         * becomes alpha_t * M[i] + beta_t * k_i * (v_t - pred).  Every written row must be
         * tracked: the prediction reads them all. */
        if (coupled) {
            for (int c = 0; c < d_v; ++c) pred[c] = 0.0;
            for (int j = 0; j < W && rc == ORACLE_OK; ++j) {
                const int32_t i = idx_w[(long)t * W + j];
                if (i < 0 || i >= N) rc = ORACLE_ERR_ARG;
                else if (pos[i] < 0) rc = ORACLE_ERR_UNTRACKED;
                else {
                    const double kj = wt_w[(long)t * W + j];
                    const double *row = S + (long)pos[i] * d_v;
                    for (int c = 0; c < d_v; ++c) pred[c] += kj * (a_t * row[c]);
                }
            }
            if (rc != ORACLE_OK) break;
            for (int j = 0; j < W; ++j) {
                const int32_t i = idx_w[(long)t * W + j];
                const double kj = wt_w[(long)t * W + j];
                double *row = S + (long)pos[i] * d_v;
                if (wlog)
                    for (int c = 0; c < d_v; ++c) wlog[((long)t * W + j) * d_v + c] = row[c];
                for (int c = 0; c < d_v; ++c)
                    row[c] = a_t * row[c] + b_t * kj * ((double)v_t[c] - pred[c]);
            }
        }
        /* step 2: gated delta write on the selected write slots */
        for (int j = 0; j < W && !coupled; ++j) {
            const int32_t i = idx_w[(long)t * W + j];
            if (i < 0 || i >= N) { rc = ORACLE_ERR_ARG; break; }
            const int p = pos[i];
            if (p < 0) { /* untracked row: cannot influence tracked ones */
                if (wlog)
                    for (int c = 0; c < d_v; ++c) wlog[((long)t * W + j) * d_v + c] = NAN;
                continue;
            }
            const double k_i = wt_w[(long)t * W + j];
            double *m = S + (long)p * d_v;
            /* the undo log: the row as the write found it */
            if (wlog)
                for (int c = 0; c < d_v; ++c) wlog[((long)t * W + j) * d_v + c] = m[c];
            for (int c = 0; c < d_v; ++c) {
                const double m_tilde = a_t * m[c];
                m[c] = m_tilde + b_t * k_i * ((double)v_t[c] - m_tilde);
            }
        }
        if (rc != ORACLE_OK) break;
        /* step 3: sparse read after the write */
        if (want_y && !want_y[t]) continue;
        if (!y) continue;
        for (int c = 0; c < d_v; ++c) acc[c] = 0.0;
        for (int j = 0; j < R; ++j) {
            const int32_t i = idx_r[(long)t * R + j];
            if (i < 0 || i >= N) { rc = ORACLE_ERR_ARG; break; }
            const int p = pos[i];
            if (p < 0) { rc = ORACLE_ERR_UNTRACKED; break; }
            const double q_i = wt_r[(long)t * R + j];
            const double *m = S + (long)p * d_v;
            for (int c = 0; c < d_v; ++c) acc[c] += q_i * m[c];
        }
        if (rc != ORACLE_OK) break;
        for (int c = 0; c < d_v; ++c) y[(long)t * d_v + c] = acc[c];
    }
    if (rc == ORACLE_OK)
        for (long e = 0; e < (long)n_rows * d_v; ++e) M_out[e] = (float)S[e];
    free(pos); free(S); free(acc); free(pred);
    return rc;
}

int sdm_oracle_pass(int T, int N, int d_v, int W, int R, const int32_t *idx_w,
                    const double *wt_w, const int32_t *idx_r, const double *wt_r,
                    const float *v, long v_stride, const float *alpha, const float *beta,
                    long ab_stride, int n_rows, const int32_t *rows, const float *M_in,
                    const uint8_t *want_y, double *y, float *M_out) {
    return pass_impl(T, N, d_v, W, R, idx_w, wt_w, idx_r, wt_r, v, v_stride, alpha, beta,
                     ab_stride, n_rows, rows, M_in, want_y, y, M_out, 0, NULL);
}

/*
 * sdm_oracle_pass that also keeps the undo log of the in-place update [m.163.com article on
 * SDM, section 八, the memory-efficiency paragraph: training updates the state in place and
 * undoes the updates during backpropagation]: wlog[(t * W + j) * d_v + c] is written slot j
 * of token t as that token's write found it, before the write (NaN for an untracked row).
 * Replaying the log backwards restores the state the pass started from.
 */
int sdm_oracle_pass_logged(int T, int N, int d_v, int W, int R, const int32_t *idx_w,
                           const double *wt_w, const int32_t *idx_r, const double *wt_r,
                           const float *v, long v_stride, const float *alpha,
                           const float *beta, long ab_stride, int n_rows, const int32_t *rows,
                           const float *M_in, const uint8_t *want_y, double *y, float *M_out,
                           double *wlog) {
    if (!wlog) return ORACLE_ERR_ARG;
    return pass_impl(T, N, d_v, W, R, idx_w, wt_w, idx_r, wt_r, v, v_stride, alpha, beta,
                     ab_stride, n_rows, rows, M_in, want_y, y, M_out, 0, wlog);
}

/*
 * Steps 2 and 3 with the coupled delta rule.  [P1] and [P3] state that SDM reduces exactly
 * to the gated delta rule (GDN) when every slot is selected; the per-slot write of [P5]
 * does not, while this one does: with the write set all N slots and key k (the slot
 * weights), M_t = alpha_t (I - beta_t k k^T) M_{t-1} + beta_t k v_t^T.  Arguments as for
 * sdm_oracle_pass; every written row must be tracked (ORACLE_ERR_UNTRACKED otherwise).
 */
int sdm_oracle_pass_coupled(int T, int N, int d_v, int W, int R, const int32_t *idx_w,
                            const double *wt_w, const int32_t *idx_r, const double *wt_r,
                            const float *v, long v_stride, const float *alpha,
                            const float *beta, long ab_stride, int n_rows,
                            const int32_t *rows, const float *M_in, const uint8_t *want_y,
                            double *y, float *M_out) {
    return pass_impl(T, N, d_v, W, R, idx_w, wt_w, idx_r, wt_r, v, v_stride, alpha, beta,
                     ab_stride, n_rows, rows, M_in, want_y, y, M_out, 1, NULL);
}

/*
 * Step 4 without the head-mixing projection [P5 step 4; P1 步骤 4]: RMS normalisation
 * of y over d_v, optional weight gamma, then elementwise gating by act(g).
 *   act: 0 = silu, g / (1 + e^-g); 1 = sigmoid, 1 / (1 + e^-g); 2 = identity.
 * g == NULL means no gating factor; gamma == NULL means unit weight.
 * Processes n vectors of d_v values.
 */
int sdm_oracle_norm_gate(long n, int d_v, const double *y, const float *g, const float *gamma,
                         double eps, int act, double *o) {
    if (n < 0 || d_v < 1 || !y || !o || act < 0 || act > 2 || eps < 0.0) return ORACLE_ERR_ARG;
    for (long r = 0; r < n; ++r) {
        const double *yr = y + r * d_v;
        double ss = 0.0;
        for (int c = 0; c < d_v; ++c) ss += yr[c] * yr[c];
        const double inv_rms = 1.0 / sqrt(ss / (double)d_v + eps);
        for (int c = 0; c < d_v; ++c) {
            double gate = 1.0;
            if (g) {
                const double x = (double)g[r * d_v + c];
                if (act == 0) gate = x / (1.0 + exp(-x));
                else if (act == 1) gate = 1.0 / (1.0 + exp(-x));
                else gate = x;
            }
            const double w = gamma ? (double)gamma[c] : 1.0;
            o[r * d_v + c] = yr[c] * inv_rms * w * gate;
        }
    }
    return ORACLE_OK;
}
