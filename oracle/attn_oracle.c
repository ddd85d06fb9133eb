/*
 * attn_oracle.c -- plain, slow FP64 CPU oracle for exact scaled-dot-product
 * attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg load this file's library.  It shares no code,
 * header, table or constant with the CUDA library.
 *
 * What it computes (one head at a time, every array row-major [B][H][N][d]):
 *   "Attention optimisation: FlashAttention and sparse attention" (mdooai,
 *   Ch.04), section "core formula (scaled dot-product / softmax attention)"
 *   and "formula key points":
 *     S_ij = (q_i . k_j) / sqrt(d_k)        -- here: scale * (q_i . k_j)
 *     A    = softmax over j of row i, rows of A sum to 1
 *     O_i  = sum_j A_ij v_j                 (O = AV)
 *   and its sparse-attention paragraph: a key j outside the allowed set S_i
 *   gets E_ij = -inf before the softmax, so A_ij = 0 there.  The allowed set
 *   is the AND of three masks: causal (j <= i), key padding (j < L_b) and a
 *   square block mask shared by every (b, h).
 *
 *   The forward also returns the per-row log-sum-exp of the scaled, masked
 *   logits, lse_i = m_i + log(sum_j exp(S_ij - m_i)), natural log.
 *
 *   The backward is the derivative of O = softmax(S) V, S = scale * Q K^T,
 *   written from the definition (no page states it):
 *     dA_ij = dO_i . v_j
 *     dS_ij = A_ij * (dA_ij - sum_k A_ik dA_ik)
 *     dQ_i  = scale * sum_j dS_ij k_j
 *     dK_j  = scale * sum_i dS_ij q_i
 *     dV_j  = sum_i A_ij dO_i
 *
 *   A row whose every key is masked has A_i. = 0, O_i = 0, lse_i = -inf, and
 *   contributes nothing to any gradient.
 *
 * S and A are materialised explicitly (N x N doubles per head).  OpenMP
 * splits independent rows (or independent key rows) across threads; every
 * sum runs in index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int N;
    int causal;
    const uint8_t *block_mask;   /* NULL or [nb][nb] */
    int block;                   /* block-mask granularity */
    int nb;                      /* ceil(N / block) */
    int L;                       /* valid key length of this batch entry */
} mask_t;

static int key_allowed(const mask_t *m, int i, int j)
{
    if (j >= m->L) return 0;
    if (m->causal && j > i) return 0;
    if (m->block_mask && !m->block_mask[(size_t)(i / m->block) * m->nb + (j / m->block)]) return 0;
    return 1;
}

static mask_t make_mask(int N, int causal, const uint8_t *block_mask, int block,
                        const int32_t *kv_len, int b)
{
    mask_t m;
    m.N = N;
    m.causal = causal;
    m.block_mask = block_mask;
    m.block = block > 0 ? block : 1;
    m.nb = (N + m.block - 1) / m.block;
    m.L = N;
    if (kv_len) {
        int L = kv_len[b];
        m.L = L < N ? (L < 0 ? 0 : L) : N;
    }
    return m;
}

/* One row of logits: s[j] = scale * q_i . k_j, or -inf where masked. */
static void logits_row(const double *qi, const double *k, int N, int d, double scale,
                       const mask_t *m, int i, double *s)
{
    for (int j = 0; j < N; ++j) {
        if (!key_allowed(m, i, j)) { s[j] = -INFINITY; continue; }
        double dot = 0.0;
        const double *kj = k + (size_t)j * d;
        for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
        s[j] = scale * dot;
    }
}

/* In place: logits row -> probability row; returns the log-sum-exp. */
static double softmax_row(double *s, int n)
{
    double mx = -INFINITY;
    for (int j = 0; j < n; ++j) if (s[j] > mx) mx = s[j];
    if (mx == -INFINITY) {
        for (int j = 0; j < n; ++j) s[j] = 0.0;
        return -INFINITY;
    }
    double sum = 0.0;
    for (int j = 0; j < n; ++j) {
        double e = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - mx);
        s[j] = e;
        sum += e;
    }
    for (int j = 0; j < n; ++j) s[j] /= sum;
    return mx + log(sum);
}

/* o = sum_j a[j] v_j */
static void weighted_sum_row(const double *a, const double *v, int n, int dv, double *o)
{
    for (int c = 0; c < dv; ++c) o[c] = 0.0;
    for (int j = 0; j < n; ++j) {
        double w = a[j];
        if (w == 0.0) continue;
        const double *vj = v + (size_t)j * dv;
        for (int c = 0; c < dv; ++c) o[c] += w * vj[c];
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Probabilities A (N x N) of one head; returns nothing else. */
void oracle_attn_probs(const double *q, const double *k, int N, int d, double scale,
                       int causal, const uint8_t *block_mask, int block, int kv_len_b,
                       double *A, double *lse)
{
    int32_t L = kv_len_b;
    mask_t m = make_mask(N, causal, block_mask, block, kv_len_b >= 0 ? &L : NULL, 0);
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < N; ++i) {
        double *Ai = A + (size_t)i * N;
        logits_row(q + (size_t)i * d, k, N, d, scale, &m, i, Ai);
        double l = softmax_row(Ai, N);
        if (lse) lse[i] = l;
    }
}

/* From given logits S (rows x cols, -inf = masked): O = softmax(S) V, lse. */
void oracle_softmax_av(const double *S, const double *v, int rows, int cols, int dv,
                       double *o, double *lse, double *A_out)
{
    #pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)cols);
        #pragma omp for schedule(static)
        for (int i = 0; i < rows; ++i) {
            memcpy(a, S + (size_t)i * cols, sizeof(double) * (size_t)cols);
            double l = softmax_row(a, cols);
            if (lse) lse[i] = l;
            if (A_out) memcpy(A_out + (size_t)i * cols, a, sizeof(double) * (size_t)cols);
            weighted_sum_row(a, v, cols, dv, o + (size_t)i * dv);
        }
        free(a);
    }
}

/* Forward over every head: S and A of one head are materialised, then O = AV. */
int oracle_attn_fwd(const double *q, const double *k, const double *v,
                    int B, int H, int N, int d, double scale, int causal,
                    const uint8_t *block_mask, int block, const int32_t *kv_len,
                    double *o, double *lse)
{
    double *A = (double *)malloc(sizeof(double) * (size_t)N * (size_t)N);
    if (!A) return -1;
    for (int b = 0; b < B; ++b) {
        mask_t m = make_mask(N, causal, block_mask, block, kv_len, b);
        for (int h = 0; h < H; ++h) {
            size_t off = ((size_t)b * H + h) * (size_t)N * d;
            const double *qh = q + off, *kh = k + off, *vh = v + off;
            double *oh = o + off;
            double *lh = lse + ((size_t)b * H + h) * (size_t)N;
            #pragma omp parallel for schedule(static)
            for (int i = 0; i < N; ++i) {
                double *Ai = A + (size_t)i * N;
                logits_row(qh + (size_t)i * d, kh, N, d, scale, &m, i, Ai);
                lh[i] = softmax_row(Ai, N);
            }
            #pragma omp parallel for schedule(static)
            for (int i = 0; i < N; ++i)
                weighted_sum_row(A + (size_t)i * N, vh, N, d, oh + (size_t)i * d);
        }
    }
    free(A);
    return 0;
}

/* Forward for selected rows only (flat index (b*H + h)*N + i): the same
 * definition restricted to those rows of S and A. */
int oracle_attn_fwd_rows(const double *q, const double *k, const double *v,
                         int B, int H, int N, int d, double scale, int causal,
                         const uint8_t *block_mask, int block, const int32_t *kv_len,
                         const int64_t *rows, int nrows, double *o_rows, double *lse_rows)
{
    (void)B;
    int bad = 0;
    #pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)N);
        #pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            int64_t flat = rows[r];
            int64_t bh = flat / N;
            int i = (int)(flat % N);
            int b = (int)(bh / H);
            if (flat < 0 || b >= B) { bad = 1; continue; }
            mask_t m = make_mask(N, causal, block_mask, block, kv_len, b);
            size_t off = (size_t)bh * (size_t)N * d;
            logits_row(q + off + (size_t)i * d, k + off, N, d, scale, &m, i, a);
            lse_rows[r] = softmax_row(a, N);
            weighted_sum_row(a, v + off, N, d, o_rows + (size_t)r * d);
        }
        free(a);
    }
    return bad ? -1 : 0;
}

/* Backward of every head listed in `heads` (flat b*H + h; NULL = all heads).
 * Gradients of unlisted heads are left untouched. */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dO,
                    int B, int H, int N, int d, double scale, int causal,
                    const uint8_t *block_mask, int block, const int32_t *kv_len,
                    const int32_t *heads, int nheads,
                    double *dq, double *dk, double *dv)
{
    size_t NN = (size_t)N * (size_t)N;
    double *A = (double *)malloc(sizeof(double) * NN);
    double *dS = (double *)malloc(sizeof(double) * NN);
    if (!A || !dS) { free(A); free(dS); return -1; }
    int count = heads ? nheads : B * H;
    for (int t = 0; t < count; ++t) {
        int bh = heads ? heads[t] : t;
        int b = bh / H;
        if (bh < 0 || b >= B) { free(A); free(dS); return -2; }
        mask_t m = make_mask(N, causal, block_mask, block, kv_len, b);
        size_t off = (size_t)bh * (size_t)N * d;
        const double *qh = q + off, *kh = k + off, *vh = v + off, *dOh = dO + off;
        double *dqh = dq + off, *dkh = dk + off, *dvh = dv + off;

        /* A = softmax(S) row by row; dA_ij = dO_i . v_j;
           dS_ij = A_ij (dA_ij - sum_k A_ik dA_ik). */
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < N; ++i) {
            double *Ai = A + (size_t)i * N;
            double *dSi = dS + (size_t)i * N;
            logits_row(qh + (size_t)i * d, kh, N, d, scale, &m, i, Ai);
            softmax_row(Ai, N);
            const double *dOi = dOh + (size_t)i * d;
            for (int j = 0; j < N; ++j) {
                double dot = 0.0;
                const double *vj = vh + (size_t)j * d;
                for (int c = 0; c < d; ++c) dot += dOi[c] * vj[c];
                dSi[j] = dot;                      /* dA_ij for now */
            }
            double delta = 0.0;
            for (int j = 0; j < N; ++j) delta += Ai[j] * dSi[j];
            for (int j = 0; j < N; ++j) dSi[j] = Ai[j] * (dSi[j] - delta);
        }
        /* dQ_i = scale * sum_j dS_ij k_j */
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < N; ++i) {
            double *out = dqh + (size_t)i * d;
            for (int c = 0; c < d; ++c) out[c] = 0.0;
            const double *dSi = dS + (size_t)i * N;
            for (int j = 0; j < N; ++j) {
                double w = dSi[j];
                if (w == 0.0) continue;
                const double *kj = kh + (size_t)j * d;
                for (int c = 0; c < d; ++c) out[c] += w * kj[c];
            }
            for (int c = 0; c < d; ++c) out[c] *= scale;
        }
        /* dK_j = scale * sum_i dS_ij q_i ;  dV_j = sum_i A_ij dO_i */
        #pragma omp parallel for schedule(static)
        for (int j = 0; j < N; ++j) {
            double *gk = dkh + (size_t)j * d;
            double *gv = dvh + (size_t)j * d;
            for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
            for (int i = 0; i < N; ++i) {
                double ws = dS[(size_t)i * N + j];
                double wa = A[(size_t)i * N + j];
                if (ws != 0.0) {
                    const double *qi = qh + (size_t)i * d;
                    for (int c = 0; c < d; ++c) gk[c] += ws * qi[c];
                }
                if (wa != 0.0) {
                    const double *dOi = dOh + (size_t)i * d;
                    for (int c = 0; c < d; ++c) gv[c] += wa * dOi[c];
                }
            }
            for (int c = 0; c < d; ++c) gk[c] *= scale;
        }
    }
    free(A);
    free(dS);
    return 0;
}

/* dQ of selected query rows only (flat index (b*H + h)*N + i): the backward's definition
 * restricted to those rows -- dQ_i needs only row i of A and of dA. */
int oracle_attn_bwd_dq_rows(const double *q, const double *k, const double *v, const double *dO,
                            int B, int H, int N, int d, double scale, int causal,
                            const uint8_t *block_mask, int block, const int32_t *kv_len,
                            const int64_t *rows, int nrows, double *dq_rows)
{
    int bad = 0;
    #pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)N);
        double *ds = (double *)malloc(sizeof(double) * (size_t)N);
        #pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            int64_t flat = rows[r];
            int64_t bh = flat / N;
            int i = (int)(flat % N);
            int b = (int)(bh / H);
            if (flat < 0 || b >= B) { bad = 1; continue; }
            mask_t m = make_mask(N, causal, block_mask, block, kv_len, b);
            size_t off = (size_t)bh * (size_t)N * d;
            const double *kh = k + off, *vh = v + off, *dOi = dO + off + (size_t)i * d;
            logits_row(q + off + (size_t)i * d, kh, N, d, scale, &m, i, a);
            softmax_row(a, N);
            double delta = 0.0;
            for (int j = 0; j < N; ++j) {
                double dot = 0.0;
                const double *vj = vh + (size_t)j * d;
                for (int c = 0; c < d; ++c) dot += dOi[c] * vj[c];
                ds[j] = dot;                               /* dA_ij */
                delta += a[j] * dot;
            }
            double *out = dq_rows + (size_t)r * d;
            for (int c = 0; c < d; ++c) out[c] = 0.0;
            for (int j = 0; j < N; ++j) {
                double w = a[j] * (ds[j] - delta);        /* dS_ij */
                if (w == 0.0) continue;
                const double *kj = kh + (size_t)j * d;
                for (int c = 0; c < d; ++c) out[c] += w * kj[c];
            }
            for (int c = 0; c < d; ++c) out[c] *= scale;
        }
        free(a);
        free(ds);
    }
    return bad ? -1 : 0;
}

/* dK and dV of selected key rows only (flat index (b*H + h)*N + j).  dK_j and dV_j are sums
 * over the query rows i of column j of dS and of A:
 *     dV_j = sum_i A_ij dO_i,    dK_j = scale * sum_i dS_ij q_i,
 *     dS_ij = A_ij (dA_ij - sum_k A_ik dA_ik),   dA_ij = dO_i . v_j,
 * and each A_ij, dS_ij needs the whole of row i (its normaliser and its sum over k).  So every
 * row i that may attend to at least one selected key of its head is materialised in full (S,
 * A and dA), exactly as in oracle_attn_bwd, and the entries of the selected columns are kept;
 * the sums over i then run in index order.  Keys of heads with no selected key cost nothing. */
int oracle_attn_bwd_kv_rows(const double *q, const double *k, const double *v, const double *dO,
                            int B, int H, int N, int d, double scale, int causal,
                            const uint8_t *block_mask, int block, const int32_t *kv_len,
                            const int64_t *rows, int nrows, double *dk_rows, double *dv_rows)
{
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] / N / H >= B) return -1;
    /* column buffers: for selected key r, colA[r*N + i] = A_ij and colS[r*N + i] = dS_ij */
    double *colA = (double *)calloc((size_t)nrows * (size_t)N, sizeof(double));
    double *colS = (double *)calloc((size_t)nrows * (size_t)N, sizeof(double));
    if ((!colA || !colS) && nrows > 0) { free(colA); free(colS); return -2; }
    for (int bh = 0; bh < B * H; ++bh) {
        /* the selected keys of this head */
        int nsel = 0;
        for (int r = 0; r < nrows; ++r) if (rows[r] / N == bh) ++nsel;
        if (nsel == 0) continue;
        int *sel = (int *)malloc(sizeof(int) * (size_t)nsel);
        nsel = 0;
        for (int r = 0; r < nrows; ++r) if (rows[r] / N == bh) sel[nsel++] = r;
        int b = bh / H;
        mask_t m = make_mask(N, causal, block_mask, block, kv_len, b);
        size_t off = (size_t)bh * (size_t)N * d;
        const double *qh = q + off, *kh = k + off, *vh = v + off, *dOh = dO + off;
        #pragma omp parallel
        {
            double *a = (double *)malloc(sizeof(double) * (size_t)N);
            double *da = (double *)malloc(sizeof(double) * (size_t)N);
            #pragma omp for schedule(dynamic, 16)
            for (int i = 0; i < N; ++i) {
                int any = 0;
                for (int s = 0; s < nsel; ++s)
                    if (key_allowed(&m, i, (int)(rows[sel[s]] % N))) { any = 1; break; }
                if (!any) continue;               /* A_ij = dS_ij = 0 for every selected j */
                logits_row(qh + (size_t)i * d, kh, N, d, scale, &m, i, a);
                softmax_row(a, N);
                const double *dOi = dOh + (size_t)i * d;
                double delta = 0.0;
                for (int j = 0; j < N; ++j) {
                    double dot = 0.0;
                    const double *vj = vh + (size_t)j * d;
                    for (int c = 0; c < d; ++c) dot += dOi[c] * vj[c];
                    da[j] = dot;                   /* dA_ij */
                    delta += a[j] * dot;
                }
                for (int s = 0; s < nsel; ++s) {
                    int r = sel[s];
                    int j = (int)(rows[r] % N);
                    colA[(size_t)r * N + i] = a[j];
                    colS[(size_t)r * N + i] = a[j] * (da[j] - delta);
                }
            }
            free(a);
            free(da);
        }
        #pragma omp parallel for schedule(static)
        for (int s = 0; s < nsel; ++s) {
            int r = sel[s];
            double *gk = dk_rows + (size_t)r * d, *gv = dv_rows + (size_t)r * d;
            for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
            for (int i = 0; i < N; ++i) {
                double ws = colS[(size_t)r * N + i], wa = colA[(size_t)r * N + i];
                if (ws != 0.0) {
                    const double *qi = qh + (size_t)i * d;
                    for (int c = 0; c < d; ++c) gk[c] += ws * qi[c];
                }
                if (wa != 0.0) {
                    const double *dOi = dOh + (size_t)i * d;
                    for (int c = 0; c < d; ++c) gv[c] += wa * dOi[c];
                }
            }
            for (int c = 0; c < d; ++c) gk[c] *= scale;
        }
        free(sel);
    }
    free(colA);
    free(colS);
    return 0;
}
