/*
 * oracle.c -- plain, slow, fp64 CPU reference for exact softmax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  The product path
 * (the CUDA library under flash_fwd_b200/) never links, loads or calls it, and
 * this file includes nothing from there.
 *
 * What it computes (per (batch, head), all arithmetic in double):
 *
 *   S_ij  = scale * sum_c Q_ic K_jc                      (pages: "FlashAttention:
 *           Fast and Memory-Efficient Exact Attention with IO-Awareness" notes,
 *           section 1.1, Attn(Q,K,V) = softmax(QK^T)V; the scale is a caller
 *           argument because that formula omits it)
 *   mask  : S_ij = -inf where key j is not visible to query i
 *           causal  -> j > i is hidden  ("FlashAttention 深度解析" section 五:
 *                      built-in causal mask; N_q = N_k so both alignments agree)
 *           sparse  -> block (i/blk, j/blk) of the block mask is 0  (notes
 *                      section 4, block-sparse FlashAttention)
 *   LSE_i = m_i + ln sum_j exp(S_ij - m_i),  m_i = max_j S_ij
 *           (the per-row statistics the forward keeps: "原理概览" section 3.2
 *            keeps m and l; one natural-log LSE = m + ln l carries both)
 *   P_ij  = exp(S_ij - LSE_i)
 *   O_i   = sum_j P_ij V_j
 *
 * Backward with upstream gradient dO (the five matrix products of
 * "深度解析" section 四; recomputation of P per "原理概览" section 3.2):
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
 *   dS = P o (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
 *
 * A row with no visible key gets O = 0, LSE = -inf and zero gradients (the
 * pages do not define it; this is the convention taken).
 *
 * Every routine materialises S and P explicitly (a whole row, or the whole
 * N x N matrix for the full backward) and uses no tiling, no fusion and no
 * reordering beyond the formulas above.  The one exception is
 * oracle_online_softmax_fwd, which is the online-softmax recurrence of
 * "深度解析" section 二 written out on purpose so that a test can pin it
 * against the two-pass definition.
 *
 * Threads: pthreads over independent work items (a (head, row) or a
 * (head, key)); each item is computed exactly as above.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------------------ */
/* visibility of key j to query i                                           */
/* ------------------------------------------------------------------------ */
static int visible(int i, int j, int flags, const uint8_t *mask, int nbk, int blk)
{
    if ((flags & ORACLE_CAUSAL) && j > i) return 0;
    if ((flags & ORACLE_SPARSE) && !mask[(size_t)(i / blk) * nbk + (j / blk)]) return 0;
    return 1;
}

/* one row of S (masked) into srow[N] */
static void score_row(const double *q, const double *k, int N, int d, double scale,
                      int flags, const uint8_t *mask, int nbk, int blk, int i, double *srow)
{
    const double *qi = q + (size_t)i * d;
    for (int j = 0; j < N; ++j) {
        if (!visible(i, j, flags, mask, nbk, blk)) { srow[j] = -INFINITY; continue; }
        const double *kj = k + (size_t)j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
        srow[j] = scale * acc;
    }
}

/* turns a score row into probabilities in place; returns LSE (natural log) */
static double softmax_row(double *srow, int N)
{
    double m = -INFINITY;
    for (int j = 0; j < N; ++j) if (srow[j] > m) m = srow[j];
    if (m == -INFINITY) {                      /* no visible key */
        for (int j = 0; j < N; ++j) srow[j] = 0.0;
        return -INFINITY;
    }
    double l = 0.0;
    for (int j = 0; j < N; ++j) l += exp(srow[j] - m);
    double lse = m + log(l);
    for (int j = 0; j < N; ++j) srow[j] = exp(srow[j] - lse);   /* exp(-inf) = 0 */
    return lse;
}

/* ------------------------------------------------------------------------ */
/* a tiny parallel-for                                                       */
/* ------------------------------------------------------------------------ */
typedef void (*item_fn)(void *ctx, long item, double *scratch);

typedef struct {
    item_fn fn;
    void *ctx;
    long nitems;
    long next;
    size_t scratch_len;
    pthread_mutex_t lock;
} pfor_t;

static void *pfor_worker(void *arg)
{
    pfor_t *p = (pfor_t *)arg;
    double *scratch = (double *)malloc(sizeof(double) * (p->scratch_len ? p->scratch_len : 1));
    for (;;) {
        pthread_mutex_lock(&p->lock);
        long it = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (it >= p->nitems) break;
        p->fn(p->ctx, it, scratch);
    }
    free(scratch);
    return NULL;
}

static void parallel_for(item_fn fn, void *ctx, long nitems, size_t scratch_len, int nthreads)
{
    pfor_t p;
    p.fn = fn; p.ctx = ctx; p.nitems = nitems; p.next = 0; p.scratch_len = scratch_len;
    pthread_mutex_init(&p.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads == 1 || nitems <= 1) {
        pfor_worker(&p);
    } else {
        pthread_t th[256];
        for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, pfor_worker, &p);
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    }
    pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------------------ */
/* forward on a subset of query rows                                         */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *q, *k, *v;
    int BH, N, d, flags, nbk, blk;
    double scale;
    const uint8_t *mask;
    const int *rows; int nrows;
    double *o, *lse;
} fwd_ctx;

static void fwd_item(void *vctx, long item, double *srow)
{
    fwd_ctx *c = (fwd_ctx *)vctx;
    long h = item / c->nrows, r = item % c->nrows;
    int i = c->rows[r];
    size_t hoff = (size_t)h * c->N * c->d;
    const double *q = c->q + hoff, *k = c->k + hoff, *v = c->v + hoff;
    score_row(q, k, c->N, c->d, c->scale, c->flags, c->mask, c->nbk, c->blk, i, srow);
    double lse = softmax_row(srow, c->N);
    double *oi = c->o + ((size_t)h * c->nrows + r) * c->d;
    for (int x = 0; x < c->d; ++x) oi[x] = 0.0;
    for (int j = 0; j < c->N; ++j) {
        double p = srow[j];
        if (p == 0.0) continue;
        const double *vj = v + (size_t)j * c->d;
        for (int x = 0; x < c->d; ++x) oi[x] += p * vj[x];
    }
    c->lse[(size_t)h * c->nrows + r] = lse;
}

int oracle_fwd_rows(const double *q, const double *k, const double *v,
                    int BH, int N, int d, double scale, int flags,
                    const uint8_t *mask, int blk, const int *rows, int nrows,
                    double *o, double *lse, int nthreads)
{
    if (BH < 1 || N < 1 || d < 1 || nrows < 0) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    fwd_ctx c = {q, k, v, BH, N, d, flags, blk > 0 ? (N + blk - 1) / blk : 0, blk > 0 ? blk : 1,
                 scale, mask, rows, nrows, o, lse};
    parallel_for(fwd_item, &c, (long)BH * nrows, (size_t)N, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* online-softmax forward (the recurrence, for pinning against two-pass)     */
/* ------------------------------------------------------------------------ */
int oracle_online_softmax_fwd(const double *q, const double *k, const double *v,
                              int N, int d, double scale, int flags,
                              const uint8_t *mask, int blk, int tile,
                              double *o, double *lse)
{
    if (N < 1 || d < 1 || tile < 1) return -1;
    int nbk = blk > 0 ? (N + blk - 1) / blk : 0;
    double *s = (double *)malloc(sizeof(double) * tile);
    for (int i = 0; i < N; ++i) {
        double m = -INFINITY, l = 0.0;
        double *oi = o + (size_t)i * d;
        for (int x = 0; x < d; ++x) oi[x] = 0.0;
        for (int j0 = 0; j0 < N; j0 += tile) {
            int jn = (j0 + tile < N) ? tile : N - j0;
            double bmax = -INFINITY;
            for (int t = 0; t < jn; ++t) {
                int j = j0 + t;
                if (!visible(i, j, flags, mask, nbk, blk > 0 ? blk : 1)) { s[t] = -INFINITY; continue; }
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += q[(size_t)i * d + c] * k[(size_t)j * d + c];
                s[t] = scale * acc;
                if (s[t] > bmax) bmax = s[t];
            }
            double m_new = m > bmax ? m : bmax;
            if (m_new == -INFINITY) continue;            /* nothing visible yet */
            double corr = exp(m - m_new);                /* exp(-inf) = 0 on the first block */
            l *= corr;
            for (int x = 0; x < d; ++x) oi[x] *= corr;
            for (int t = 0; t < jn; ++t) {
                double p = exp(s[t] - m_new);
                l += p;
                if (p == 0.0) continue;
                const double *vj = v + (size_t)(j0 + t) * d;
                for (int x = 0; x < d; ++x) oi[x] += p * vj[x];
            }
            m = m_new;
        }
        if (l > 0.0) {
            for (int x = 0; x < d; ++x) oi[x] /= l;     /* one division at the end */
            lse[i] = m + log(l);
        } else {
            lse[i] = -INFINITY;
        }
    }
    free(s);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* full backward of one head, materialising the N x N matrices               */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *q, *k, *v, *dout;
    int BH, N, d, flags, nbk, blk;
    double scale;
    const uint8_t *mask;
    double *o, *lse, *dq, *dk, *dv;
} bwd_ctx;

static void bwd_full_item(void *vctx, long h, double *unused)
{
    (void)unused;
    bwd_ctx *c = (bwd_ctx *)vctx;
    int N = c->N, d = c->d;
    size_t hoff = (size_t)h * N * d;
    const double *q = c->q + hoff, *k = c->k + hoff, *v = c->v + hoff, *dout = c->dout + hoff;
    double *o = c->o + hoff, *dq = c->dq + hoff, *dk = c->dk + hoff, *dv = c->dv + hoff;
    double *lse = c->lse + (size_t)h * N;

    double *P = (double *)malloc(sizeof(double) * (size_t)N * N);
    double *dP = (double *)malloc(sizeof(double) * (size_t)N * N);
    double *D = (double *)malloc(sizeof(double) * (size_t)N);

    /* forward: S, P, O, LSE */
    for (int i = 0; i < N; ++i) {
        double *pr = P + (size_t)i * N;
        score_row(q, k, N, d, c->scale, c->flags, c->mask, c->nbk, c->blk, i, pr);
        lse[i] = softmax_row(pr, N);
    }
    for (int i = 0; i < N; ++i)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int j = 0; j < N; ++j) acc += P[(size_t)i * N + j] * v[(size_t)j * d + x];
            o[(size_t)i * d + x] = acc;
        }
    /* dV = P^T dO */
    for (int j = 0; j < N; ++j)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int i = 0; i < N; ++i) acc += P[(size_t)i * N + j] * dout[(size_t)i * d + x];
            dv[(size_t)j * d + x] = acc;
        }
    /* dP = dO V^T */
    for (int i = 0; i < N; ++i)
        for (int j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int x = 0; x < d; ++x) acc += dout[(size_t)i * d + x] * v[(size_t)j * d + x];
            dP[(size_t)i * N + j] = acc;
        }
    /* D_i = sum_c dO_ic O_ic */
    for (int i = 0; i < N; ++i) {
        double acc = 0.0;
        for (int x = 0; x < d; ++x) acc += dout[(size_t)i * d + x] * o[(size_t)i * d + x];
        D[i] = acc;
    }
    /* dS = P o (dP - D), stored over dP */
    for (int i = 0; i < N; ++i)
        for (int j = 0; j < N; ++j)
            dP[(size_t)i * N + j] = P[(size_t)i * N + j] * (dP[(size_t)i * N + j] - D[i]);
    /* dQ = scale dS K ; dK = scale dS^T Q */
    for (int i = 0; i < N; ++i)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int j = 0; j < N; ++j) acc += dP[(size_t)i * N + j] * k[(size_t)j * d + x];
            dq[(size_t)i * d + x] = c->scale * acc;
        }
    for (int j = 0; j < N; ++j)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int i = 0; i < N; ++i) acc += dP[(size_t)i * N + j] * q[(size_t)i * d + x];
            dk[(size_t)j * d + x] = c->scale * acc;
        }
    free(P); free(dP); free(D);
}

int oracle_bwd_full(const double *q, const double *k, const double *v, const double *dout,
                    int BH, int N, int d, double scale, int flags,
                    const uint8_t *mask, int blk,
                    double *o, double *lse, double *dq, double *dk, double *dv, int nthreads)
{
    if (BH < 1 || N < 1 || d < 1) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    bwd_ctx c = {q, k, v, dout, BH, N, d, flags, blk > 0 ? (N + blk - 1) / blk : 0,
                 blk > 0 ? blk : 1, scale, mask, o, lse, dq, dk, dv};
    parallel_for(bwd_full_item, &c, BH, 0, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* sampled backward: dQ on chosen rows, dK/dV on chosen keys                 */
/* ------------------------------------------------------------------------ */

/* per row i: S_i, P_i, O_i, D_i; then dS_i and dQ_i.  srow holds 2N doubles. */
typedef struct {
    const double *q, *k, *v, *dout;
    int BH, N, d, flags, nbk, blk;
    double scale;
    const uint8_t *mask;
    const int *rows; int nrows;
    double *dq;               /* [BH][nrows][d] */
} dq_ctx;

static void dq_item(void *vctx, long item, double *scratch)
{
    dq_ctx *c = (dq_ctx *)vctx;
    long h = item / c->nrows, r = item % c->nrows;
    int i = c->rows[r], N = c->N, d = c->d;
    size_t hoff = (size_t)h * N * d;
    const double *q = c->q + hoff, *k = c->k + hoff, *v = c->v + hoff, *dout = c->dout + hoff;
    double *prow = scratch, *oi = scratch + N;
    double *dqi = c->dq + ((size_t)h * c->nrows + r) * d;

    score_row(q, k, N, d, c->scale, c->flags, c->mask, c->nbk, c->blk, i, prow);
    softmax_row(prow, N);
    for (int x = 0; x < d; ++x) oi[x] = 0.0;
    for (int j = 0; j < N; ++j) {
        if (prow[j] == 0.0) continue;
        for (int x = 0; x < d; ++x) oi[x] += prow[j] * v[(size_t)j * d + x];
    }
    double D = 0.0;
    for (int x = 0; x < d; ++x) D += dout[(size_t)i * d + x] * oi[x];
    for (int x = 0; x < d; ++x) dqi[x] = 0.0;
    for (int j = 0; j < N; ++j) {
        if (prow[j] == 0.0) continue;
        double dp = 0.0;
        for (int x = 0; x < d; ++x) dp += dout[(size_t)i * d + x] * v[(size_t)j * d + x];
        double ds = prow[j] * (dp - D);
        for (int x = 0; x < d; ++x) dqi[x] += ds * k[(size_t)j * d + x];
    }
    for (int x = 0; x < d; ++x) dqi[x] *= c->scale;
}

int oracle_bwd_dq_rows(const double *q, const double *k, const double *v, const double *dout,
                       int BH, int N, int d, double scale, int flags,
                       const uint8_t *mask, int blk, const int *rows, int nrows,
                       double *dq, int nthreads)
{
    if (BH < 1 || N < 1 || d < 1 || nrows < 0) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    dq_ctx c = {q, k, v, dout, BH, N, d, flags, blk > 0 ? (N + blk - 1) / blk : 0,
                blk > 0 ? blk : 1, scale, mask, rows, nrows, dq};
    parallel_for(dq_item, &c, (long)BH * nrows, (size_t)N + d, nthreads);
    return 0;
}

/* stage 1 of dK/dV: LSE_i and D_i for the listed (head, row) items */
typedef struct {
    const double *q, *k, *v, *dout;
    int BH, N, d, flags, nbk, blk;
    double scale;
    const uint8_t *mask;
    const long *items;        /* h * N + i */
    double *lse, *D;          /* [BH][N] */
} stat_ctx;

static void stat_item(void *vctx, long it, double *scratch)
{
    stat_ctx *c = (stat_ctx *)vctx;
    long code = c->items[it];
    long h = code / c->N;
    int i = (int)(code % c->N), N = c->N, d = c->d;
    size_t hoff = (size_t)h * N * d;
    const double *q = c->q + hoff, *k = c->k + hoff, *v = c->v + hoff, *dout = c->dout + hoff;
    double *prow = scratch, *oi = scratch + N;
    score_row(q, k, N, d, c->scale, c->flags, c->mask, c->nbk, c->blk, i, prow);
    double lse = softmax_row(prow, N);
    for (int x = 0; x < d; ++x) oi[x] = 0.0;
    for (int j = 0; j < N; ++j) {
        if (prow[j] == 0.0) continue;
        for (int x = 0; x < d; ++x) oi[x] += prow[j] * v[(size_t)j * d + x];
    }
    double D = 0.0;
    for (int x = 0; x < d; ++x) D += dout[(size_t)i * d + x] * oi[x];
    c->lse[code] = lse;
    c->D[code] = D;
}

/* stage 2: for key j, dV_j = sum_i P_ij dO_i and dK_j = scale sum_i dS_ij Q_i */
typedef struct {
    const double *q, *k, *v, *dout;
    int BH, N, d, flags, nbk, blk;
    double scale;
    const uint8_t *mask;
    const double *lse, *D;
    const int *cols; int ncols;
    double *dk, *dv;          /* [BH][ncols][d] */
} kv_ctx;

static void kv_item(void *vctx, long item, double *unused)
{
    (void)unused;
    kv_ctx *c = (kv_ctx *)vctx;
    long h = item / c->ncols, r = item % c->ncols;
    int j = c->cols[r], N = c->N, d = c->d;
    size_t hoff = (size_t)h * N * d;
    const double *q = c->q + hoff, *k = c->k + hoff, *v = c->v + hoff, *dout = c->dout + hoff;
    const double *lse = c->lse + (size_t)h * N, *D = c->D + (size_t)h * N;
    double *dkj = c->dk + ((size_t)h * c->ncols + r) * d;
    double *dvj = c->dv + ((size_t)h * c->ncols + r) * d;
    for (int x = 0; x < d; ++x) { dkj[x] = 0.0; dvj[x] = 0.0; }
    for (int i = 0; i < N; ++i) {
        if (!visible(i, j, c->flags, c->mask, c->nbk, c->blk)) continue;
        if (lse[i] == -INFINITY) continue;
        double s = 0.0, dp = 0.0;
        for (int x = 0; x < d; ++x) {
            s += q[(size_t)i * d + x] * k[(size_t)j * d + x];
            dp += dout[(size_t)i * d + x] * v[(size_t)j * d + x];
        }
        double p = exp(c->scale * s - lse[i]);        /* P_ij recomputed from LSE_i */
        double ds = p * (dp - D[i]);
        for (int x = 0; x < d; ++x) {
            dvj[x] += p * dout[(size_t)i * d + x];
            dkj[x] += ds * q[(size_t)i * d + x];
        }
    }
    for (int x = 0; x < d; ++x) dkj[x] *= c->scale;
}

int oracle_bwd_dkdv_cols(const double *q, const double *k, const double *v, const double *dout,
                         int BH, int N, int d, double scale, int flags,
                         const uint8_t *mask, int blk, const int *cols, int ncols,
                         double *dk, double *dv, int nthreads)
{
    if (BH < 1 || N < 1 || d < 1 || ncols < 0) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    int nbk = blk > 0 ? (N + blk - 1) / blk : 0;
    if (blk < 1) blk = 1;
    double *lse = (double *)malloc(sizeof(double) * (size_t)BH * N);
    double *D = (double *)malloc(sizeof(double) * (size_t)BH * N);
    char *need = (char *)calloc((size_t)N, 1);
    long *items = (long *)malloc(sizeof(long) * ((size_t)BH * N + 1));
    if (!lse || !D || !need || !items) { free(lse); free(D); free(need); free(items); return -2; }
    for (size_t t = 0; t < (size_t)BH * N; ++t) { lse[t] = -INFINITY; D[t] = 0.0; }

    /* only rows that see at least one requested key enter dK/dV */
    for (int i = 0; i < N; ++i)
        for (int r = 0; r < ncols && !need[i]; ++r)
            if (visible(i, cols[r], flags, mask, nbk, blk)) need[i] = 1;
    long nitems = 0;
    for (long h = 0; h < BH; ++h)
        for (int i = 0; i < N; ++i)
            if (need[i]) items[nitems++] = h * N + i;

    stat_ctx sc = {q, k, v, dout, BH, N, d, flags, nbk, blk, scale, mask, items, lse, D};
    parallel_for(stat_item, &sc, nitems, (size_t)N + d, nthreads);

    kv_ctx kc = {q, k, v, dout, BH, N, d, flags, nbk, blk, scale, mask, lse, D, cols, ncols, dk, dv};
    parallel_for(kv_item, &kc, (long)BH * ncols, 0, nthreads);

    free(lse); free(D); free(need); free(items);
    return 0;
}
