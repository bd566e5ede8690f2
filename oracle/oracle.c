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
 *   mask  : S_ij = -inf where key j is not visible to query i.  With N_q
 *           query rows and N_k keys, off = N_k - N_q aligns the last query
 *           with the last key (bottom-right; off = 0 when N_q = N_k):
 *           causal  -> j > i + off is hidden  ("FlashAttention 深度解析"
 *                      section 五: built-in causal mask)
 *           window  -> visible iff i + off - left <= j <= i + off + right
 *                      (深度解析 section 五: built-in sliding-window mask; a
 *                      negative left or right leaves that side unbounded)
 *           sparse  -> block (i/blk, j/blk) of the block mask is 0  (notes
 *                      section 4, block-sparse FlashAttention)
 *   bias  : ALiBi (深度解析 section 五: built-in ALiBi mode) adds
 *           -slope_h * |i + off - j| to S_ij, slope_h the head's slope
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
/* what a head sees: sizes, mask modes, bias                                 */
/* ------------------------------------------------------------------------ */
typedef struct {
    int Nq, Nk;                 /* query rows and keys per head */
    int flags;                  /* ORACLE_CAUSAL | ORACLE_SPARSE | ORACLE_WINDOW | ORACLE_ALIBI */
    int left, right;            /* window sides (ORACLE_WINDOW); negative = unbounded */
    const uint8_t *mask;        /* [ceil(Nq/blk)][ceil(Nk/blk)] (ORACLE_SPARSE) */
    int blk, nbk;               /* block size and key blocks of the mask */
    const double *slopes;       /* [H] ALiBi slopes (ORACLE_ALIBI) */
    int H;                      /* heads: head of batch-head bh is bh % H */
} spec_t;

static spec_t make_spec(int Nq, int Nk, int flags, int left, int right, const uint8_t *mask, int blk,
                        const double *slopes, int H)
{
    spec_t s;
    s.Nq = Nq; s.Nk = Nk; s.flags = flags; s.left = left; s.right = right;
    s.mask = mask; s.blk = blk > 0 ? blk : 1; s.nbk = (Nk + s.blk - 1) / s.blk;
    s.slopes = slopes; s.H = H > 0 ? H : 1;
    return s;
}

/* visibility of key j to query i */
static int visible(const spec_t *sp, int i, int j)
{
    const long off = (long)sp->Nk - sp->Nq;
    if ((sp->flags & ORACLE_CAUSAL) && j > i + off) return 0;
    if (sp->flags & ORACLE_WINDOW) {
        if (sp->left >= 0 && j < i + off - sp->left) return 0;
        if (sp->right >= 0 && j > i + off + sp->right) return 0;
    }
    if ((sp->flags & ORACLE_SPARSE) && !sp->mask[(size_t)(i / sp->blk) * sp->nbk + (j / sp->blk)]) return 0;
    return 1;
}

/* additive score bias of (query i, key j) in head h */
static double bias(const spec_t *sp, long h, int i, int j)
{
    if (!(sp->flags & ORACLE_ALIBI)) return 0.0;
    const double dist = fabs((double)i + ((double)sp->Nk - sp->Nq) - (double)j);
    return -sp->slopes[h % sp->H] * dist;
}

/* one row of S (masked, biased) into srow[Nk] */
static void score_row(const spec_t *sp, long h, const double *q, const double *k, int d, double scale,
                      int i, double *srow)
{
    const double *qi = q + (size_t)i * d;
    for (int j = 0; j < sp->Nk; ++j) {
        if (!visible(sp, i, j)) { srow[j] = -INFINITY; continue; }
        const double *kj = k + (size_t)j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
        srow[j] = scale * acc + bias(sp, h, i, j);
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
    int BH, d;
    spec_t sp;
    double scale;
    const int *rows; int nrows;
    double *o, *lse;
} fwd_ctx;

static void fwd_item(void *vctx, long item, double *srow)
{
    fwd_ctx *c = (fwd_ctx *)vctx;
    const int Nq = c->sp.Nq, Nk = c->sp.Nk, d = c->d;
    long h = item / c->nrows, r = item % c->nrows;
    int i = c->rows[r];
    const double *q = c->q + (size_t)h * Nq * d;
    const double *k = c->k + (size_t)h * Nk * d, *v = c->v + (size_t)h * Nk * d;
    score_row(&c->sp, h, q, k, d, c->scale, i, srow);
    double lse = softmax_row(srow, Nk);
    double *oi = c->o + ((size_t)h * c->nrows + r) * d;
    for (int x = 0; x < d; ++x) oi[x] = 0.0;
    for (int j = 0; j < Nk; ++j) {
        double p = srow[j];
        if (p == 0.0) continue;
        const double *vj = v + (size_t)j * d;
        for (int x = 0; x < d; ++x) oi[x] += p * vj[x];
    }
    c->lse[(size_t)h * c->nrows + r] = lse;
}

int oracle_fwd_rows_ex(const double *q, const double *k, const double *v,
                       int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                       const double *slopes, const uint8_t *mask, int blk, const int *rows, int nrows,
                       double *o, double *lse, int nthreads)
{
    if (BH < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || nrows < 0) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    if ((flags & ORACLE_ALIBI) && !slopes) return -1;
    fwd_ctx c = {q, k, v, BH, d, make_spec(Nq, Nk, flags, left, right, mask, blk, slopes, H), scale,
                 rows, nrows, o, lse};
    parallel_for(fwd_item, &c, (long)BH * nrows, (size_t)Nk, nthreads);
    return 0;
}

int oracle_fwd_rows(const double *q, const double *k, const double *v,
                    int BH, int N, int d, double scale, int flags,
                    const uint8_t *mask, int blk, const int *rows, int nrows,
                    double *o, double *lse, int nthreads)
{
    return oracle_fwd_rows_ex(q, k, v, BH, 1, N, N, d, scale, flags & (ORACLE_CAUSAL | ORACLE_SPARSE), -1, -1,
                              NULL, mask, blk, rows, nrows, o, lse, nthreads);
}

/* ------------------------------------------------------------------------ */
/* online-softmax forward (the recurrence, for pinning against two-pass)     */
/* ------------------------------------------------------------------------ */
int oracle_online_softmax_fwd_ex(const double *q, const double *k, const double *v,
                                 int Nq, int Nk, int d, double scale, int flags, int left, int right,
                                 const double *slope, const uint8_t *mask, int blk, int tile,
                                 double *o, double *lse)
{
    if (Nq < 1 || Nk < 1 || d < 1 || tile < 1) return -1;
    if ((flags & ORACLE_ALIBI) && !slope) return -1;
    const spec_t sp = make_spec(Nq, Nk, flags, left, right, mask, blk, slope, 1);
    double *s = (double *)malloc(sizeof(double) * tile);
    for (int i = 0; i < Nq; ++i) {
        double m = -INFINITY, l = 0.0;
        double *oi = o + (size_t)i * d;
        for (int x = 0; x < d; ++x) oi[x] = 0.0;
        for (int j0 = 0; j0 < Nk; j0 += tile) {
            int jn = (j0 + tile < Nk) ? tile : Nk - j0;
            double bmax = -INFINITY;
            for (int t = 0; t < jn; ++t) {
                int j = j0 + t;
                if (!visible(&sp, i, j)) { s[t] = -INFINITY; continue; }
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += q[(size_t)i * d + c] * k[(size_t)j * d + c];
                s[t] = scale * acc + bias(&sp, 0, i, j);
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

int oracle_online_softmax_fwd(const double *q, const double *k, const double *v,
                              int N, int d, double scale, int flags,
                              const uint8_t *mask, int blk, int tile,
                              double *o, double *lse)
{
    return oracle_online_softmax_fwd_ex(q, k, v, N, N, d, scale, flags & (ORACLE_CAUSAL | ORACLE_SPARSE), -1, -1,
                                        NULL, mask, blk, tile, o, lse);
}

/* ------------------------------------------------------------------------ */
/* full backward of one head, materialising the Nq x Nk matrices             */
/* ------------------------------------------------------------------------ */
typedef struct {
    const double *q, *k, *v, *dout;
    int BH, d;
    spec_t sp;
    double scale;
    double *o, *lse, *dq, *dk, *dv;
} bwd_ctx;

static void bwd_full_item(void *vctx, long h, double *unused)
{
    (void)unused;
    bwd_ctx *c = (bwd_ctx *)vctx;
    const int Nq = c->sp.Nq, Nk = c->sp.Nk, d = c->d;
    const size_t qoff = (size_t)h * Nq * d, koff = (size_t)h * Nk * d;
    const double *q = c->q + qoff, *dout = c->dout + qoff, *k = c->k + koff, *v = c->v + koff;
    double *o = c->o + qoff, *dq = c->dq + qoff, *dk = c->dk + koff, *dv = c->dv + koff;
    double *lse = c->lse + (size_t)h * Nq;

    double *P = (double *)malloc(sizeof(double) * (size_t)Nq * Nk);
    double *dP = (double *)malloc(sizeof(double) * (size_t)Nq * Nk);
    double *D = (double *)malloc(sizeof(double) * (size_t)Nq);

    /* forward: S, P, O, LSE */
    for (int i = 0; i < Nq; ++i) {
        double *pr = P + (size_t)i * Nk;
        score_row(&c->sp, h, q, k, d, c->scale, i, pr);
        lse[i] = softmax_row(pr, Nk);
    }
    for (int i = 0; i < Nq; ++i)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int j = 0; j < Nk; ++j) acc += P[(size_t)i * Nk + j] * v[(size_t)j * d + x];
            o[(size_t)i * d + x] = acc;
        }
    /* dV = P^T dO */
    for (int j = 0; j < Nk; ++j)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int i = 0; i < Nq; ++i) acc += P[(size_t)i * Nk + j] * dout[(size_t)i * d + x];
            dv[(size_t)j * d + x] = acc;
        }
    /* dP = dO V^T */
    for (int i = 0; i < Nq; ++i)
        for (int j = 0; j < Nk; ++j) {
            double acc = 0.0;
            for (int x = 0; x < d; ++x) acc += dout[(size_t)i * d + x] * v[(size_t)j * d + x];
            dP[(size_t)i * Nk + j] = acc;
        }
    /* D_i = sum_c dO_ic O_ic */
    for (int i = 0; i < Nq; ++i) {
        double acc = 0.0;
        for (int x = 0; x < d; ++x) acc += dout[(size_t)i * d + x] * o[(size_t)i * d + x];
        D[i] = acc;
    }
    /* dS = P o (dP - D), stored over dP (the bias is a constant: it enters only through P) */
    for (int i = 0; i < Nq; ++i)
        for (int j = 0; j < Nk; ++j)
            dP[(size_t)i * Nk + j] = P[(size_t)i * Nk + j] * (dP[(size_t)i * Nk + j] - D[i]);
    /* dQ = scale dS K ; dK = scale dS^T Q */
    for (int i = 0; i < Nq; ++i)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int j = 0; j < Nk; ++j) acc += dP[(size_t)i * Nk + j] * k[(size_t)j * d + x];
            dq[(size_t)i * d + x] = c->scale * acc;
        }
    for (int j = 0; j < Nk; ++j)
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int i = 0; i < Nq; ++i) acc += dP[(size_t)i * Nk + j] * q[(size_t)i * d + x];
            dk[(size_t)j * d + x] = c->scale * acc;
        }
    free(P); free(dP); free(D);
}

int oracle_bwd_full_ex(const double *q, const double *k, const double *v, const double *dout,
                       int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                       const double *slopes, const uint8_t *mask, int blk,
                       double *o, double *lse, double *dq, double *dk, double *dv, int nthreads)
{
    if (BH < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    if ((flags & ORACLE_ALIBI) && !slopes) return -1;
    bwd_ctx c = {q, k, v, dout, BH, d, make_spec(Nq, Nk, flags, left, right, mask, blk, slopes, H), scale,
                 o, lse, dq, dk, dv};
    parallel_for(bwd_full_item, &c, BH, 0, nthreads);
    return 0;
}

int oracle_bwd_full(const double *q, const double *k, const double *v, const double *dout,
                    int BH, int N, int d, double scale, int flags,
                    const uint8_t *mask, int blk,
                    double *o, double *lse, double *dq, double *dk, double *dv, int nthreads)
{
    return oracle_bwd_full_ex(q, k, v, dout, BH, 1, N, N, d, scale, flags & (ORACLE_CAUSAL | ORACLE_SPARSE), -1, -1,
                              NULL, mask, blk, o, lse, dq, dk, dv, nthreads);
}

/* ------------------------------------------------------------------------ */
/* sampled backward: dQ on chosen rows, dK/dV on chosen keys                 */
/* ------------------------------------------------------------------------ */

/* per row i: S_i, P_i, O_i, D_i; then dS_i and dQ_i.  scratch holds Nk + d doubles. */
typedef struct {
    const double *q, *k, *v, *dout;
    int BH, d;
    spec_t sp;
    double scale;
    const int *rows; int nrows;
    double *dq;               /* [BH][nrows][d] */
} dq_ctx;

static void dq_item(void *vctx, long item, double *scratch)
{
    dq_ctx *c = (dq_ctx *)vctx;
    const int Nq = c->sp.Nq, Nk = c->sp.Nk, d = c->d;
    long h = item / c->nrows, r = item % c->nrows;
    int i = c->rows[r];
    const double *q = c->q + (size_t)h * Nq * d, *dout = c->dout + (size_t)h * Nq * d;
    const double *k = c->k + (size_t)h * Nk * d, *v = c->v + (size_t)h * Nk * d;
    double *prow = scratch, *oi = scratch + Nk;
    double *dqi = c->dq + ((size_t)h * c->nrows + r) * d;

    score_row(&c->sp, h, q, k, d, c->scale, i, prow);
    softmax_row(prow, Nk);
    for (int x = 0; x < d; ++x) oi[x] = 0.0;
    for (int j = 0; j < Nk; ++j) {
        if (prow[j] == 0.0) continue;
        for (int x = 0; x < d; ++x) oi[x] += prow[j] * v[(size_t)j * d + x];
    }
    double D = 0.0;
    for (int x = 0; x < d; ++x) D += dout[(size_t)i * d + x] * oi[x];
    for (int x = 0; x < d; ++x) dqi[x] = 0.0;
    for (int j = 0; j < Nk; ++j) {
        if (prow[j] == 0.0) continue;
        double dp = 0.0;
        for (int x = 0; x < d; ++x) dp += dout[(size_t)i * d + x] * v[(size_t)j * d + x];
        double ds = prow[j] * (dp - D);
        for (int x = 0; x < d; ++x) dqi[x] += ds * k[(size_t)j * d + x];
    }
    for (int x = 0; x < d; ++x) dqi[x] *= c->scale;
}

int oracle_bwd_dq_rows_ex(const double *q, const double *k, const double *v, const double *dout,
                          int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                          const double *slopes, const uint8_t *mask, int blk, const int *rows, int nrows,
                          double *dq, int nthreads)
{
    if (BH < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || nrows < 0) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    if ((flags & ORACLE_ALIBI) && !slopes) return -1;
    dq_ctx c = {q, k, v, dout, BH, d, make_spec(Nq, Nk, flags, left, right, mask, blk, slopes, H), scale,
                rows, nrows, dq};
    parallel_for(dq_item, &c, (long)BH * nrows, (size_t)Nk + d, nthreads);
    return 0;
}

int oracle_bwd_dq_rows(const double *q, const double *k, const double *v, const double *dout,
                       int BH, int N, int d, double scale, int flags,
                       const uint8_t *mask, int blk, const int *rows, int nrows,
                       double *dq, int nthreads)
{
    return oracle_bwd_dq_rows_ex(q, k, v, dout, BH, 1, N, N, d, scale, flags & (ORACLE_CAUSAL | ORACLE_SPARSE),
                                 -1, -1, NULL, mask, blk, rows, nrows, dq, nthreads);
}

/* stage 1 of dK/dV: LSE_i and D_i for the listed (head, row) items */
typedef struct {
    const double *q, *k, *v, *dout;
    int BH, d;
    spec_t sp;
    double scale;
    const long *items;        /* h * Nq + i */
    double *lse, *D;          /* [BH][Nq] */
} stat_ctx;

static void stat_item(void *vctx, long it, double *scratch)
{
    stat_ctx *c = (stat_ctx *)vctx;
    const int Nq = c->sp.Nq, Nk = c->sp.Nk, d = c->d;
    long code = c->items[it];
    long h = code / Nq;
    int i = (int)(code % Nq);
    const double *q = c->q + (size_t)h * Nq * d, *dout = c->dout + (size_t)h * Nq * d;
    const double *k = c->k + (size_t)h * Nk * d, *v = c->v + (size_t)h * Nk * d;
    double *prow = scratch, *oi = scratch + Nk;
    score_row(&c->sp, h, q, k, d, c->scale, i, prow);
    double lse = softmax_row(prow, Nk);
    for (int x = 0; x < d; ++x) oi[x] = 0.0;
    for (int j = 0; j < Nk; ++j) {
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
    int BH, d;
    spec_t sp;
    double scale;
    const double *lse, *D;
    const int *cols; int ncols;
    double *dk, *dv;          /* [BH][ncols][d] */
} kv_ctx;

static void kv_item(void *vctx, long item, double *unused)
{
    (void)unused;
    kv_ctx *c = (kv_ctx *)vctx;
    const int Nq = c->sp.Nq, Nk = c->sp.Nk, d = c->d;
    long h = item / c->ncols, r = item % c->ncols;
    int j = c->cols[r];
    const double *q = c->q + (size_t)h * Nq * d, *dout = c->dout + (size_t)h * Nq * d;
    const double *k = c->k + (size_t)h * Nk * d, *v = c->v + (size_t)h * Nk * d;
    const double *lse = c->lse + (size_t)h * Nq, *D = c->D + (size_t)h * Nq;
    double *dkj = c->dk + ((size_t)h * c->ncols + r) * d;
    double *dvj = c->dv + ((size_t)h * c->ncols + r) * d;
    for (int x = 0; x < d; ++x) { dkj[x] = 0.0; dvj[x] = 0.0; }
    for (int i = 0; i < Nq; ++i) {
        if (!visible(&c->sp, i, j)) continue;
        if (lse[i] == -INFINITY) continue;
        double s = 0.0, dp = 0.0;
        for (int x = 0; x < d; ++x) {
            s += q[(size_t)i * d + x] * k[(size_t)j * d + x];
            dp += dout[(size_t)i * d + x] * v[(size_t)j * d + x];
        }
        double p = exp(c->scale * s + bias(&c->sp, h, i, j) - lse[i]);   /* P_ij recomputed from LSE_i */
        double ds = p * (dp - D[i]);
        for (int x = 0; x < d; ++x) {
            dvj[x] += p * dout[(size_t)i * d + x];
            dkj[x] += ds * q[(size_t)i * d + x];
        }
    }
    for (int x = 0; x < d; ++x) dkj[x] *= c->scale;
}

int oracle_bwd_dkdv_cols_ex(const double *q, const double *k, const double *v, const double *dout,
                            int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                            const double *slopes, const uint8_t *mask, int blk, const int *cols, int ncols,
                            double *dk, double *dv, int nthreads)
{
    if (BH < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || ncols < 0) return -1;
    if ((flags & ORACLE_SPARSE) && (!mask || blk < 1)) return -1;
    if ((flags & ORACLE_ALIBI) && !slopes) return -1;
    const spec_t sp = make_spec(Nq, Nk, flags, left, right, mask, blk, slopes, H);
    double *lse = (double *)malloc(sizeof(double) * (size_t)BH * Nq);
    double *D = (double *)malloc(sizeof(double) * (size_t)BH * Nq);
    char *need = (char *)calloc((size_t)Nq, 1);
    long *items = (long *)malloc(sizeof(long) * ((size_t)BH * Nq + 1));
    if (!lse || !D || !need || !items) { free(lse); free(D); free(need); free(items); return -2; }
    for (size_t t = 0; t < (size_t)BH * Nq; ++t) { lse[t] = -INFINITY; D[t] = 0.0; }

    /* only rows that see at least one requested key enter dK/dV */
    for (int i = 0; i < Nq; ++i)
        for (int r = 0; r < ncols && !need[i]; ++r)
            if (visible(&sp, i, cols[r])) need[i] = 1;
    long nitems = 0;
    for (long h = 0; h < BH; ++h)
        for (int i = 0; i < Nq; ++i)
            if (need[i]) items[nitems++] = h * Nq + i;

    stat_ctx sc = {q, k, v, dout, BH, d, sp, scale, items, lse, D};
    parallel_for(stat_item, &sc, nitems, (size_t)Nk + d, nthreads);

    kv_ctx kc = {q, k, v, dout, BH, d, sp, scale, lse, D, cols, ncols, dk, dv};
    parallel_for(kv_item, &kc, (long)BH * ncols, 0, nthreads);

    free(lse); free(D); free(need); free(items);
    return 0;
}

int oracle_bwd_dkdv_cols(const double *q, const double *k, const double *v, const double *dout,
                         int BH, int N, int d, double scale, int flags,
                         const uint8_t *mask, int blk, const int *cols, int ncols,
                         double *dk, double *dv, int nthreads)
{
    return oracle_bwd_dkdv_cols_ex(q, k, v, dout, BH, 1, N, N, d, scale, flags & (ORACLE_CAUSAL | ORACLE_SPARSE),
                                   -1, -1, NULL, mask, blk, cols, ncols, dk, dv, nthreads);
}

/* ------------------------------------------------------------------------ */
/* FP8 forward: block quantisation with incoherent processing                */
/* ------------------------------------------------------------------------ */
/*
 * "FlashAttention 深度解析" section 四 says FlashAttention-3 adds FP8 block
 * quantisation, paired with incoherent processing to lower the FP8 error
 * (2.6x below plain FP8).  The page gives no more than that; the readings
 * taken here are:
 *   E4M3   1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no
 *          infinities; exponent 1111 with mantissa 111 is NaN, so the largest
 *          magnitude is 1.75 * 2^8 = 448; exponent 0000 holds m * 2^-9.
 *          Rounding: to the nearest code, ties to the even code, magnitudes
 *          of 448 and above saturate to 448.
 *   incoherent processing
 *          Q and K are multiplied by the same orthogonal matrix
 *          M = diag(signs) H_d / sqrt(d) (H_d the Sylvester Hadamard matrix,
 *          signs +-1), which leaves Q K^T unchanged and spreads an outlier
 *          over all d channels before rounding.  V is not rotated.
 *   block quantisation
 *          one scale per block of `rows` rows of one (batch, head):
 *          scale = amax / 448, code = E4M3(x * (448 / amax)); an all-zero
 *          block gets scale 1.  Q and K use 128-row blocks (the kernel's
 *          tiles, so the scales fold into the score coefficient per tile
 *          pair); V uses one block per head (its scale multiplies P V over
 *          every key block, so it folds into the final normalisation).
 *   attention on the quantised operands
 *          S_ij = scale * sq_(i) * sk_(j) * sum_c q8_ic k8_jc (code values),
 *          P_ij = exp(S_ij - m_i), LSE_i = m_i + ln sum_j P_ij,
 *          P8_ij = E4M3(P_ij) (the P.V product runs on FP8 operands too),
 *          O_i = sv * sum_j P8_ij v8_j / sum_j P8_ij (normalised by the sum
 *          of the rounded P, so that a row with one visible key, or identical
 *          V rows, comes out exact).
 * The quantiser works in float, one IEEE operation at a time in the order
 * written below, so that its codes are a definition the GPU quantiser can
 * meet bit for bit (the rotation's butterflies are fixed: stages h = 1, 2,
 * 4, ..., d/2, pair (c, c + h) -> (a + b, a - b)).
 */
double oracle_e4m3_value(int code)
{
    const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);              /* subnormal: (m / 8) 2^(1 - 7) */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

int oracle_e4m3_round(double x)
{
    if (isnan(x)) return 0x7f;
    const int s = signbit(x) ? 0x80 : 0;
    const double a = fabs(x);
    if (a >= 448.0) return s | 0x7e;
    /* the nearest of the non-negative finite codes (their values increase
       with the code); on a tie the even code (mantissa bit 0 clear) wins */
    int best = 0;
    double bd = a;
    for (int c = 1; c <= 0x7e; ++c) {
        const double dd = fabs(oracle_e4m3_value(c) - a);
        if (dd < bd || (dd == bd && (c & 1) == 0)) {
            best = c;
            bd = dd;
        }
    }
    return s | best;
}

int oracle_e4m3_round_array(const double *x, long n, uint8_t *codes)
{
    if (n < 0) return -1;
    for (long i = 0; i < n; ++i) codes[i] = (uint8_t)oracle_e4m3_round(x[i]);
    return 0;
}

/* one row x[d] <- (x o signs) H_d / sqrt(d), in float (see above) */
static void rotate_row_f32(float *x, int d, const float *signs)
{
    for (int c = 0; c < d; ++c) x[c] = x[c] * signs[c];
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int c = i; c < i + h; ++c) {
                const float a = x[c], b = x[c + h];
                x[c] = a + b;
                x[c + h] = a - b;
            }
    const float r = (float)(1.0 / sqrt((double)d));
    for (int c = 0; c < d; ++c) x[c] = x[c] * r;
}

int oracle_rotate_f32(float *x, long nrows, int d, const float *signs)
{
    if (nrows < 0 || d < 1 || (d & (d - 1)) || !signs) return -1;
    for (long r = 0; r < nrows; ++r) rotate_row_f32(x + r * d, d, signs);
    return 0;
}

int oracle_fp8_quantize(const float *x, int BH, int N, int d, int rows, const float *signs,
                        uint8_t *codes, float *scales)
{
    if (BH < 1 || N < 1 || d < 1 || rows < 1) return -1;
    if (signs && (d & (d - 1))) return -1;
    const int nb = (N + rows - 1) / rows;
    float *t = (float *)malloc(sizeof(float) * (size_t)rows * d);
    if (!t) return -2;
    for (long h = 0; h < BH; ++h)
        for (int b = 0; b < nb; ++b) {
            const int r0 = b * rows, r1 = (r0 + rows < N) ? r0 + rows : N;
            const size_t base = ((size_t)h * N + r0) * d;
            const size_t n = (size_t)(r1 - r0) * d;
            memcpy(t, x + base, n * sizeof(float));
            if (signs)
                for (int r = 0; r < r1 - r0; ++r) rotate_row_f32(t + (size_t)r * d, d, signs);
            float amax = 0.0f;
            for (size_t e = 0; e < n; ++e) amax = fmaxf(amax, fabsf(t[e]));
            const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
            const float inv = amax > 0.0f ? 448.0f / amax : 1.0f;
            scales[h * nb + b] = sc;
            for (size_t e = 0; e < n; ++e) {
                const float y = t[e] * inv;
                codes[base + e] = (uint8_t)oracle_e4m3_round((double)y);
            }
        }
    free(t);
    return 0;
}

typedef struct {
    const uint8_t *q8, *k8, *v8;
    const float *sq, *sk, *sv;
    int N, d, rows, causal, quant_p;
    double scale;
    const int *qrows; int nrows;
    double *o, *lse;
    double val[256];
} fp8_ctx;

static void fp8_item(void *vctx, long item, double *scratch)
{
    fp8_ctx *c = (fp8_ctx *)vctx;
    const int N = c->N, d = c->d, nb = (N + c->rows - 1) / c->rows;
    const long h = item / c->nrows, r = item % c->nrows;
    const int i = c->qrows[r];
    double *s = scratch, *p8 = scratch + N;
    const uint8_t *qi = c->q8 + ((size_t)h * N + i) * d;
    const int nk = c->causal ? i + 1 : N;
    double m = -INFINITY;
    for (int j = 0; j < nk; ++j) {
        const uint8_t *kj = c->k8 + ((size_t)h * N + j) * d;
        double dot = 0.0;
        for (int x = 0; x < d; ++x) dot += c->val[qi[x]] * c->val[kj[x]];
        s[j] = c->scale * (double)c->sq[h * nb + i / c->rows] * (double)c->sk[h * nb + j / c->rows] * dot;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0, l8 = 0.0;
    for (int j = 0; j < nk; ++j) {
        const double pj = exp(s[j] - m);
        l += pj;
        p8[j] = c->quant_p ? oracle_e4m3_value(oracle_e4m3_round(pj)) : pj;
        l8 += p8[j];
    }
    double *oi = c->o + ((size_t)h * c->nrows + r) * d;
    for (int x = 0; x < d; ++x) oi[x] = 0.0;
    for (int j = 0; j < nk; ++j) {
        if (p8[j] == 0.0) continue;
        const uint8_t *vj = c->v8 + ((size_t)h * N + j) * d;
        for (int x = 0; x < d; ++x) oi[x] += p8[j] * c->val[vj[x]];
    }
    const double f = (double)c->sv[h] / l8;
    for (int x = 0; x < d; ++x) oi[x] *= f;
    c->lse[(size_t)h * c->nrows + r] = m + log(l);
}

int oracle_fwd_fp8(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8, const float *sq, const float *sk,
                   const float *sv, int BH, int N, int d, int rows, double scale, int causal, int quant_p,
                   const int *qrows, int nrows, double *o, double *lse, int nthreads)
{
    if (BH < 1 || N < 1 || d < 1 || rows < 1 || nrows < 0) return -1;
    fp8_ctx *c = (fp8_ctx *)malloc(sizeof(fp8_ctx));
    if (!c) return -2;
    *c = (fp8_ctx){q8, k8, v8, sq, sk, sv, N, d, rows, causal, quant_p, scale, qrows, nrows, o, lse, {0}};
    for (int code = 0; code < 256; ++code) c->val[code] = oracle_e4m3_value(code);
    parallel_for(fp8_item, c, (long)BH * nrows, (size_t)2 * N, nthreads);
    free(c);
    return 0;
}
