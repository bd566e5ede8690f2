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
