/*
 * oracle.h -- fp64 CPU reference for exact softmax attention.
 * TEST INFRASTRUCTURE ONLY: the product library never includes or links this.
 *
 * All arrays are row-major double, one (batch, head) after another:
 * q, k, v, dout, o, dq, dk, dv are [BH][N][d]; lse is [BH][N] (natural log).
 * mask (used when flags has ORACLE_SPARSE) is uint8 [nb][nb], nb = ceil(N/blk),
 * shared by every head: block (i/blk, j/blk) nonzero means "kept".
 * Functions return 0 on success, negative on bad arguments.
 */
#ifndef FA_ORACLE_H
#define FA_ORACLE_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_CAUSAL 1
#define ORACLE_SPARSE 2

/* O and LSE on the query rows listed in rows[nrows]; o is [BH][nrows][d], lse [BH][nrows] */
int oracle_fwd_rows(const double *q, const double *k, const double *v,
                    int BH, int N, int d, double scale, int flags,
                    const uint8_t *mask, int blk, const int *rows, int nrows,
                    double *o, double *lse, int nthreads);

/* one head, the online-softmax recurrence over key tiles of `tile` keys */
int oracle_online_softmax_fwd(const double *q, const double *k, const double *v,
                              int N, int d, double scale, int flags,
                              const uint8_t *mask, int blk, int tile,
                              double *o, double *lse);

/* full forward + backward, materialising the N x N matrices of every head */
int oracle_bwd_full(const double *q, const double *k, const double *v, const double *dout,
                    int BH, int N, int d, double scale, int flags,
                    const uint8_t *mask, int blk,
                    double *o, double *lse, double *dq, double *dk, double *dv, int nthreads);

/* dQ on the listed query rows; dq is [BH][nrows][d] */
int oracle_bwd_dq_rows(const double *q, const double *k, const double *v, const double *dout,
                       int BH, int N, int d, double scale, int flags,
                       const uint8_t *mask, int blk, const int *rows, int nrows,
                       double *dq, int nthreads);

/* dK and dV on the listed keys; dk, dv are [BH][ncols][d] */
int oracle_bwd_dkdv_cols(const double *q, const double *k, const double *v, const double *dout,
                         int BH, int N, int d, double scale, int flags,
                         const uint8_t *mask, int blk, const int *cols, int ncols,
                         double *dk, double *dv, int nthreads);

#ifdef __cplusplus
}
#endif
#endif
