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
#define ORACLE_WINDOW 4   /* sliding window (left, right) */
#define ORACLE_ALIBI 8    /* ALiBi bias -slope_h |i + Nk - Nq - j| */

/*
 * The _ex variants take Nq query rows and Nk keys per head (q, o, dout, dq:
 * [BH][Nq][d]; k, v, dk, dv: [BH][Nk][d]; lse [BH][Nq]), bottom-right aligned
 * (query i meets key i + Nk - Nq on the diagonal), a window (left, right)
 * used with ORACLE_WINDOW (negative = unbounded side), ALiBi slopes [H]
 * used with ORACLE_ALIBI (batch-head bh has head bh % H), and the block mask
 * [ceil(Nq/blk)][ceil(Nk/blk)].  The plain variants are Nq = Nk = N, H = 1.
 */
int oracle_fwd_rows_ex(const double *q, const double *k, const double *v,
                       int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                       const double *slopes, const uint8_t *mask, int blk, const int *rows, int nrows,
                       double *o, double *lse, int nthreads);
int oracle_online_softmax_fwd_ex(const double *q, const double *k, const double *v,
                                 int Nq, int Nk, int d, double scale, int flags, int left, int right,
                                 const double *slope, const uint8_t *mask, int blk, int tile,
                                 double *o, double *lse);
int oracle_bwd_full_ex(const double *q, const double *k, const double *v, const double *dout,
                       int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                       const double *slopes, const uint8_t *mask, int blk,
                       double *o, double *lse, double *dq, double *dk, double *dv, int nthreads);
int oracle_bwd_dq_rows_ex(const double *q, const double *k, const double *v, const double *dout,
                          int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                          const double *slopes, const uint8_t *mask, int blk, const int *rows, int nrows,
                          double *dq, int nthreads);
int oracle_bwd_dkdv_cols_ex(const double *q, const double *k, const double *v, const double *dout,
                            int BH, int H, int Nq, int Nk, int d, double scale, int flags, int left, int right,
                            const double *slopes, const uint8_t *mask, int blk, const int *cols, int ncols,
                            double *dk, double *dv, int nthreads);

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

/*
 * FP8 (E4M3) forward with block quantisation and incoherent processing (the
 * readings are written out above the FP8 section of oracle.c).
 *   oracle_e4m3_value / _round: decode a code; round a value to a code.
 *   oracle_rotate_f32: x [nrows][d] <- (x o signs) H_d / sqrt(d) in float.
 *   oracle_fp8_quantize: x float [BH][N][d] -> codes [BH][N][d] and scales
 *     [BH][ceil(N/rows)] (rows per block), rotating first when signs != NULL.
 *   oracle_fwd_fp8: O [BH][nrows][d], LSE [BH][nrows] on query rows qrows from
 *     the codes and scales (sq, sk [BH][ceil(N/rows)], sv [BH]); quant_p = 0
 *     keeps P unrounded.
 */
double oracle_e4m3_value(int code);
int oracle_e4m3_round(double x);
int oracle_e4m3_round_array(const double *x, long n, uint8_t *codes);
int oracle_rotate_f32(float *x, long nrows, int d, const float *signs);
int oracle_fp8_quantize(const float *x, int BH, int N, int d, int rows, const float *signs,
                        uint8_t *codes, float *scales);
int oracle_fwd_fp8(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8, const float *sq, const float *sk,
                   const float *sv, int BH, int N, int d, int rows, double scale, int causal, int quant_p,
                   const int *qrows, int nrows, double *o, double *lse, int nthreads);

#ifdef __cplusplus
}
#endif
#endif
