/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library libfa_b200.so.
 *
 * Computes exact softmax attention O = softmax(scale * Q K^T [+ mask]) V
 * ("FlashAttention: Fast and Memory-Efficient Exact Attention with
 * IO-Awareness" notes, section 1.1) with the tiled online softmax of
 * "FlashAttention 深度解析" section 二, so the N x N score and probability
 * matrices never reach device memory ("FlashAttention原理概览" section 3.1).
 * The forward saves one fp32 log-sum-exp per query row; the backward
 * recomputes P from it ("原理概览" section 3.2; notes section 2.5).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout     q, k, v, o, dout, dq, dk, dv are contiguous [B][H][N][d] arrays
 *            of 16-bit floats (d innermost); lse is contiguous fp32 [B][H][N].
 *            All are DEVICE pointers on the current CUDA device.
 * dtype      FA_F16 or FA_BF16, the element type of every 16-bit array.
 *            Products accumulate in fp32; P is rounded to dtype before P.V
 *            and outputs are rounded to nearest even.
 * d          64, 128 or 256 (the head-dimension limit of "深度解析" section
 *            五; a multiple of 16 per "原理概览" section 3.4).
 * N          any N >= 1; a ragged last tile is masked.  N is both the query
 *            and the key length.
 * scale      the softmax scale, supplied by the caller (usually 1/sqrt(d));
 *            it must be positive and finite, else FA_ERR_INVALID_ARG.
 * causal     nonzero: query i sees key j only when j <= i ("深度解析" 五).
 * stream     a cudaStream_t passed as void*; NULL means the legacy default
 *            stream.  Every call is asynchronous on it.
 * Ownership  the caller allocates and frees every buffer; the library
 *            allocates no device memory.  Inputs are only read; outputs are
 *            completely overwritten.  Buffers must not overlap.
 * Alignment  every pointer must be 16-byte aligned, else FA_ERR_MISALIGNED.
 * Errors     a non-zero fa_status; nothing is launched when the arguments
 *            are rejected.  A failed launch returns FA_ERR_CUDA.  Kernels
 *            bound every wait; one that gives up records FA_ERR_TIMEOUT in a
 *            device word that fa_last_device_status() returns after the
 *            caller has synchronised.
 * Rows with no visible key (possible only with a hand-made block mask whose
 * whole block row is zero) get O = 0, LSE = -inf and zero gradients.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

typedef enum { FA_F16 = 0, FA_BF16 = 1 } fa_dtype;

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad flag, scale not positive and finite */
    FA_ERR_UNSUPPORTED = 2,  /* d not in {64, 128, 256}, or a size beyond the kernel limits */
    FA_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
    FA_ERR_WORKSPACE = 4,    /* workspace missing or smaller than fa_bwd_workspace_bytes() */
    FA_ERR_CUDA = 5,         /* a CUDA runtime/driver call or a launch failed */
    FA_ERR_TIMEOUT = 6,      /* a kernel gave up waiting (see fa_last_device_status) */
    FA_ERR_SCRATCH_LIMIT = 7 /* fa_bwd_noalloc: the problem needs more than its built-in scratch */
} fa_status;

/* Side length of one block-mask block, in rows and keys. */
#define FA_BLOCK 128

/*
 * Forward pass.  Writes o [B][H][N][d] and lse [B][H][N] with
 * lse_i = ln sum_j exp(scale * q_i . k_j) over the keys visible to row i
 * (the row statistics m and l of "原理概览" section 3.2 folded into one
 * natural-log value).
 */
FA_API int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int H, int N, int d, float scale, int causal, int dtype,
                  void *stream);

/*
 * Block-sparse forward ("FlashAttention" notes, section 4): block_mask is a
 * DEVICE uint8 array [nb][nb], nb = ceil(N / FA_BLOCK), row-major, shared by
 * every (batch, head).  Query block r attends to key block c only when
 * block_mask[r * nb + c] != 0; skipped blocks are never loaded or computed.
 * causal may be combined with the mask (diagonal blocks then get the
 * element-wise causal mask as well).
 */
FA_API int fa_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse,
                              const uint8_t *block_mask,
                              int B, int H, int N, int d, float scale, int causal, int dtype,
                              void *stream);

/*
 * General forward: query and key lengths may differ, and the built-in mask
 * modes other than causal ("深度解析" section 五: causal, sliding window,
 * ALiBi) are available.
 *   q, o      [B][H][Nq][d];  k, v [B][H][Nk][d];  lse [B][H][Nq]
 *   alignment bottom-right: query i meets key i + (Nk - Nq) on the diagonal
 *             (the same as top-left when Nq == Nk)
 *   causal    key j visible to query i only if j <= i + Nk - Nq
 *   window    key j visible only if i + Nk - Nq - window_left <= j <=
 *             i + Nk - Nq + window_right; a negative side is unbounded
 *             (window_left = window_right = -1: no window); combined with
 *             causal the right side is 0
 *   alibi_slopes  DEVICE float [H] (4-byte aligned) or NULL: adds
 *             -alibi_slopes[h] * |i + Nk - Nq - j| to the scaled score
 *             scale * q_i . k_j of head h (every batch shares the slopes)
 *   block_mask    DEVICE uint8 [ceil(Nq/FA_BLOCK)][ceil(Nk/FA_BLOCK)] or NULL
 * A query row that sees no key gets O = 0 and LSE = -inf (rows 0 .. Nq-Nk-1
 * under causal when Nq > Nk, for instance).  Nq, Nk <= 2^28.
 */
FA_API int fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int H, int Nq, int Nk, int d, float scale, int causal,
                     int window_left, int window_right, const float *alibi_slopes,
                     const uint8_t *block_mask, int dtype, void *stream);

/*
 * Bytes of device workspace fa_bwd needs: two fp32 per-row statistics
 * (LSE * log2 e and D = rowsum(dO * O)), each [B][H][Npad] with N padded up
 * to a multiple of FA_BLOCK, then an fp32 dQ accumulator [B][H][N][d].
 * Returns 0 for invalid sizes.
 */
FA_API size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass ("深度解析" section 四: five matrix products; P recomputed
 * from lse per "原理概览" section 3.2).  Reads q, k, v, o, dout and the lse
 * written by fa_fwd with the same arguments; writes dq, dk, dv.  workspace is
 * a caller-owned DEVICE buffer of at least fa_bwd_workspace_bytes() bytes,
 * 16-byte aligned; its contents on entry do not matter and on exit are
 * unspecified.  dq is accumulated with fp32 atomics, so its low bits may
 * differ from run to run; dk and dv are deterministic.
 */
FA_API int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                  const float *lse, void *dq, void *dk, void *dv,
                  void *workspace, size_t workspace_bytes,
                  int B, int H, int N, int d, float scale, int causal, int dtype,
                  void *stream);

/* Workspace of fa_bwd_ex: it depends on the query side only (Nq rows). */
FA_API size_t fa_bwd_ex_workspace_bytes(int B, int H, int Nq, int Nk, int d);

/*
 * General backward, the arguments and layouts of fa_fwd_ex: dq [B][H][Nq][d],
 * dk, dv [B][H][Nk][d].  Reads the lse fa_fwd_ex wrote with the same
 * arguments.  Keys that no query sees get zero dk, dv.
 */
FA_API int fa_bwd_ex(const void *q, const void *k, const void *v, const void *o, const void *dout,
                     const float *lse, void *dq, void *dk, void *dv,
                     void *workspace, size_t workspace_bytes,
                     int B, int H, int Nq, int Nk, int d, float scale, int causal,
                     int window_left, int window_right, const float *alibi_slopes,
                     const uint8_t *block_mask, int dtype, void *stream);

/*
 * Packed variable-length batches (the varlen form of the flash_attn_func
 * interface of "FlashAttention原理概览" section 3.4): B sequences of
 * different lengths concatenated along the token axis, each attending only
 * within itself.
 *   q, o      [total_q][H][d]   k, v [total_k][H][d]   (token major, d innermost)
 *   lse       fp32 [H][total_q]
 *   cu_seqlens_q, cu_seqlens_k   DEVICE int32 [B + 1], 4-byte aligned: the
 *             cumulative lengths; sequence b owns query rows
 *             cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and key rows
 *             cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1.  They should start at
 *             0, never decrease and end at total_q / total_k; sequences may
 *             be empty.
 *   max_seqlen_q, max_seqlen_k   host upper bounds of the lengths (they size
 *             the grids), 1 <= max_seqlen <= total.
 * Within sequence b the problem is the one of fa_fwd_ex with Nq, Nk its own
 * lengths: causal and window are bottom-right aligned per sequence, and
 * alibi_slopes are per head.  Query rows of a sequence with no keys get
 * O = 0, LSE = -inf.  Block masks are not accepted (FA_ERR_UNSUPPORTED).
 * The library cannot read cu_seqlens on the host: the kernels clamp every
 * bound into [0, total] and every length to max_seqlen, so that nothing
 * outside the buffers is touched whatever the arrays hold, and record
 * FA_ERR_INVALID_ARG for fa_last_device_status() when a clamp changed
 * anything (the outputs are then incomplete).
 */
FA_API int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                         const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int H, int total_q, int total_k,
                         int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal, int window_left,
                         int window_right, const float *alibi_slopes, int dtype, void *stream);

/*
 * Workspace of fa_bwd_varlen: the two fp32 statistics [B][H][Npad] (Npad =
 * max_seqlen_q rounded up to FA_BLOCK) and the fp32 dQ accumulator
 * [H][total_q][d].  0 for invalid sizes.
 */
FA_API size_t fa_bwd_varlen_workspace_bytes(int B, int H, int total_q, int max_seqlen_q, int d);

/*
 * Backward of fa_fwd_varlen with the same arguments: dq [total_q][H][d],
 * dk, dv [total_k][H][d], d = 64, 128 or 256.  dq is accumulated with fp32
 * atomics as in fa_bwd.
 */
FA_API int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const void *dout,
                         const float *lse, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                         const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int H, int total_q, int total_k,
                         int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal, int window_left,
                         int window_right, const float *alibi_slopes, int dtype, void *stream);

/* Workspace of fa_bwd_varlen_deterministic: the two statistics only. */
FA_API size_t fa_bwd_varlen_deterministic_workspace_bytes(int B, int H, int total_q, int max_seqlen_q, int d);

/*
 * fa_bwd_varlen with bitwise reproducible dq, dk, dv: as fa_bwd_deterministic,
 * dQ is summed over each query tile's key blocks in a fixed order by a second
 * pass instead of with atomics.  Same arguments as fa_bwd_varlen; the
 * workspace is fa_bwd_varlen_deterministic_workspace_bytes().
 */
FA_API int fa_bwd_varlen_deterministic(const void *q, const void *k, const void *v, const void *o,
                                       const void *dout, const float *lse, void *dq, void *dk, void *dv,
                                       void *workspace, size_t workspace_bytes, const int *cu_seqlens_q,
                                       const int *cu_seqlens_k, int B, int H, int total_q, int total_k,
                                       int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal,
                                       int window_left, int window_right, const float *alibi_slopes, int dtype,
                                       void *stream);

/*
 * Bytes of device workspace fa_bwd_deterministic needs: the two fp32 per-row
 * statistics [B][H][Npad] only (no dQ accumulator).  0 for invalid sizes.
 */
FA_API size_t fa_bwd_deterministic_workspace_bytes(int B, int H, int Nq, int Nk, int d);

/*
 * Deterministic backward: the arguments, layouts and results of fa_bwd_ex,
 * with every output bitwise reproducible from run to run ("深度解析"
 * section 五 notes that a fully deterministic backward costs speed).  dK and
 * dV come from the key-block kernel as in fa_bwd_ex (same bits); dQ comes
 * from a second sweep, one CTA per 128 query rows, that recomputes S and dP
 * and sums dS K over the visible key blocks in increasing order in tensor
 * memory -- no atomics.  It performs seven matrix products per visible
 * block pair instead of five.  workspace: at least
 * fa_bwd_deterministic_workspace_bytes() bytes, 16-byte aligned.
 */
FA_API int fa_bwd_deterministic(const void *q, const void *k, const void *v, const void *o,
                                const void *dout, const float *lse, void *dq, void *dk, void *dv,
                                void *workspace, size_t workspace_bytes,
                                int B, int H, int Nq, int Nk, int d, float scale, int causal,
                                int window_left, int window_right, const float *alibi_slopes,
                                const uint8_t *block_mask, int dtype, void *stream);

/* Block-sparse backward; block_mask as for fa_fwd_blocksparse. */
FA_API int fa_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o,
                              const void *dout, const float *lse, void *dq, void *dk, void *dv,
                              void *workspace, size_t workspace_bytes,
                              const uint8_t *block_mask,
                              int B, int H, int N, int d, float scale, int causal, int dtype,
                              void *stream);

/*
 * Backward pass that allocates nothing and takes no workspace.
 *
 * The FlashAttention pages have no counterpart to this entry point; it exists
 * for callers that cannot allocate device memory themselves: a plugin or
 * custom-op interface that hands the library its input and output buffers but
 * no allocator, or code that must not call cudaMalloc on its path (the call
 * can synchronise the device, and it fails once a framework's caching
 * allocator has reserved most of the memory).
 *
 * Same arguments and results as fa_bwd, minus the workspace.  The scratch the
 * backward needs (fa_bwd_workspace_bytes(B, H, N, d) bytes: two fp32 per-row
 * statistics and an fp32 dQ accumulator) comes from one array of
 * FA_NOALLOC_SCRATCH_BYTES bytes that the library holds in device memory on
 * every GPU that loads it, until the process exits.  Problems that need more
 * are rejected with FA_ERR_SCRATCH_LIMIT before anything is launched.
 *
 * Every call looks up the current device's address of the array
 * (cudaGetSymbolAddress, with that device current); the first call on a
 * device also loads the library's module there, so make that first call
 * before any stream capture.  Every call on a device shares the one array, so
 * calls whose kernels overlap on the GPU (different streams without ordering
 * between them) race and give wrong results; order them on one stream.  The
 * array keeps the last call's contents; each call clears what it needs zeroed.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
FA_API int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                          const void *dout, const float *lse, void *dq, void *dk, void *dv,
                          int B, int H, int N, int d, float scale, int causal, int dtype,
                          void *stream);

/*
 * FP8 forward with block quantisation and incoherent processing
 * ("深度解析" section 四: FlashAttention-3's FP8 block quantisation, paired
 * with incoherent processing to lower the FP8 error).
 *
 * fa_fp8_quantize_qkv: q, k, v [B][H][N][d] (DEVICE, dtype FA_F16/FA_BF16,
 * d in {64, 128, 256}) -> E4M3 codes q8, k8, v8 [B][H][N][d] (DEVICE uint8,
 * caller-owned) and fp32 scales sq, sk, sv [B][H][ceil(N/128)] (DEVICE):
 *   - with signs (DEVICE float [d] of +1/-1) Q and K are first multiplied by
 *     diag(signs) H_d / sqrt(d) (H_d the Sylvester Hadamard matrix), which
 *     leaves Q K^T unchanged; signs = NULL skips the rotation.  V is never
 *     rotated.
 *   - Q and K get one scale per 128-row block, V one per head (stored in every
 *     block slot of sv): scale = amax / 448, code = E4M3(x * 448 / amax),
 *     rounded to nearest even and saturating at 448; an all-zero block gets
 *     scale 1.  The rotation and the quantiser run in fp32 in a fixed operation
 *     order, so the codes are a pure function of the inputs.
 * Three launches on `stream`.  Pointers: the tensors 16-byte aligned, the
 * scales and signs 4-byte aligned.
 *
 * fa_fwd_fp8: the forward on those codes (d = 64, 128 or 256, N = Nq = Nk, causal
 * or dense, no mask): S = scale * sq * sk * q8 . k8 with fp32 accumulation,
 * the online softmax in fp32, P rounded to E4M3 for the P V product,
 * O = sv * sum P8 v8 / sum P8 written as out_dtype (FA_F16/FA_BF16) [B][H][N][d],
 * lse [B][H][N] fp32 as fa_fwd.  Returns FA_ERR_UNSUPPORTED for other d.
 */
FA_API int fa_fp8_quantize_qkv(const void *q, const void *k, const void *v,
                               uint8_t *q8, uint8_t *k8, uint8_t *v8,
                               float *sq, float *sk, float *sv,
                               int B, int H, int N, int d, const float *signs, int dtype,
                               void *stream);
FA_API int fa_fwd_fp8(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8,
                      const float *sq, const float *sk, const float *sv,
                      void *o, float *lse, int B, int H, int N, int d,
                      float scale, int causal, int out_dtype, void *stream);

/* A static, human-readable name for a status code. */
FA_API const char *fa_status_string(int status);

/*
 * The device error word written by kernels that gave up waiting
 * (FA_ERR_TIMEOUT) since the last call, then cleared.  Synchronises the
 * current device.  FA_OK when nothing went wrong.
 */
FA_API int fa_last_device_status(void);

/*
 * Where the first wait that gave up (FA_ERR_TIMEOUT) was, for diagnosis:
 * site[0..4] = block x, block y, warp, shared-memory address of the
 * mbarrier, phase parity waited for.  site is a HOST array of 5 ints.  The
 * record is kept until a later timeout overwrites it (it is not cleared by
 * fa_last_device_status).  Synchronises the current device.
 */
FA_API int fa_last_timeout_site(int *site);

/*
 * Failure-detection self-test.  Launches one CTA of `warps` warps (1 .. 32)
 * on `stream` in which every warp waits, with the library's bounded wait,
 * for an mbarrier phase that nothing completes; warp w starts its wait
 * w x 100 ms after the CTA starts.  The first warp to reach the bound (3 s)
 * raises the CTA's abort flag, which the other warps see at once although
 * their own bounds have not run out, and records FA_ERR_TIMEOUT and where it
 * waited; the kernel then returns (after about 3 s, not 3 s + 100 ms x
 * (warps - 1)),
 * with nothing in flight and the context usable.  The call synchronises the
 * stream and returns the recorded status: FA_ERR_TIMEOUT when the wait gave
 * up as designed (FA_OK would mean the wait completed: a defect).
 * site[0..4] (a HOST array of 5 ints) receives block x, block y, warp,
 * shared-memory address of the mbarrier and the parity waited for.  Uses its
 * own copies of the device words: fa_last_device_status() and
 * fa_last_timeout_site() are not touched.  FA_ERR_INVALID_ARG for warps
 * outside 1 .. 32 or a null site, before anything is launched; FA_ERR_CUDA
 * on a CUDA error.  Takes about 3 s.
 */
FA_API int fa_selftest_wait_timeout(int warps, void *stream, int *site);

/*
 * Per-kernel timing, for benchmarks.  While enabled (on != 0), every call
 * records a pair of CUDA events on the caller's stream around each kernel it
 * launches.  fa_profile_read() waits for those events, writes the summed
 * milliseconds and launch counts per kernel kind, clears the record and
 * returns FA_OK.  Kinds: 0 forward, 1 backward pre-pass (D and accumulator
 * reset), 2 backward main kernel, 3 backward dQ conversion, 4 dQ pass of the
 * deterministic backward, 5 FP8 quantiser, 6 FP8 forward.  ms and launches
 * are HOST arrays of FA_PROFILE_KINDS entries.  Events are created and
 * destroyed by the library; no device memory is allocated.
 */
#define FA_PROFILE_KINDS 7
FA_API int fa_profile_enable(int on);
FA_API int fa_profile_read(float *ms, int *launches);

/* Library version, major * 10000 + minor * 100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
