"""ctypes wrapper over liboracle.so, the plain fp64 C reference (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the benchmark's
CPU-baseline leg, never by the product package.

Every function takes float64 numpy arrays laid out [BH, N, d] (one batch-head
after another, the same order as the CUDA path's BHND tensors flattened over
B and H) and returns float64 arrays.  Queries and keys may differ in length:
q and dout are [BH, Nq, d], k and v [BH, Nk, d] (bottom-right aligned).
Optional modes: window=(left, right) (a negative side is unbounded) and
slopes=[H] for ALiBi (batch-head bh uses slopes[bh % H]).  The definitions
computed are written out at the top of oracle.c with the passages they follow.
"""
import ctypes
import os
import subprocess

import numpy as np

CAUSAL = 1
SPARSE = 2
WINDOW = 4
ALIBI = 8

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def library_path():
    """liboracle.so next to this file; ORACLE_LIB overrides it (used only by
    the mutation test, which loads deliberately broken builds)."""
    return os.environ.get("ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")


def build(force=False):
    """Compile oracle.c with gcc into liboracle.so next to it."""
    out = library_path()
    src = os.path.join(_HERE, "oracle.c")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-fPIC", "-shared", "-o", out, src, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True, cwd=_HERE)
    return out


def _lib():
    global _LIB
    if _LIB is None:
        if not os.environ.get("ORACLE_LIB"):
            build()
        lib = ctypes.CDLL(library_path())
        D = ctypes.POINTER(ctypes.c_double)
        U8 = ctypes.POINTER(ctypes.c_uint8)
        I32 = ctypes.POINTER(ctypes.c_int)
        i, f = ctypes.c_int, ctypes.c_double
        lib.oracle_fwd_rows_ex.argtypes = [D, D, D, i, i, i, i, i, f, i, i, i, D, U8, i, I32, i, D, D, i]
        lib.oracle_online_softmax_fwd_ex.argtypes = [D, D, D, i, i, i, f, i, i, i, D, U8, i, i, D, D]
        lib.oracle_bwd_full_ex.argtypes = [D, D, D, D, i, i, i, i, i, f, i, i, i, D, U8, i, D, D, D, D, D, i]
        lib.oracle_bwd_dq_rows_ex.argtypes = [D, D, D, D, i, i, i, i, i, f, i, i, i, D, U8, i, I32, i, D, i]
        lib.oracle_bwd_dkdv_cols_ex.argtypes = [D, D, D, D, i, i, i, i, i, f, i, i, i, D, U8, i, I32, i, D, D, i]
        F32 = ctypes.POINTER(ctypes.c_float)
        lib.oracle_e4m3_value.argtypes = [i]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_round.argtypes = [f]
        lib.oracle_e4m3_round_array.argtypes = [D, ctypes.c_long, U8]
        lib.oracle_rotate_f32.argtypes = [F32, ctypes.c_long, i, F32]
        lib.oracle_fp8_quantize.argtypes = [F32, i, i, i, i, F32, U8, F32]
        lib.oracle_fwd_fp8.argtypes = [U8, U8, U8, F32, F32, F32, i, i, i, i, f, i, i, I32, i, D, D, i]
        for fn in (lib.oracle_fwd_rows_ex, lib.oracle_online_softmax_fwd_ex, lib.oracle_bwd_full_ex,
                   lib.oracle_bwd_dq_rows_ex, lib.oracle_bwd_dkdv_cols_ex, lib.oracle_e4m3_round,
                   lib.oracle_e4m3_round_array, lib.oracle_rotate_f32, lib.oracle_fp8_quantize, lib.oracle_fwd_fp8):
            fn.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _f64(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _mask_arg(mask):
    if mask is None:
        return None, None
    m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
    return m, m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _threads(n):
    """Threads for one call: n, else ORACLE_THREADS, else every core."""
    if n:
        return int(n)
    return int(os.environ.get("ORACLE_THREADS", "0")) or (os.cpu_count() or 1)


def _check_qkv(q, k, v):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim == 2:
        q, k, v = q[None], k[None], v[None]
    assert q.ndim == 3 and k.shape == v.shape and k.ndim == 3, "expected [BH, N, d]"
    assert q.shape[0] == k.shape[0] and q.shape[2] == k.shape[2], "q [BH, Nq, d] and k, v [BH, Nk, d]"
    return q, k, v


def _modes(flags, window, slopes):
    """flags with WINDOW / ALIBI set from the arguments; (left, right, slopes array, H)."""
    flags = int(flags)
    left = right = -1
    if window is not None:
        flags |= WINDOW
        left, right = int(window[0]), int(window[1])
    sl = None
    H = 1
    if slopes is not None:
        flags |= ALIBI
        sl = np.ascontiguousarray(np.asarray(slopes, dtype=np.float64).reshape(-1))
        H = len(sl)
    return flags, left, right, sl, H


def _sp(a):
    return None if a is None else _dp(a)


def fwd_rows(q, k, v, scale, flags=0, mask=None, blk=128, rows=None, nthreads=None, window=None, slopes=None):
    """O [BH, len(rows), d] and LSE [BH, len(rows)] on the given query rows."""
    q, k, v = _check_qkv(q, k, v)
    BH, Nq, d = q.shape
    Nk = k.shape[1]
    fl, left, right, sl, H = _modes(flags, window, slopes)
    rows = np.arange(Nq, dtype=np.int32) if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    o = np.zeros((BH, len(rows), d))
    lse = np.zeros((BH, len(rows)))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_fwd_rows_ex(_dp(q), _dp(k), _dp(v), BH, H, Nq, Nk, d, float(scale), fl, left, right,
                                   _sp(sl), mp, int(blk), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                   len(rows), _dp(o), _dp(lse), _threads(nthreads))
    assert rc == 0, rc
    return o, lse


def fwd(q, k, v, scale, flags=0, mask=None, blk=128, nthreads=None, window=None, slopes=None):
    """O and LSE on every query row."""
    return fwd_rows(q, k, v, scale, flags, mask, blk, None, nthreads, window, slopes)


def online_softmax_fwd(q, k, v, scale, tile, flags=0, mask=None, blk=128, window=None, slope=None):
    """One head (q [Nq, d], k, v [Nk, d]): the tiled online-softmax recurrence with `tile` keys per step."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Nq, d = q.shape
    Nk = k.shape[0]
    fl, left, right, sl, _ = _modes(flags, window, None if slope is None else [slope])
    o = np.zeros((Nq, d))
    lse = np.zeros(Nq)
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_online_softmax_fwd_ex(_dp(q), _dp(k), _dp(v), Nq, Nk, d, float(scale), fl, left, right,
                                             _sp(sl), mp, int(blk), int(tile), _dp(o), _dp(lse))
    assert rc == 0, rc
    return o, lse


def bwd_full(q, k, v, dout, scale, flags=0, mask=None, blk=128, nthreads=None, window=None, slopes=None):
    """(O, LSE, dQ, dK, dV), materialising the Nq x Nk matrices of every head."""
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout).reshape(q.shape)
    BH, Nq, d = q.shape
    Nk = k.shape[1]
    fl, left, right, sl, H = _modes(flags, window, slopes)
    o, dq = np.zeros_like(q), np.zeros_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(k)
    lse = np.zeros((BH, Nq))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_bwd_full_ex(_dp(q), _dp(k), _dp(v), _dp(dout), BH, H, Nq, Nk, d, float(scale), fl, left,
                                   right, _sp(sl), mp, int(blk), _dp(o), _dp(lse), _dp(dq), _dp(dk), _dp(dv),
                                   _threads(nthreads))
    assert rc == 0, rc
    return o, lse, dq, dk, dv


def bwd_dq_rows(q, k, v, dout, scale, rows, flags=0, mask=None, blk=128, nthreads=None, window=None, slopes=None):
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout).reshape(q.shape)
    BH, Nq, d = q.shape
    Nk = k.shape[1]
    fl, left, right, sl, H = _modes(flags, window, slopes)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    dq = np.zeros((BH, len(rows), d))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_bwd_dq_rows_ex(_dp(q), _dp(k), _dp(v), _dp(dout), BH, H, Nq, Nk, d, float(scale), fl, left,
                                      right, _sp(sl), mp, int(blk), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                      len(rows), _dp(dq), _threads(nthreads))
    assert rc == 0, rc
    return dq


def bwd_dkdv_cols(q, k, v, dout, scale, cols, flags=0, mask=None, blk=128, nthreads=None, window=None,
                  slopes=None):
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout).reshape(q.shape)
    BH, Nq, d = q.shape
    Nk = k.shape[1]
    fl, left, right, sl, H = _modes(flags, window, slopes)
    cols = np.ascontiguousarray(cols, dtype=np.int32)
    dk = np.zeros((BH, len(cols), d))
    dv = np.zeros((BH, len(cols), d))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_bwd_dkdv_cols_ex(_dp(q), _dp(k), _dp(v), _dp(dout), BH, H, Nq, Nk, d, float(scale), fl,
                                        left, right, _sp(sl), mp, int(blk),
                                        cols.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), len(cols),
                                        _dp(dk), _dp(dv), _threads(nthreads))
    assert rc == 0, rc
    return dk, dv


# --------------------------------------------------------------------------
# Packed variable-length batches.  Sequence b is an attention problem of its
# own: query rows cu_q[b] .. cu_q[b+1]-1 against key rows cu_k[b] ..
# cu_k[b+1]-1 (bottom-right aligned as above), so the packed result is the
# per-sequence definition applied to each slice ("FlashAttention原理概览"
# section 3.4 interface, its variable-length form).  Packed tensors are
# [total, H, d]; LSE is [H, total_q].  A row whose sequence has no keys gets
# O = 0, LSE = -inf and zero gradients.
# --------------------------------------------------------------------------
def _bounds(cu):
    cu = np.asarray(cu, dtype=np.int64).reshape(-1)
    assert cu.ndim == 1 and len(cu) >= 2 and cu[0] == 0 and np.all(np.diff(cu) >= 0), "cumulative lengths"
    return cu


def _heads(x):
    """[n, H, d] packed slice -> [H, n, d]."""
    return np.ascontiguousarray(np.transpose(_f64(x), (1, 0, 2)))


def fwd_varlen(q, k, v, cu_q, cu_k, scale, flags=0, window=None, slopes=None, nthreads=None):
    """O [total_q, H, d] and LSE [H, total_q] of a packed batch."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq, ck = _bounds(cu_q), _bounds(cu_k)
    assert len(cq) == len(ck) and cq[-1] == q.shape[0] and ck[-1] == k.shape[0]
    total_q, H, d = q.shape
    o = np.zeros((total_q, H, d))
    lse = np.full((H, total_q), -np.inf)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0 or k1 == k0:
            continue
        ob, lb = fwd(_heads(q[q0:q1]), _heads(k[k0:k1]), _heads(v[k0:k1]), scale, flags, nthreads=nthreads,
                     window=window, slopes=slopes)
        o[q0:q1] = np.transpose(ob, (1, 0, 2))
        lse[:, q0:q1] = lb
    return o, lse


def bwd_varlen(q, k, v, dout, cu_q, cu_k, scale, flags=0, window=None, slopes=None, nthreads=None):
    """(O, LSE, dQ, dK, dV) of a packed batch, each sequence by bwd_full."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    cq, ck = _bounds(cu_q), _bounds(cu_k)
    assert len(cq) == len(ck) and cq[-1] == q.shape[0] and ck[-1] == k.shape[0]
    total_q, H, d = q.shape
    o, dq = np.zeros_like(q), np.zeros_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(k)
    lse = np.full((H, total_q), -np.inf)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0 or k1 == k0:
            continue
        ob, lb, dqb, dkb, dvb = bwd_full(_heads(q[q0:q1]), _heads(k[k0:k1]), _heads(v[k0:k1]),
                                         _heads(dout[q0:q1]), scale, flags, nthreads=nthreads, window=window,
                                         slopes=slopes)
        o[q0:q1] = np.transpose(ob, (1, 0, 2))
        lse[:, q0:q1] = lb
        dq[q0:q1] = np.transpose(dqb, (1, 0, 2))
        dk[k0:k1] = np.transpose(dkb, (1, 0, 2))
        dv[k0:k1] = np.transpose(dvb, (1, 0, 2))
    return o, lse, dq, dk, dv


# --------------------------------------------------------------------------
# FP8 forward (block quantisation + incoherent processing); the readings are
# written out above the FP8 section of oracle.c
# --------------------------------------------------------------------------
def _u8p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _f32p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def e4m3_values():
    """float64 [256]: the value of every E4M3 code (NaN for the two NaN codes)."""
    return np.array([_lib().oracle_e4m3_value(c) for c in range(256)])


def e4m3_round(x):
    """uint8 codes of the values x (nearest, ties to even, saturating at 448)."""
    x = _f64(x)
    codes = np.zeros(x.shape, dtype=np.uint8)
    rc = _lib().oracle_e4m3_round_array(_dp(x), x.size, _u8p(codes))
    assert rc == 0, rc
    return codes


def rotate_f32(x, signs):
    """float32 rows x [..., d] <- (x o signs) H_d / sqrt(d), in float."""
    x = np.ascontiguousarray(np.array(x, dtype=np.float32))
    s = np.ascontiguousarray(np.asarray(signs, dtype=np.float32))
    d = x.shape[-1]
    rc = _lib().oracle_rotate_f32(_f32p(x), x.size // d, d, _f32p(s))
    assert rc == 0, rc
    return x


def fp8_quantize(x, rows, signs=None):
    """x [BH, N, d] (float32) -> (codes uint8 [BH, N, d], scales float32 [BH, ceil(N / rows)])."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if x.ndim == 2:
        x = x[None]
    BH, N, d = x.shape
    nb = (N + rows - 1) // rows
    codes = np.zeros((BH, N, d), dtype=np.uint8)
    scales = np.zeros((BH, nb), dtype=np.float32)
    s = None if signs is None else np.ascontiguousarray(np.asarray(signs, dtype=np.float32))
    rc = _lib().oracle_fp8_quantize(_f32p(x), BH, N, d, int(rows), None if s is None else _f32p(s),
                                    _u8p(codes), _f32p(scales))
    assert rc == 0, rc
    return codes, scales


def fwd_fp8(q8, k8, v8, sq, sk, sv, scale, causal=False, rows=None, quant_p=True, blk=128, nthreads=None):
    """O [BH, len(rows), d] and LSE [BH, len(rows)] of FP8 attention on the codes
    (q8, k8, v8 uint8 [BH, N, d]) and scales (sq, sk [BH, ceil(N / blk)], sv [BH])."""
    q8, k8, v8 = (np.ascontiguousarray(np.asarray(t, dtype=np.uint8)) for t in (q8, k8, v8))
    sq, sk, sv = (np.ascontiguousarray(np.asarray(t, dtype=np.float32)) for t in (sq, sk, sv))
    BH, N, d = q8.shape
    rows = np.arange(N, dtype=np.int32) if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    o = np.zeros((BH, len(rows), d))
    lse = np.zeros((BH, len(rows)))
    rc = _lib().oracle_fwd_fp8(_u8p(q8), _u8p(k8), _u8p(v8), _f32p(sq), _f32p(sk), _f32p(sv), BH, N, d, int(blk),
                               float(scale), int(bool(causal)), int(bool(quant_p)),
                               rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), len(rows), _dp(o), _dp(lse),
                               _threads(nthreads))
    assert rc == 0, rc
    return o, lse


def fp8_o_bounds(q8, k8, v8, sq, sk, sv, scale, causal, rows, o_ref, blk=128):
    """Bars on |O_kernel - O_oracle| of FP8 attention for query `rows` of ONE
    (batch, head): q8, k8, v8 uint8 [N, d], sq, sk float32 [ceil(N / blk)],
    sv the head's V scale, o_ref the oracle's O on those rows.

    Both sides round each P_j to E4M3 and divide by the sum of the rounded
    values; they take the rounding on differently scaled P (the kernel relative
    to its lazily rescaled running maximum, the oracle relative to the exact
    maximum), so each error e_j is within the half step
    u_j = max(2^-4 P_j, 2^-10) of P_j <= 1 (3 mantissa bits; the subnormal
    step 2^-9).  With O_o the oracle's result,
        O_k - O_o = sum_j (e_j - e'_j) (v_j - O_o) / sum_j (P_j + e_j),
    so |O_k - O_o| <= sum_j 2 u_j |v_j - O_o| / (sum_j P_j - sum_j u_j).
    Returns (worst, six_sigma): the worst case above, and 6 standard
    deviations of the same sum with the e_j independent and uniform; each plus
    the 16-bit rounding of the kernel's output and 1e-4 for its fp32 sums.
    """
    vals = e4m3_values()
    N = q8.shape[0]
    b = np.arange(N) // blk
    Q = vals[q8] * np.asarray(sq, dtype=np.float64)[b][:, None]
    K = vals[k8] * np.asarray(sk, dtype=np.float64)[b][:, None]
    V = vals[v8] * float(sv)
    rows = np.asarray(rows)
    S = scale * Q[rows] @ K.T
    if causal:
        S = np.where(np.arange(N)[None, :] > rows[:, None], -np.inf, S)
    P = np.exp(S - S.max(1, keepdims=True))
    u = np.minimum(P, np.maximum(P * 2.0 ** -4, 2.0 ** -10))   # below 2^-10 the code may be 0: error P
    den = P.sum(1, keepdims=True)
    worst = np.empty_like(o_ref)
    for r0 in range(0, len(rows), 32):                      # |v_j - O_o| for 32 rows at a time
        dev = np.abs(V[None, :, :] - o_ref[r0:r0 + 32, None, :])
        worst[r0:r0 + 32] = np.einsum("rn,rnd->rd", 2 * u[r0:r0 + 32], dev)
    worst /= den - u.sum(1, keepdims=True)
    w = (2 * u) ** 2 / 3.0
    var = w @ (V ** 2) - 2 * (w @ V) * o_ref + w.sum(1, keepdims=True) * o_ref ** 2
    sigma = np.sqrt(np.maximum(var, 0.0)) / den
    tail = lambda x: x + 2.0 ** -8 * (np.abs(o_ref) + x) + 1e-4   # noqa: E731
    return tail(worst), tail(6 * sigma)
