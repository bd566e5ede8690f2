"""ctypes wrapper over liboracle.so, the plain fp64 C reference (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the benchmark's
CPU-baseline leg, never by the product package.

Every function takes float64 numpy arrays laid out [BH, N, d] (one batch-head
after another, the same order as the CUDA path's BHND tensors flattened over
B and H) and returns float64 arrays.  The definitions computed are written out
at the top of oracle.c with the passages they follow.
"""
import ctypes
import os
import subprocess

import numpy as np

CAUSAL = 1
SPARSE = 2

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
        lib.oracle_fwd_rows.argtypes = [D, D, D, i, i, i, f, i, U8, i, I32, i, D, D, i]
        lib.oracle_online_softmax_fwd.argtypes = [D, D, D, i, i, f, i, U8, i, i, D, D]
        lib.oracle_bwd_full.argtypes = [D, D, D, D, i, i, i, f, i, U8, i, D, D, D, D, D, i]
        lib.oracle_bwd_dq_rows.argtypes = [D, D, D, D, i, i, i, f, i, U8, i, I32, i, D, i]
        lib.oracle_bwd_dkdv_cols.argtypes = [D, D, D, D, i, i, i, f, i, U8, i, I32, i, D, D, i]
        for fn in (lib.oracle_fwd_rows, lib.oracle_online_softmax_fwd, lib.oracle_bwd_full,
                   lib.oracle_bwd_dq_rows, lib.oracle_bwd_dkdv_cols):
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
    return int(n) if n else (os.cpu_count() or 1)


def _check_qkv(q, k, v):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim == 2:
        q, k, v = q[None], k[None], v[None]
    assert q.shape == k.shape == v.shape and q.ndim == 3, "expected [BH, N, d]"
    return q, k, v


def fwd_rows(q, k, v, scale, flags=0, mask=None, blk=128, rows=None, nthreads=None):
    """O [BH, len(rows), d] and LSE [BH, len(rows)] on the given query rows."""
    q, k, v = _check_qkv(q, k, v)
    BH, N, d = q.shape
    rows = np.arange(N, dtype=np.int32) if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    o = np.zeros((BH, len(rows), d))
    lse = np.zeros((BH, len(rows)))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_fwd_rows(_dp(q), _dp(k), _dp(v), BH, N, d, float(scale), int(flags), mp, int(blk),
                                rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), len(rows),
                                _dp(o), _dp(lse), _threads(nthreads))
    assert rc == 0, rc
    return o, lse


def fwd(q, k, v, scale, flags=0, mask=None, blk=128, nthreads=None):
    """O and LSE on every query row."""
    return fwd_rows(q, k, v, scale, flags, mask, blk, None, nthreads)


def online_softmax_fwd(q, k, v, scale, tile, flags=0, mask=None, blk=128):
    """One head [N, d]: the tiled online-softmax recurrence with `tile` keys per step."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, d = q.shape
    o = np.zeros((N, d))
    lse = np.zeros(N)
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_online_softmax_fwd(_dp(q), _dp(k), _dp(v), N, d, float(scale), int(flags), mp,
                                          int(blk), int(tile), _dp(o), _dp(lse))
    assert rc == 0, rc
    return o, lse


def bwd_full(q, k, v, dout, scale, flags=0, mask=None, blk=128, nthreads=None):
    """(O, LSE, dQ, dK, dV), materialising the N x N matrices of every head."""
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout).reshape(q.shape)
    BH, N, d = q.shape
    o, dq, dk, dv = (np.zeros_like(q) for _ in range(4))
    lse = np.zeros((BH, N))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_bwd_full(_dp(q), _dp(k), _dp(v), _dp(dout), BH, N, d, float(scale), int(flags), mp,
                                int(blk), _dp(o), _dp(lse), _dp(dq), _dp(dk), _dp(dv), _threads(nthreads))
    assert rc == 0, rc
    return o, lse, dq, dk, dv


def bwd_dq_rows(q, k, v, dout, scale, rows, flags=0, mask=None, blk=128, nthreads=None):
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout).reshape(q.shape)
    BH, N, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    dq = np.zeros((BH, len(rows), d))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_bwd_dq_rows(_dp(q), _dp(k), _dp(v), _dp(dout), BH, N, d, float(scale), int(flags), mp,
                                   int(blk), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), len(rows),
                                   _dp(dq), _threads(nthreads))
    assert rc == 0, rc
    return dq


def bwd_dkdv_cols(q, k, v, dout, scale, cols, flags=0, mask=None, blk=128, nthreads=None):
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout).reshape(q.shape)
    BH, N, d = q.shape
    cols = np.ascontiguousarray(cols, dtype=np.int32)
    dk = np.zeros((BH, len(cols), d))
    dv = np.zeros((BH, len(cols), d))
    m, mp = _mask_arg(mask)
    rc = _lib().oracle_bwd_dkdv_cols(_dp(q), _dp(k), _dp(v), _dp(dout), BH, N, d, float(scale), int(flags), mp,
                                     int(blk), cols.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), len(cols),
                                     _dp(dk), _dp(dv), _threads(nthreads))
    assert rc == 0, rc
    return dk, dv
