"""flash_fwd_b200 -- exact softmax attention on B200 (sm_100a).

A thin ctypes binding over ``libfa_b200.so`` (declared in ``include/fa.h``).
The functions below only marshal arguments: every step of the attention runs
in the library's CUDA kernels.  PyTorch supplies device memory and streams.

If the library has not been built the binding raises; there is no fallback.
"""
import ctypes
import os

import torch

__all__ = [
    "FaError", "load_library", "library_path", "fa_fwd", "fa_fwd_blocksparse", "fa_bwd",
    "fa_bwd_blocksparse", "fa_bwd_workspace_bytes", "fa_status_string", "fa_last_device_status", "fa_last_timeout_site",
    "fa_version", "attention_fwd", "attention_bwd", "FA_BLOCK", "fa_profile_enable", "fa_profile_read",
    "fa_fwd_ex", "fa_bwd_ex", "fa_bwd_ex_workspace_bytes", "fa_bwd_deterministic",
    "fa_bwd_deterministic_workspace_bytes", "fa_fp8_quantize_qkv", "fa_fwd_fp8", "attention_fwd_fp8",
    "fa_bwd_noalloc", "fa_fwd_varlen", "fa_bwd_varlen", "fa_bwd_varlen_workspace_bytes", "attention_fwd_varlen",
    "attention_bwd_varlen", "fa_bwd_varlen_deterministic", "fa_bwd_varlen_deterministic_workspace_bytes",
    "fa_selftest_wait_timeout",
]

FA_BLOCK = 128
_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB = None

FA_F16, FA_BF16 = 0, 1
_DTYPE = {torch.float16: FA_F16, torch.bfloat16: FA_BF16}


class FaError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: status {status} ({fa_status_string(status)})")


def library_path():
    return os.path.join(_PKG, "libfa_b200.so")


def load_library():
    """Loads libfa_b200.so once; raises if it is missing."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m flash_fwd_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    lib.fa_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    lib.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_bytes.restype = sz
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, i, vp]
    lib.fa_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, i, i, i, i, f, i, i, vp]
    lib.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, vp, i, vp]
    lib.fa_bwd_ex_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.fa_bwd_ex_workspace_bytes.restype = sz
    lib.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, i, vp, vp, i, vp]
    lib.fa_bwd_deterministic_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.fa_bwd_deterministic_workspace_bytes.restype = sz
    lib.fa_bwd_deterministic.argtypes = list(lib.fa_bwd_ex.argtypes)
    lib.fa_fp8_quantize_qkv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp, i, vp]
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    lib.fa_bwd_noalloc.argtypes = [vp] * 9 + [i, i, i, i, f, i, i, vp]
    lib.fa_fwd_varlen.argtypes = [vp] * 7 + [i] * 7 + [f, i, i, i, vp, i, vp]
    lib.fa_bwd_varlen_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.fa_bwd_varlen_workspace_bytes.restype = sz
    lib.fa_bwd_varlen.argtypes = [vp] * 10 + [sz, vp, vp] + [i] * 7 + [f, i, i, i, vp, i, vp]
    lib.fa_bwd_varlen_deterministic_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.fa_bwd_varlen_deterministic_workspace_bytes.restype = sz
    lib.fa_bwd_varlen_deterministic.argtypes = list(lib.fa_bwd_varlen.argtypes)
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_device_status.argtypes = []
    lib.fa_version.argtypes = []
    lib.fa_last_timeout_site.argtypes = [ctypes.POINTER(ctypes.c_int)]
    lib.fa_selftest_wait_timeout.argtypes = [i, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]
    lib.fa_profile_enable.argtypes = [i]
    lib.fa_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]
    for fn in (lib.fa_fwd, lib.fa_fwd_blocksparse, lib.fa_bwd, lib.fa_bwd_blocksparse, lib.fa_fwd_ex, lib.fa_bwd_ex,
               lib.fa_bwd_deterministic, lib.fa_fp8_quantize_qkv, lib.fa_fwd_fp8, lib.fa_bwd_noalloc,
               lib.fa_fwd_varlen, lib.fa_bwd_varlen, lib.fa_bwd_varlen_deterministic,
               lib.fa_last_device_status, lib.fa_last_timeout_site, lib.fa_version, lib.fa_profile_enable, lib.fa_profile_read,
               lib.fa_selftest_wait_timeout):
        fn.restype = ctypes.c_int
    _LIB = lib
    return lib


def fa_status_string(status):
    return load_library().fa_status_string(int(status)).decode()


def fa_last_device_status():
    return load_library().fa_last_device_status()


def fa_last_timeout_site():
    """(block x, block y, warp, mbarrier shared address, parity) of the first wait that gave up."""
    site = (ctypes.c_int * 5)()
    rc = load_library().fa_last_timeout_site(site)
    if rc != 0:
        raise FaError(rc, "fa_last_timeout_site")
    return tuple(site)


def fa_version():
    return load_library().fa_version()


def fa_selftest_wait_timeout(warps, stream=None):
    """Runs the failure self-test of the library (one CTA whose `warps` warps
    wait, bounded, for an mbarrier phase that nothing completes) and returns
    (status, site): FA_ERR_TIMEOUT (6) and the (block x, block y, warp,
    mbarrier shared address, parity) of the wait that gave up.  Synchronises
    the stream; takes about 3 s.  `stream` is a torch.cuda.Stream (None:
    the current stream).  Without a GPU the library answers FA_ERR_CUDA
    (FA_ERR_INVALID_ARG for a bad `warps`, checked first)."""
    site = (ctypes.c_int * 5)()
    s = _stream(stream) if torch.cuda.is_available() else ctypes.c_void_p(None)
    rc = load_library().fa_selftest_wait_timeout(int(warps), s, site)
    return rc, tuple(site)


PROFILE_KINDS = ("fwd", "bwd_pre", "bwd_main", "bwd_post", "bwd_dq", "fp8_quant", "fwd_fp8")


def fa_profile_enable(on=True):
    _check(load_library().fa_profile_enable(int(bool(on))), "fa_profile_enable")


def fa_profile_read():
    """{kind: (milliseconds, launches)} summed since the last read."""
    ms = (ctypes.c_float * len(PROFILE_KINDS))()
    n = (ctypes.c_int * len(PROFILE_KINDS))()
    _check(load_library().fa_profile_read(ms, n), "fa_profile_read")
    return {k: (float(ms[i]), int(n[i])) for i, k in enumerate(PROFILE_KINDS)}


def fa_bwd_workspace_bytes(B, H, N, d):
    return load_library().fa_bwd_workspace_bytes(B, H, N, d)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _current_device():
    """Index of the current CUDA device, where the library launches (asked once per call)."""
    return torch.cuda.current_device()


def _on_device(t, dev):
    """Is t in the memory of CUDA device dev?"""
    return t.is_cuda and t.get_device() == dev


_HALF = (torch.float16, torch.bfloat16)
_F32 = (torch.float32,)
_U8 = (torch.uint8,)


def _need(name, t, dev, dtypes=None, shape=None, numel=None):
    """Checks one tensor argument before its address goes to the library, which
    cannot check a pointer: a contiguous tensor in the current device's memory,
    of an accepted dtype and of the given shape (or element count).  Raises
    TypeError / ValueError; nothing is launched."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if not _on_device(t, dev):
        raise ValueError(f"{name}: must be a CUDA tensor on the current device (got {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not accepted ({', '.join(str(x) for x in dtypes)})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected {numel}")


def _need_attention(q, k, v, o, lse, square, dout=None, dq=None, dk=None, dv=None, workspace=None,
                    block_mask=None, alibi_slopes=None):
    """Checks the tensors of one attention call; returns (B, H, Nq, Nk, d)."""
    dev = _current_device() if isinstance(q, torch.Tensor) and q.is_cuda else -1
    _need("q", q, dev, _HALF)
    B, H, Nq, d = _shape(q)
    _need("k", k, dev, (q.dtype,))
    if k.dim() != 4 or tuple(k.shape[:2]) != (B, H) or int(k.shape[3]) != d or (square and k.shape[2] != Nq):
        raise ValueError(f"k: shape {tuple(k.shape)} does not match q {tuple(q.shape)}")
    Nk = int(k.shape[2])
    _need("v", v, dev, (q.dtype,), shape=k.shape)
    _need("o", o, dev, (q.dtype,), shape=q.shape)
    _need("lse", lse, dev, _F32, numel=B * H * Nq)
    for name, t, like in (("dout", dout, q), ("dq", dq, q), ("dk", dk, k), ("dv", dv, k)):
        if t is not None:
            _need(name, t, dev, (q.dtype,), shape=like.shape)
    if workspace is not None:
        _need("workspace", workspace, dev)          # its size is the library's check
    if block_mask is not None:
        _need("block_mask", block_mask, dev, _U8, numel=((Nq + 127) // 128) * ((Nk + 127) // 128))
    if alibi_slopes is not None:
        _need("alibi_slopes", alibi_slopes, dev, _F32, numel=H)
    return B, H, Nq, Nk, d


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _dtype(q):
    if q.dtype not in _DTYPE:
        raise ValueError("q, k, v must be float16 or bfloat16")
    return _DTYPE[q.dtype]


def _scale(scale, d):
    return float(scale) if scale is not None else 1.0 / float(d) ** 0.5


def _check(rc, what):
    if rc != 0:
        raise FaError(rc, what)


def fa_fwd(q, k, v, o, lse, causal=False, scale=None, stream=None):
    """O and LSE of exact attention; all tensors [B, H, N, d] (lse [B, H, N] fp32)."""
    B, H, N, _, d = _need_attention(q, k, v, o, lse, square=True)
    rc = load_library().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                               _scale(scale, d), int(bool(causal)), _dtype(q), _stream(stream))
    _check(rc, "fa_fwd")


def fa_fwd_blocksparse(q, k, v, o, lse, block_mask, causal=False, scale=None, stream=None):
    B, H, N, _, d = _need_attention(q, k, v, o, lse, square=True, block_mask=block_mask)
    rc = load_library().fa_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(block_mask),
                                           B, H, N, d, _scale(scale, d), int(bool(causal)), _dtype(q),
                                           _stream(stream))
    _check(rc, "fa_fwd_blocksparse")


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal=False, scale=None, stream=None):
    B, H, N, _, d = _need_attention(q, k, v, o, lse, True, dout, dq, dk, dv, workspace)
    rc = load_library().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                               _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               B, H, N, d, _scale(scale, d), int(bool(causal)), _dtype(q), _stream(stream))
    _check(rc, "fa_bwd")


def fa_bwd_blocksparse(q, k, v, o, dout, lse, dq, dk, dv, workspace, block_mask, causal=False, scale=None,
                       stream=None):
    B, H, N, _, d = _need_attention(q, k, v, o, lse, True, dout, dq, dk, dv, workspace, block_mask)
    rc = load_library().fa_bwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                                           _ptr(dk), _ptr(dv), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _ptr(block_mask),
                                           B, H, N, d, _scale(scale, d), int(bool(causal)), _dtype(q),
                                           _stream(stream))
    _check(rc, "fa_bwd_blocksparse")


def _window(window):
    return (-1, -1) if window is None else (int(window[0]), int(window[1]))


def fa_fwd_ex(q, k, v, o, lse, causal=False, scale=None, window=None, alibi_slopes=None, block_mask=None,
              stream=None):
    """General forward: q, o [B, H, Nq, d]; k, v [B, H, Nk, d]; lse [B, H, Nq] fp32.
    window=(left, right) (a negative side is unbounded), alibi_slopes: fp32 [H] on the device."""
    B, H, Nq, Nk, d = _need_attention(q, k, v, o, lse, False, block_mask=block_mask, alibi_slopes=alibi_slopes)
    wl, wr = _window(window)
    rc = load_library().fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                                  _scale(scale, d), int(bool(causal)), wl, wr, _ptr(alibi_slopes), _ptr(block_mask),
                                  _dtype(q), _stream(stream))
    _check(rc, "fa_fwd_ex")


def fa_bwd_ex_workspace_bytes(B, H, Nq, Nk, d):
    return load_library().fa_bwd_ex_workspace_bytes(B, H, Nq, Nk, d)


def fa_bwd_ex(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal=False, scale=None, window=None,
              alibi_slopes=None, block_mask=None, stream=None):
    B, H, Nq, Nk, d = _need_attention(q, k, v, o, lse, False, dout, dq, dk, dv, workspace, block_mask,
                                      alibi_slopes)
    wl, wr = _window(window)
    rc = load_library().fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  B, H, Nq, Nk, d, _scale(scale, d), int(bool(causal)), wl, wr, _ptr(alibi_slopes),
                                  _ptr(block_mask), _dtype(q), _stream(stream))
    _check(rc, "fa_bwd_ex")


def fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, causal=False, scale=None, stream=None):
    """fa_bwd without a workspace: the library's own device scratch serves (see include/fa.h)."""
    B, H, N, _, d = _need_attention(q, k, v, o, lse, True, dout, dq, dk, dv)
    rc = load_library().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                       _ptr(dv), B, H, N, d, _scale(scale, d), int(bool(causal)), _dtype(q),
                                       _stream(stream))
    _check(rc, "fa_bwd_noalloc")


def fa_bwd_deterministic_workspace_bytes(B, H, Nq, Nk, d):
    return load_library().fa_bwd_deterministic_workspace_bytes(B, H, Nq, Nk, d)


def fa_bwd_deterministic(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal=False, scale=None, window=None,
                         alibi_slopes=None, block_mask=None, stream=None):
    """fa_bwd_ex with bitwise reproducible outputs (dQ by a second sweep, no atomics)."""
    B, H, Nq, Nk, d = _need_attention(q, k, v, o, lse, False, dout, dq, dk, dv, workspace, block_mask,
                                      alibi_slopes)
    wl, wr = _window(window)
    rc = load_library().fa_bwd_deterministic(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
        workspace.numel() * workspace.element_size(), B, H, Nq, Nk, d, _scale(scale, d), int(bool(causal)), wl, wr,
        _ptr(alibi_slopes), _ptr(block_mask), _dtype(q), _stream(stream))
    _check(rc, "fa_bwd_deterministic")


def _general(q, k, window, alibi_slopes):
    return k.shape[2] != q.shape[2] or window is not None or alibi_slopes is not None


def attention_fwd(q, k, v, causal=False, scale=None, block_mask=None, stream=None, window=None,
                  alibi_slopes=None):
    """Allocates O and LSE with torch and runs the forward; returns (o, lse).
    k, v may have a different length from q (bottom-right aligned)."""
    B, H, Nq, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    if _general(q, k, window, alibi_slopes):
        fa_fwd_ex(q, k, v, o, lse, causal, scale, window, alibi_slopes, block_mask, stream)
    elif block_mask is None:
        fa_fwd(q, k, v, o, lse, causal, scale, stream)
    else:
        fa_fwd_blocksparse(q, k, v, o, lse, block_mask, causal, scale, stream)
    return o, lse


def attention_bwd(q, k, v, o, dout, lse, causal=False, scale=None, block_mask=None, workspace=None,
                  stream=None, window=None, alibi_slopes=None, deterministic=False):
    """Allocates dQ, dK, dV (and the workspace unless given) and runs the backward.
    deterministic=True gives bitwise reproducible dQ (a second sweep instead of atomics)."""
    B, H, Nq, d = _shape(q)
    Nk = int(k.shape[2])
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        nbytes = (fa_bwd_deterministic_workspace_bytes if deterministic else fa_bwd_ex_workspace_bytes)(B, H, Nq, Nk, d)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    if deterministic:
        fa_bwd_deterministic(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal, scale, window, alibi_slopes,
                             block_mask, stream)
    elif _general(q, k, window, alibi_slopes):
        fa_bwd_ex(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal, scale, window, alibi_slopes, block_mask,
                  stream)
    elif block_mask is None:
        fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, causal, scale, stream)
    else:
        fa_bwd_blocksparse(q, k, v, o, dout, lse, dq, dk, dv, workspace, block_mask, causal, scale, stream)
    return dq, dk, dv


def fa_fp8_quantize_qkv(q, k, v, signs=None, stream=None):
    """E4M3 codes and scales of q, k, v [B, H, N, d] (16-bit, on the device):
    returns (q8, k8, v8 uint8 [B, H, N, d], sq, sk, sv fp32 [B, H, ceil(N / 128)]).
    signs (fp32 [d] of +-1 on the device) rotates Q and K by diag(signs) H_d / sqrt(d)."""
    dev = _current_device() if isinstance(q, torch.Tensor) and q.is_cuda else -1
    _need("q", q, dev, _HALF)
    B, H, N, d = _shape(q)
    _need("k", k, dev, (q.dtype,), shape=q.shape)
    _need("v", v, dev, (q.dtype,), shape=q.shape)
    if signs is not None:
        _need("signs", signs, dev, _F32, numel=d)
    nb = (N + 127) // 128
    q8, k8, v8 = (torch.empty((B, H, N, d), dtype=torch.uint8, device=q.device) for _ in range(3))
    sq, sk, sv = (torch.empty((B, H, nb), dtype=torch.float32, device=q.device) for _ in range(3))
    rc = load_library().fa_fp8_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq),
                                            _ptr(sk), _ptr(sv), B, H, N, d, _ptr(signs), _dtype(q), _stream(stream))
    _check(rc, "fa_fp8_quantize_qkv")
    return q8, k8, v8, sq, sk, sv


def fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, causal=False, scale=None, stream=None):
    """FP8 forward on the codes and scales of fa_fp8_quantize_qkv; o [B, H, N, d]
    (float16 or bfloat16) and lse [B, H, N] fp32 are written."""
    dev = _current_device() if isinstance(q8, torch.Tensor) and q8.is_cuda else -1
    _need("q8", q8, dev, _U8)
    B, H, N, d = _shape(q8)
    nb = (N + 127) // 128
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _need(name, t, dev, _U8, shape=q8.shape)
    for name, t in (("sq", sq), ("sk", sk), ("sv", sv)):
        _need(name, t, dev, _F32, numel=B * H * nb)
    _need("o", o, dev, _HALF, shape=q8.shape)
    _need("lse", lse, dev, _F32, numel=B * H * N)
    rc = load_library().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(o), _ptr(lse),
                                   B, H, N, d, _scale(scale, d), int(bool(causal)), _dtype(o), _stream(stream))
    _check(rc, "fa_fwd_fp8")


def attention_fwd_fp8(q, k, v, causal=False, scale=None, signs=None, stream=None):
    """Quantises q, k, v to E4M3 (rotating Q and K when signs are given) and runs
    the FP8 forward; returns (o, lse) with o in q's dtype."""
    B, H, N, d = _shape(q)
    q8, k8, v8, sq, sk, sv = fa_fp8_quantize_qkv(q, k, v, signs, stream)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, causal, scale, stream)
    return o, lse


# ---------------------------------------------------------------- packed variable-length batches
_I32 = (torch.int32,)


def _need_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dout=None, dq=None,
                 dk=None, dv=None, workspace=None, alibi_slopes=None):
    """Checks the tensors of one packed call; returns (B, H, total_q, total_k, d)."""
    dev = _current_device() if isinstance(q, torch.Tensor) and q.is_cuda else -1
    _need("q", q, dev, _HALF)
    if q.dim() != 3:
        raise ValueError("packed q, k, v: expected [total, H, d] tensors")
    total_q, H, d = (int(x) for x in q.shape)
    _need("k", k, dev, (q.dtype,))
    if k.dim() != 3 or int(k.shape[1]) != H or int(k.shape[2]) != d:
        raise ValueError(f"k: shape {tuple(k.shape)} does not match q {tuple(q.shape)}")
    total_k = int(k.shape[0])
    _need("v", v, dev, (q.dtype,), shape=k.shape)
    _need("o", o, dev, (q.dtype,), shape=q.shape)
    _need("lse", lse, dev, _F32, shape=(H, total_q))
    _need("cu_seqlens_q", cu_seqlens_q, dev, _I32)
    _need("cu_seqlens_k", cu_seqlens_k, dev, _I32, shape=cu_seqlens_q.shape)
    if cu_seqlens_q.dim() != 1 or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens: expected [B + 1] int32 tensors")
    B = cu_seqlens_q.numel() - 1
    for name, t, like in (("dout", dout, q), ("dq", dq, q), ("dk", dk, k), ("dv", dv, k)):
        if t is not None:
            _need(name, t, dev, (q.dtype,), shape=like.shape)
    if workspace is not None:
        _need("workspace", workspace, dev)
    if alibi_slopes is not None:
        _need("alibi_slopes", alibi_slopes, dev, _F32, numel=H)
    return B, H, total_q, total_k, d


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False,
                  scale=None, window=None, alibi_slopes=None, stream=None):
    """Forward of a packed batch: q, o [total_q, H, d]; k, v [total_k, H, d]; lse [H, total_q] fp32;
    cu_seqlens_q / _k int32 [B + 1] on the device; max_seqlen_* host ints bounding the lengths."""
    B, H, tq, tk, d = _need_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                                   alibi_slopes=alibi_slopes)
    wl, wr = _window(window)
    rc = load_library().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                                      _ptr(cu_seqlens_k), B, H, tq, tk, int(max_seqlen_q), int(max_seqlen_k), d,
                                      _scale(scale, d), int(bool(causal)), wl, wr, _ptr(alibi_slopes), _dtype(q),
                                      _stream(stream))
    _check(rc, "fa_fwd_varlen")


def fa_bwd_varlen_workspace_bytes(B, H, total_q, max_seqlen_q, d):
    return load_library().fa_bwd_varlen_workspace_bytes(B, H, total_q, max_seqlen_q, d)


def fa_bwd_varlen_deterministic_workspace_bytes(B, H, total_q, max_seqlen_q, d):
    return load_library().fa_bwd_varlen_deterministic_workspace_bytes(B, H, total_q, max_seqlen_q, d)


def fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                  max_seqlen_k, causal=False, scale=None, window=None, alibi_slopes=None, stream=None,
                  deterministic=False):
    """Backward of a packed batch; deterministic=True: bitwise reproducible (fa_bwd_varlen_deterministic)."""
    B, H, tq, tk, d = _need_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dout,
                                   dq, dk, dv, workspace, alibi_slopes)
    wl, wr = _window(window)
    lib = load_library()
    rc = (lib.fa_bwd_varlen_deterministic if deterministic else lib.fa_bwd_varlen)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                      _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, H, tq, tk, int(max_seqlen_q),
                                      int(max_seqlen_k), d, _scale(scale, d), int(bool(causal)), wl, wr,
                                      _ptr(alibi_slopes), _dtype(q), _stream(stream))
    _check(rc, "fa_bwd_varlen_deterministic" if deterministic else "fa_bwd_varlen")


def attention_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False, scale=None,
                         window=None, alibi_slopes=None, stream=None):
    """Allocates O [total_q, H, d] and LSE [H, total_q] and runs the packed forward; returns (o, lse)."""
    o = torch.empty_like(q)
    lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, scale, window,
                  alibi_slopes, stream)
    return o, lse


def attention_bwd_varlen(q, k, v, o, dout, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                         causal=False, scale=None, window=None, alibi_slopes=None, workspace=None, stream=None,
                         deterministic=False):
    """Allocates dQ, dK, dV (and the workspace unless given) and runs the packed backward."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        ws = fa_bwd_varlen_deterministic_workspace_bytes if deterministic else fa_bwd_varlen_workspace_bytes
        nbytes = ws(cu_seqlens_q.numel() - 1, int(q.shape[1]), int(q.shape[0]), int(max_seqlen_q), int(q.shape[2]))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                  max_seqlen_k, causal, scale, window, alibi_slopes, stream, deterministic)
    return dq, dk, dv
