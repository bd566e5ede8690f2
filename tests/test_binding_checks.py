"""The binding's argument checks, on the CPU.

The C ABI receives raw device addresses and cannot tell a host pointer, a
strided view or a short buffer from a good one, so the Python binding checks
every tensor before its address leaves it.  Here:
* CPU tensors are refused by every compute wrapper (the library never runs on
  the host and there is no fallback);
* with the device test replaced and the library replaced by a recorder, the
  call patterns the GPU tests, the benchmark and smoke() use reach the library,
  and malformed calls (wrong shape, dtype, element count, a strided view) are
  refused before it.
"""
import pytest
import torch

import flash_fwd_b200 as fa

BF, F16, F32, U8 = torch.bfloat16, torch.float16, torch.float32, torch.uint8


class _Stream:
    cuda_stream = 0


S = _Stream()


class _FakeLib:
    """Records each entry point called; workspace sizes are 1 KB, calls succeed."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, len(args)))
            return 1024 if name.endswith("workspace_bytes") else 0
        return fn


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    monkeypatch.setattr(fa, "load_library", lambda: lib)
    monkeypatch.setattr(fa, "_on_device", lambda t, dev: True)
    monkeypatch.setattr(fa, "_current_device", lambda: 0)
    return lib


def _t(*shape, dtype=BF):
    return torch.zeros(shape, dtype=dtype)


def _fwd_args(B=1, H=2, Nq=200, Nk=None, d=64, dtype=BF):
    Nk = Nq if Nk is None else Nk
    return dict(q=_t(B, H, Nq, d, dtype=dtype), k=_t(B, H, Nk, d, dtype=dtype), v=_t(B, H, Nk, d, dtype=dtype),
                o=_t(B, H, Nq, d, dtype=dtype), lse=_t(B, H, Nq, dtype=F32))


def _bwd_args(B=1, H=2, Nq=200, Nk=None, d=64, dtype=BF):
    a = _fwd_args(B, H, Nq, Nk, d, dtype)
    a.update(dout=torch.zeros_like(a["q"]), dq=torch.zeros_like(a["q"]), dk=torch.zeros_like(a["k"]),
             dv=torch.zeros_like(a["v"]), workspace=_t(64, dtype=U8))
    return a


def _call_fwd(a, fn=fa.fa_fwd, **kw):
    fn(a["q"], a["k"], a["v"], a["o"], a["lse"], stream=S, **kw)


def _call_bwd(a, fn=fa.fa_bwd, **kw):
    fn(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"], a["workspace"], stream=S,
       **kw)


# ------------------------------------------------------------ host memory is refused
def test_cpu_tensors_are_refused_by_every_wrapper():
    a = _bwd_args()
    mask = _t(2, 2, dtype=U8)
    with pytest.raises(ValueError, match="CUDA"):
        _call_fwd(a)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_fwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["lse"], mask, stream=S)
    with pytest.raises(ValueError, match="CUDA"):
        _call_fwd(a, fa.fa_fwd_ex)
    for fn in (fa.fa_bwd, fa.fa_bwd_ex, fa.fa_bwd_deterministic):
        with pytest.raises(ValueError, match="CUDA"):
            _call_bwd(a, fn)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_bwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"],
                              a["workspace"], mask, stream=S)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_bwd_noalloc(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"], stream=S)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_fp8_quantize_qkv(a["q"], a["k"], a["v"], stream=S)
    q8 = _t(1, 2, 200, 128, dtype=U8)
    sc = _t(1, 2, 2, dtype=F32)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fa_fwd_fp8(q8, q8, q8, sc, sc, sc, _t(1, 2, 200, 128), _t(1, 2, 200, dtype=F32), stream=S)
    with pytest.raises(TypeError):
        fa.fa_fwd(None, a["k"], a["v"], a["o"], a["lse"], stream=S)


# ------------------------------------------------------------ accepted call patterns
def test_square_patterns_reach_the_library(fake):
    for d, dtype in ((64, BF), (128, F16), (256, BF)):
        a = _bwd_args(B=2, H=3, Nq=300, d=d, dtype=dtype)
        _call_fwd(a)
        _call_bwd(a)
        fa.fa_bwd_noalloc(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"], stream=S)
        mask = _t(3, 3, dtype=U8)
        fa.fa_fwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["lse"], mask, stream=S)
        fa.fa_bwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"],
                              a["workspace"], mask, stream=S)
    names = [c[0] for c in fake.calls]
    assert names.count("fa_fwd") == 3 and names.count("fa_bwd_blocksparse") == 3
    # every call carried as many arguments as the header declares
    from test_abi import declared_arity
    arity = declared_arity()
    assert all(n == arity[name] for name, n in fake.calls)


def test_general_patterns_reach_the_library(fake):
    # cross attention (Nq != Nk) with a window, ALiBi and a block mask, as the mode tests use them
    a = _bwd_args(B=1, H=4, Nq=300, Nk=700, d=128)
    mask = _t(3, 6, dtype=U8)
    slopes = _t(4, dtype=F32)
    _call_fwd(a, fa.fa_fwd_ex, window=(300, -1), alibi_slopes=slopes, block_mask=mask)
    _call_bwd(a, fa.fa_bwd_ex, window=(300, -1), alibi_slopes=slopes, block_mask=mask)
    _call_bwd(a, fa.fa_bwd_deterministic, block_mask=mask)
    o, lse = fa.attention_fwd(a["q"], a["k"], a["v"], causal=True, alibi_slopes=slopes, stream=S)
    assert o.shape == a["q"].shape and lse.shape == (1, 4, 300)
    dq, dk, dv = fa.attention_bwd(a["q"], a["k"], a["v"], o, a["dout"], lse, causal=True, stream=S,
                                  deterministic=True)
    assert dk.shape == a["k"].shape
    names = [c[0] for c in fake.calls]
    assert names.count("fa_fwd_ex") == 2 and "fa_bwd_deterministic_workspace_bytes" in names


def test_fp8_patterns_reach_the_library(fake):
    q = _t(1, 2, 300, 128)
    q8, k8, v8, sq, sk, sv = fa.fa_fp8_quantize_qkv(q, q.clone(), q.clone(), _t(128, dtype=F32), stream=S)
    assert q8.dtype == U8 and sq.shape == (1, 2, 3)
    fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, torch.zeros_like(q), _t(1, 2, 300, dtype=F32), True, stream=S)
    o, lse = fa.attention_fwd_fp8(q, q.clone(), q.clone(), stream=S)
    assert [c[0] for c in fake.calls].count("fa_fwd_fp8") == 2


def test_undersized_workspace_is_left_to_the_library(fake):
    # the library's own check reports FA_ERR_WORKSPACE; the binding does not pre-empt it
    a = _bwd_args()
    a["workspace"] = _t(1, dtype=U8)
    _call_bwd(a, fa.fa_bwd_deterministic)
    assert fake.calls[-1][0] == "fa_bwd_deterministic"


# ------------------------------------------------------------ refused call patterns
@pytest.mark.parametrize("bad", [
    "o_shape", "lse_numel", "lse_dtype", "k_dtype", "k_head_dim", "v_len", "k_len_square", "strided_q",
    "q_3d", "q_f32", "dk_shape", "dout_dtype", "mask_numel", "mask_dtype", "slopes_numel", "workspace_strided",
])
def test_malformed_calls_are_refused_before_the_library(fake, bad):
    a = _bwd_args(B=1, H=2, Nq=200, Nk=None, d=64)
    kw, fn = {}, fa.fa_bwd_ex
    if bad == "o_shape":
        a["o"] = _t(1, 2, 199, 64)
    elif bad == "lse_numel":
        a["lse"] = _t(1, 2, 199, dtype=F32)
    elif bad == "lse_dtype":
        a["lse"] = _t(1, 2, 200)
    elif bad == "k_dtype":
        a["k"] = _t(1, 2, 200, 64, dtype=F16)
    elif bad == "k_head_dim":
        a["k"] = _t(1, 2, 200, 128)
    elif bad == "v_len":
        a["v"] = _t(1, 2, 201, 64)
    elif bad == "k_len_square":
        a["k"], a["v"] = _t(1, 2, 300, 64), _t(1, 2, 300, 64)
        a["dk"], a["dv"] = _t(1, 2, 300, 64), _t(1, 2, 300, 64)
        fn = fa.fa_bwd                       # the square entry point needs Nk = Nq
    elif bad == "strided_q":
        a["q"] = _t(1, 2, 64, 200).transpose(2, 3)
    elif bad == "q_3d":
        a["q"] = _t(2, 200, 64)
    elif bad == "q_f32":
        a["q"] = _t(1, 2, 200, 64, dtype=F32)
    elif bad == "dk_shape":
        a["dk"] = _t(1, 2, 100, 64)
    elif bad == "dout_dtype":
        a["dout"] = _t(1, 2, 200, 64, dtype=F16)
    elif bad == "mask_numel":
        kw["block_mask"] = _t(2, 3, dtype=U8)
    elif bad == "mask_dtype":
        kw["block_mask"] = _t(2, 2, dtype=torch.bool)
    elif bad == "slopes_numel":
        kw["alibi_slopes"] = _t(3, dtype=F32)
    elif bad == "workspace_strided":
        a["workspace"] = _t(8, 8, dtype=U8)[:, ::2]
    with pytest.raises(ValueError):
        _call_bwd(a, fn, **kw)
    assert fake.calls == []


@pytest.mark.parametrize("bad", ["scale_numel", "code_dtype", "o_shape", "signs_numel"])
def test_malformed_fp8_calls_are_refused(fake, bad):
    q = _t(1, 2, 300, 128)
    q8, k8, v8 = (_t(1, 2, 300, 128, dtype=U8) for _ in range(3))
    sq, sk, sv = (_t(1, 2, 3, dtype=F32) for _ in range(3))
    o, lse = _t(1, 2, 300, 128), _t(1, 2, 300, dtype=F32)
    with pytest.raises(ValueError):
        if bad == "signs_numel":
            fa.fa_fp8_quantize_qkv(q, q.clone(), q.clone(), _t(64, dtype=F32), stream=S)
        else:
            if bad == "scale_numel":
                sk = _t(1, 2, 2, dtype=F32)
            elif bad == "code_dtype":
                v8 = _t(1, 2, 300, 128)
            elif bad == "o_shape":
                o = _t(1, 2, 300, 64)
            fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, stream=S)
    assert fake.calls == []
