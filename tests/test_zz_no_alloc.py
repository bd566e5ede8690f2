"""fa_bwd_noalloc: the backward entry point for callers that cannot allocate.

Some callers only receive input and output buffers (a plugin or custom-op
interface with no allocator), or must keep cudaMalloc off their path; for them
fa_bwd_noalloc takes no workspace and uses scratch the library keeps in device
memory.  These tests call it through the C ABI and check that two calls in a
row match fa_bwd's results on the same inputs and the fp64 oracle's
gradients, and that a problem too large for the built-in scratch is refused
before anything runs.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

import flash_fwd_b200 as fa
from flash_fwd_b200 import inputs
from parity import TOL_GRAD_REL, check_bwd, grad_norm

pytestmark = pytest.mark.gpu

FA_ERR_SCRATCH_LIMIT = 7
SCRATCH_BYTES = 32 * 1024 * 1024


def _noalloc_fn():
    lib = fa.load_library()
    fn = lib.fa_bwd_noalloc
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [vp] * 9 + [i, i, i, i, f, i, i, vp]
    fn.restype = ctypes.c_int
    return fn


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(t, causal, scale, dtype_code):
    B, H, N, d = t["q"].shape
    dq, dk, dv = (torch.full_like(t["q"], float("nan")) for _ in range(3))
    rc = _noalloc_fn()(_p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["o"]), _p(t["do"]), _p(t["lse"]),
                       _p(dq), _p(dk), _p(dv), B, H, N, d, scale, int(causal), dtype_code,
                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, fa.fa_status_string(rc)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return dq, dk, dv


def _close(a, b):
    a, b = a.float(), b.float()
    return (a - b).abs().max().item() <= TOL_GRAD_REL * grad_norm(b.abs().max().item())


@pytest.mark.parametrize("B,H,N,d,dtype,causal", [
    (2, 4, 1000, 128, "bf16", True),
    (1, 3, 777, 64, "f16", False),
    (1, 2, 300, 256, "bf16", True),
])
def test_noalloc_matches_fa_bwd_twice(B, H, N, d, dtype, causal):
    assert fa.fa_bwd_workspace_bytes(B, H, N, d) <= SCRATCH_BYTES
    q, k, v, do = inputs.make_qkv(B, H, N, d, dtype, seed=21)
    dev = torch.device("cuda:0")
    t = {n: x.to(dev) for n, x in (("q", q), ("k", k), ("v", v), ("do", do))}
    scale = inputs.default_scale(d)
    t["o"], t["lse"] = fa.attention_fwd(t["q"], t["k"], t["v"], causal=causal, scale=scale)
    ref = fa.attention_bwd(t["q"], t["k"], t["v"], t["o"], t["do"], t["lse"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    code = 1 if dtype == "bf16" else 0
    first = _call_noalloc(t, causal, scale, code)
    second = _call_noalloc(t, causal, scale, code)
    for got in (first, second):
        for g, r in zip(got, ref):
            assert torch.isfinite(g.float()).all()
            assert _close(g, r)
        # dK and dV are accumulated without atomics: identical to fa_bwd
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
        # and every element against the fp64 oracle's gradients
        check_bwd(tuple(g.cpu() for g in got), q, k, v, do, causal, scale)


def test_noalloc_refuses_problems_beyond_its_scratch():
    B, H, N, d = 4, 16, 4096, 128        # needs ~269 MB of scratch
    assert fa.fa_bwd_workspace_bytes(B, H, N, d) > SCRATCH_BYTES
    # null buffers: the refusal comes before any launch; were the size check
    # ever moved behind the buffer checks, the call would still launch nothing
    # (FA_ERR_INVALID_ARG) instead of running over buffers of the wrong size
    null = ctypes.c_void_p(None)
    rc = _noalloc_fn()(*([null] * 9), B, H, N, d, 0.088, 1, 1, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == FA_ERR_SCRATCH_LIMIT
    assert "scratch" in fa.fa_status_string(rc)
