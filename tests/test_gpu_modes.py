"""Parity of the general entry points (fa_fwd_ex / fa_bwd_ex) with the fp64
oracle: query and key lengths that differ (cross attention, bottom-right
aligned), sliding windows and ALiBi -- the built-in mask modes of
"深度解析" section 五 -- alone and combined with causal and block-sparse
masks, over every head dim and both 16-bit types, with ragged tails.
Every element of O, LSE, dQ, dK, dV is compared; rows that see no key must
come back as O = 0, LSE = -inf and zero gradients.
"""
import numpy as np
import pytest
import torch

import oracle
from flash_fwd_b200 import inputs
from parity import TOL_GRAD_REL, TOL_LSE, TOL_O, grad_norm

pytestmark = pytest.mark.gpu


def _run(q, k, v, do, causal, scale, window=None, slopes=None, mask=None):
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    sl = None if slopes is None else slopes.to(dev)
    md = None if mask is None else mask.to(dev)
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, scale=scale, block_mask=md, window=window,
                              alibi_slopes=sl)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale, block_mask=md,
                                  window=window, alibi_slopes=sl)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return [t.cpu() for t in (o, lse, dq, dk, dv)]


def _check(got, q, k, v, do, causal, scale, dtype, window=None, slopes=None, mask=None):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    f = lambda t, n: t.reshape(B * H, n, d).double().numpy()   # noqa: E731
    flags = (oracle.CAUSAL if causal else 0) | (oracle.SPARSE if mask is not None else 0)
    ref = oracle.bwd_full(f(q, Nq), f(k, Nk), f(v, Nk), f(do, Nq), scale, flags,
                          None if mask is None else mask.numpy(), 128, window=window,
                          slopes=None if slopes is None else slopes.double().numpy())
    o, lse, dq, dk, dv = got
    o, dq = f(o, Nq), f(dq, Nq)
    dk, dv = f(dk, Nk), f(dv, Nk)
    lse = lse.reshape(B * H, Nq).double().numpy()
    r_o, r_lse, r_dq, r_dk, r_dv = ref
    for x in (o, dq, dk, dv):
        assert np.isfinite(x).all()
    assert np.abs(o - r_o).max() <= TOL_O[dtype]
    hidden = np.isinf(r_lse)
    np.testing.assert_array_equal(lse[hidden], -np.inf)
    if (~hidden).any():
        assert np.abs(lse[~hidden] - r_lse[~hidden]).max() <= TOL_LSE
    for name, g, r in (("dq", dq, r_dq), ("dk", dk, r_dk), ("dv", dv, r_dv)):
        err = np.abs(g - r).max() / grad_norm(np.abs(r).max())
        assert err <= TOL_GRAD_REL, (name, err)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(100, 300), (300, 100), (129, 257), (1, 513), (257, 1)])
def test_cross_attention(nq, nk, causal, d):
    q, k, v, do = inputs.make_qkv_cross(1, 2, nq, nk, d, "bf16", seed=nq + 3 * nk + d)
    scale = inputs.default_scale(d)
    got = _run(q, k, v, do, causal, scale)
    _check(got, q, k, v, do, causal, scale, "bf16")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("window,causal", [((64, 0), False), ((100, 50), False), ((0, 0), False),
                                           ((200, -1), False), ((-1, 37), False), ((150, 10), True)])
def test_sliding_window(window, causal, d):
    N = 500
    q, k, v, do = inputs.make_qkv(1, 2, N, d, "bf16", seed=11 + d)
    scale = inputs.default_scale(d)
    got = _run(q, k, v, do, causal, scale, window=window)
    _check(got, q, k, v, do, causal, scale, "bf16", window=window)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_alibi(causal, d, dtype):
    N, H = 300, 3
    q, k, v, do = inputs.make_qkv(1, H, N, d, dtype, seed=21 + d)
    scale = inputs.default_scale(d)
    slopes = inputs.alibi_slopes(H)
    got = _run(q, k, v, do, causal, scale, slopes=slopes)
    _check(got, q, k, v, do, causal, scale, dtype, slopes=slopes)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_everything_combined(d):
    # cross attention + window + ALiBi + block-sparse mask + causal
    nq, nk, H = 400, 700, 2
    q, k, v, do = inputs.make_qkv_cross(1, H, nq, nk, d, "bf16", seed=5 + d)
    g = torch.Generator().manual_seed(9)
    mask = (torch.rand(((nq + 127) // 128, (nk + 127) // 128), generator=g) < 0.7).to(torch.uint8)
    scale = inputs.default_scale(d)
    slopes = inputs.alibi_slopes(H)
    got = _run(q, k, v, do, True, scale, window=(300, -1), slopes=slopes, mask=mask)
    _check(got, q, k, v, do, True, scale, "bf16", window=(300, -1), slopes=slopes, mask=mask)


def test_long_cross_attention_sampled():
    # B=2 H=4 Nq=1024 Nk=4096 d=128 causal: a decoder chunk against a longer context
    B, H, nq, nk, d = 2, 4, 1024, 4096, 128
    q, k, v, do = inputs.make_qkv_cross(B, H, nq, nk, d, "bf16", seed=77)
    scale = inputs.default_scale(d)
    o, lse, dq, dk, dv = _run(q, k, v, do, True, scale)
    f = lambda t, n: t.reshape(B * H, n, d).double().numpy()   # noqa: E731
    Q, K, V, DO = f(q, nq), f(k, nk), f(v, nk), f(do, nq)
    rows = np.array([0, 1, 511, 777, 1023], dtype=np.int32)
    cols = np.array([0, 2000, 3071, 3072, 4095], dtype=np.int32)
    for h in (0, 5):
        sl = slice(h, h + 1)
        r_o, r_l = oracle.fwd_rows(Q[sl], K[sl], V[sl], scale, oracle.CAUSAL, rows=rows)
        assert np.abs(f(o, nq)[h, rows] - r_o[0]).max() <= TOL_O["bf16"]
        assert np.abs(lse.reshape(B * H, nq).double().numpy()[h, rows] - r_l[0]).max() <= TOL_LSE
        r_dq = oracle.bwd_dq_rows(Q[sl], K[sl], V[sl], DO[sl], scale, rows, oracle.CAUSAL)[0]
        r_dk, r_dv = oracle.bwd_dkdv_cols(Q[sl], K[sl], V[sl], DO[sl], scale, cols, oracle.CAUSAL)
        for g, r in ((f(dq, nq)[h, rows], r_dq), (f(dk, nk)[h, cols], r_dk[0]), (f(dv, nk)[h, cols], r_dv[0])):
            assert np.abs(g - r).max() / grad_norm(np.abs(r).max()) <= TOL_GRAD_REL


@pytest.mark.parametrize("name", ["window128", "cross128", "alibi128"])
def test_bench_workloads_sampled(name):
    # the general workloads bench.py times, at their full size, on sampled rows and keys
    w = dict(window128=dict(B=4, H=16, Nq=4096, Nk=4096, window=(1024, 0), alibi=False),
             cross128=dict(B=4, H=16, Nq=1024, Nk=8192, window=None, alibi=False),
             alibi128=dict(B=4, H=16, Nq=4096, Nk=4096, window=None, alibi=True))[name]
    B, H, nq, nk, d = w["B"], w["H"], w["Nq"], w["Nk"], 128
    q, k, v, do = inputs.make_qkv_cross(B, H, nq, nk, d, "bf16", seed=0)
    scale = inputs.default_scale(d)
    slopes = inputs.alibi_slopes(H) if w["alibi"] else None
    o, lse, dq, dk, dv = _run(q, k, v, do, True, scale, window=w["window"], slopes=slopes)
    f = lambda t, n: t.reshape(B * H, n, d).double().numpy()   # noqa: E731
    Q, K, V, DO = f(q, nq), f(k, nk), f(v, nk), f(do, nq)
    O, L = f(o, nq), lse.reshape(B * H, nq).double().numpy()
    dQ, dK, dV = f(dq, nq), f(dk, nk), f(dv, nk)
    for bh in (0, 37, 63):
        rows = inputs.sample_rows(nq, 8, 0, bh).numpy()
        cols = inputs.sample_rows(nk, 8, 7, bh).numpy()
        sl = slice(bh, bh + 1)
        kw = dict(window=w["window"], slopes=None if slopes is None else slopes[bh % H:bh % H + 1].double().numpy())
        r_o, r_l = oracle.fwd_rows(Q[sl], K[sl], V[sl], scale, oracle.CAUSAL, rows=rows, **kw)
        assert np.abs(O[bh, rows] - r_o[0]).max() <= TOL_O["bf16"]
        assert np.abs(L[bh, rows] - r_l[0]).max() <= TOL_LSE
        r_dq = oracle.bwd_dq_rows(Q[sl], K[sl], V[sl], DO[sl], scale, rows, oracle.CAUSAL, **kw)[0]
        r_dk, r_dv = oracle.bwd_dkdv_cols(Q[sl], K[sl], V[sl], DO[sl], scale, cols, oracle.CAUSAL, **kw)
        for g, r in ((dQ[bh, rows], r_dq), (dK[bh, cols], r_dk[0]), (dV[bh, cols], r_dv[0])):
            assert np.abs(g - r).max() / grad_norm(np.abs(r).max()) <= TOL_GRAD_REL
