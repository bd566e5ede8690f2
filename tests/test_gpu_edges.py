"""Edge cases of the launch geometry: one-dimensional grids beyond 65,535 CTAs
(the largest y/z extent), many (batch, head) pairs with tiny sequences, and
ALiBi head indexing with a large head count -- checked against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from flash_fwd_b200 import inputs
from parity import TOL_GRAD_REL, TOL_LSE, TOL_O, grad_norm

pytestmark = pytest.mark.gpu


def _grads_close(got, want):
    return np.abs(got - want).max() / grad_norm(np.abs(want).max()) <= TOL_GRAD_REL


@pytest.mark.parametrize("deterministic", [False, True])
def test_grid_beyond_65535_ctas_sampled(deterministic):
    # B=2 H=512 N=8192 d=64 causal: 65,536 key-block CTAs in the backward (and
    # 65,536 query-tile CTAs in the deterministic dQ pass), 32,768 in the forward
    import flash_fwd_b200 as fa
    B, H, N, d = 2, 512, 8192, 64
    q, k, v, do = inputs.make_qkv(B, H, N, d, "bf16", seed=11)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    scale = inputs.default_scale(d)
    o, lse = fa.attention_fwd(qd, kd, vd, causal=True, scale=scale)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=True, scale=scale, deterministic=deterministic)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    f = lambda t: t.reshape(B * H, N, d)   # noqa: E731
    for bh in (0, 511, 1023):
        rows = inputs.sample_rows(N, 6, 1, bh).numpy()
        sl = slice(bh, bh + 1)
        Q, K, V, DO = (f(t)[sl].double().numpy() for t in (q, k, v, do))
        r_o, r_l = oracle.fwd_rows(Q, K, V, scale, oracle.CAUSAL, rows=rows)
        assert np.abs(f(o)[bh, rows].double().cpu().numpy() - r_o[0]).max() <= TOL_O["bf16"]
        assert np.abs(lse.reshape(B * H, N)[bh, rows].cpu().numpy() - r_l[0]).max() <= TOL_LSE
        r_dq = oracle.bwd_dq_rows(Q, K, V, DO, scale, rows, oracle.CAUSAL)[0]
        r_dk, r_dv = oracle.bwd_dkdv_cols(Q, K, V, DO, scale, rows, oracle.CAUSAL)
        assert _grads_close(f(dq)[bh, rows].double().cpu().numpy(), r_dq)
        assert _grads_close(f(dk)[bh, rows].double().cpu().numpy(), r_dk[0])
        assert _grads_close(f(dv)[bh, rows].double().cpu().numpy(), r_dv[0])


def test_many_heads_tiny_sequences_with_alibi():
    # 65,536 (batch, head) pairs of 17 rows; ALiBi slopes over 1024 heads
    import flash_fwd_b200 as fa
    B, H, N, d = 64, 1024, 17, 64
    q, k, v, do = inputs.make_qkv(B, H, N, d, "f16", seed=12)
    slopes = inputs.alibi_slopes(H)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    scale = inputs.default_scale(d)
    o, lse = fa.attention_fwd(qd, kd, vd, causal=True, scale=scale, alibi_slopes=slopes.to(dev))
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=True, scale=scale,
                                  alibi_slopes=slopes.to(dev))
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    f = lambda t: t.reshape(B * H, N, d).double().cpu().numpy()   # noqa: E731
    ref = oracle.bwd_full(f(q), f(k), f(v), f(do), scale, oracle.CAUSAL, slopes=slopes.double().numpy())
    assert np.abs(f(o) - ref[0]).max() <= TOL_O["f16"]
    assert np.abs(lse.reshape(B * H, N).double().cpu().numpy() - ref[1]).max() <= TOL_LSE
    for got, want in ((dq, ref[2]), (dk, ref[3]), (dv, ref[4])):
        assert _grads_close(f(got), want)
