"""The deterministic backward (fa_bwd_deterministic): parity of dQ, dK, dV
with the fp64 oracle in every mode the general entry points take (square,
causal, cross attention, sliding windows, ALiBi, block-sparse masks) over
every head dim and both 16-bit types, and bitwise reproducibility: repeated
calls return identical bytes, and its dK, dV are the bytes the default
backward returns (the same key-block kernel computes them).
"""
import numpy as np
import pytest
import torch

import oracle
from flash_fwd_b200 import inputs
from parity import TOL_GRAD_REL, check_bwd, grad_norm

pytestmark = pytest.mark.gpu


def _fwd(qd, kd, vd, causal, scale, window=None, slopes=None, mask=None):
    import flash_fwd_b200 as fa
    return fa.attention_fwd(qd, kd, vd, causal=causal, scale=scale, block_mask=mask, window=window,
                            alibi_slopes=slopes)


def _det(qd, kd, vd, o, dod, lse, causal, scale, window=None, slopes=None, mask=None):
    import flash_fwd_b200 as fa
    g = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale, block_mask=mask, window=window,
                         alibi_slopes=slopes, deterministic=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return g


def _run(q, k, v, do, causal, scale, window=None, slopes=None, mask=None):
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    sl = None if slopes is None else slopes.to(dev)
    md = None if mask is None else mask.to(dev)
    o, lse = _fwd(qd, kd, vd, causal, scale, window, sl, md)
    return [t.cpu() for t in _det(qd, kd, vd, o, dod, lse, causal, scale, window, sl, md)]


def _check(grads, q, k, v, do, causal, scale, window=None, slopes=None, mask=None):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    f = lambda t, n: t.reshape(B * H, n, d).double().numpy()   # noqa: E731
    flags = (oracle.CAUSAL if causal else 0) | (oracle.SPARSE if mask is not None else 0)
    ref = oracle.bwd_full(f(q, Nq), f(k, Nk), f(v, Nk), f(do, Nq), scale, flags,
                          None if mask is None else mask.numpy(), 128, window=window,
                          slopes=None if slopes is None else slopes.double().numpy())
    dq, dk, dv = grads
    for name, g, r in (("dq", f(dq, Nq), ref[2]), ("dk", f(dk, Nk), ref[3]), ("dv", f(dv, Nk), ref[4])):
        assert np.isfinite(g).all(), name
        err = np.abs(g - r).max() / grad_norm(np.abs(r).max())
        assert err <= TOL_GRAD_REL, (name, err)


@pytest.mark.parametrize("N", [1, 129, 300])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_det_small(N, d, dtype, causal):
    q, k, v, do = inputs.make_qkv(1, 2, N, d, dtype, seed=300 + N + d)
    scale = inputs.default_scale(d)
    grads = _run(q, k, v, do, causal, scale)
    check_bwd(grads, q, k, v, do, causal, scale)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("nq,nk,causal", [(100, 300, True), (300, 100, False), (1, 513, True), (257, 1, False),
                                          (129, 700, False)])
def test_det_cross_attention(nq, nk, causal, d):
    q, k, v, do = inputs.make_qkv_cross(1, 2, nq, nk, d, "bf16", seed=nq + 5 * nk + d)
    scale = inputs.default_scale(d)
    _check(_run(q, k, v, do, causal, scale), q, k, v, do, causal, scale)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("window,causal", [((100, 50), False), ((0, 0), False), ((150, 10), True),
                                           ((-1, 37), False)])
def test_det_sliding_window(window, causal, d):
    q, k, v, do = inputs.make_qkv(1, 2, 500, d, "bf16", seed=13 + d)
    scale = inputs.default_scale(d)
    _check(_run(q, k, v, do, causal, scale, window=window), q, k, v, do, causal, scale, window=window)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_det_alibi_sparse_combined(d, dtype):
    # cross attention + window + ALiBi + block-sparse mask + causal
    nq, nk, H = 400, 700, 2
    q, k, v, do = inputs.make_qkv_cross(1, H, nq, nk, d, dtype, seed=7 + d)
    g = torch.Generator().manual_seed(3)
    mask = (torch.rand(((nq + 127) // 128, (nk + 127) // 128), generator=g) < 0.7).to(torch.uint8)
    scale = inputs.default_scale(d)
    slopes = inputs.alibi_slopes(H)
    grads = _run(q, k, v, do, True, scale, window=(300, -1), slopes=slopes, mask=mask)
    _check(grads, q, k, v, do, True, scale, window=(300, -1), slopes=slopes, mask=mask)


def test_det_empty_mask_column_and_row():
    # key block 1 is seen by no query block and query block 1 sees nothing:
    # the dQ pass has a tile with no key block and must still write zeros
    N, d = 384, 128
    q, k, v, do = inputs.make_qkv(1, 1, N, d, "bf16", seed=4)
    mask = torch.ones((3, 3), dtype=torch.uint8)
    mask[:, 1] = 0
    mask[1, :] = 0
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    md = mask.to(dev)
    o, lse = _fwd(qd, kd, vd, False, 0.125, mask=md)
    import flash_fwd_b200 as fa
    B, H = 1, 1
    dq = torch.full_like(qd, float("nan"))   # poisoned: every element must be written
    dk, dv = torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(fa.fa_bwd_deterministic_workspace_bytes(B, H, N, N, d), dtype=torch.uint8, device=dev)
    fa.fa_bwd_deterministic(qd, kd, vd, o, dod, lse, dq, dk, dv, ws, False, 0.125, block_mask=md)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    assert torch.all(dq[0, 0, 128:256] == 0)
    assert torch.all(dk[0, 0, 128:256] == 0) and torch.all(dv[0, 0, 128:256] == 0)
    check_bwd((dq, dk, dv), q, k, v, do, False, 0.125, mask=mask)


@pytest.mark.parametrize("d,causal", [(64, True), (128, True), (128, False), (256, True)])
def test_det_bitwise_reproducible(d, causal):
    import flash_fwd_b200 as fa
    B, H, N = 2, 4, 2000
    q, k, v, do = inputs.make_qkv(B, H, N, d, "bf16", seed=40 + d)
    scale = inputs.default_scale(d)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = _fwd(qd, kd, vd, causal, scale)
    runs = [_det(qd, kd, vd, o, dod, lse, causal, scale) for _ in range(3)]
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)
    # dK, dV: the same bytes as the default backward; dQ: equal up to the
    # summation order of the default backward's atomics
    dq_a, dk_a, dv_a = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(dk_a, runs[0][1]) and torch.equal(dv_a, runs[0][2])
    diff = (dq_a.float() - runs[0][0].float()).abs().max().item()
    assert diff <= 2e-2 * grad_norm(dq_a.float().abs().max().item())


def test_det_workspace_and_errors():
    import flash_fwd_b200 as fa
    B, H, Nq, Nk, d = 2, 3, 300, 500, 128
    # two fp32 statistics per padded query row, no dQ accumulator
    assert fa.fa_bwd_deterministic_workspace_bytes(B, H, Nq, Nk, d) == 2 * B * H * 384 * 4
    assert fa.fa_bwd_deterministic_workspace_bytes(B, H, Nq, Nk, 96) == 0
    q, k, v, do = inputs.make_qkv_cross(B, H, Nq, Nk, d, "bf16", seed=1)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = _fwd(qd, kd, vd, False, 0.1)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    small = torch.empty(fa.fa_bwd_deterministic_workspace_bytes(B, H, Nq, Nk, d) - 16, dtype=torch.uint8,
                        device=dev)
    with pytest.raises(fa.FaError) as e:
        fa.fa_bwd_deterministic(qd, kd, vd, o, dod, lse, dq, dk, dv, small, False, 0.1)
    assert "workspace" in str(e.value)
