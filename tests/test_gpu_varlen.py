"""Parity of the packed variable-length entry points (fa_fwd_varlen /
fa_bwd_varlen) with the fp64 oracle (oracle.fwd_varlen / bwd_varlen): B
sequences of different lengths, including empty ones, single rows, exact
tile multiples and ragged tails, concatenated along the token axis, in every
mask mode, both 16-bit types and every head dim, for the default and the
deterministic backward.  Every element of O, LSE, dQ, dK, dV is compared; a
sequence's partial last tile must not touch the rows of the sequence after
it.
"""
import numpy as np
import pytest
import torch

import oracle
from flash_fwd_b200 import inputs
from parity import TOL_GRAD_REL, TOL_LSE, TOL_O, grad_norm

pytestmark = pytest.mark.gpu

SELF = [300, 1, 0, 128, 129, 517, 255]
CROSS = [200, 5, 17, 0, 384, 517, 256]


def _gpu(cu_q, cu_k, q, k, v, do, causal, scale, window=None, slopes=None, bwd=True):
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    cq, ck, qd, kd, vd, dod = (t.to(dev) for t in (cu_q, cu_k, q, k, v, do))
    sl = None if slopes is None else slopes.to(dev)
    mq = int((cu_q[1:] - cu_q[:-1]).max())
    mk = max(int((cu_k[1:] - cu_k[:-1]).max()), 1)
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cq, ck, mq, mk, causal=causal, scale=scale, window=window,
                                     alibi_slopes=sl)
    out = [o, lse]
    if bwd:
        out += list(fa.attention_bwd_varlen(qd, kd, vd, o, dod, lse, cq, ck, mq, mk, causal=causal, scale=scale,
                                            window=window, alibi_slopes=sl))
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return [t.cpu() for t in out]


def _check(got, ref, dtype):
    f = lambda t: t.double().numpy()   # noqa: E731
    o, lse = f(got[0]), f(got[1])
    r_o, r_lse = ref[0], ref[1]
    assert np.isfinite(o).all()
    assert np.abs(o - r_o).max() <= TOL_O[dtype]
    hidden = np.isinf(r_lse)
    np.testing.assert_array_equal(lse[hidden], -np.inf)
    if (~hidden).any():
        assert np.abs(lse[~hidden] - r_lse[~hidden]).max() <= TOL_LSE
    if len(got) > 2:
        for name, g, r in zip(("dq", "dk", "dv"), got[2:], ref[2:]):
            g = f(g)
            assert np.isfinite(g).all(), name
            err = np.abs(g - r).max() / grad_norm(np.abs(r).max())
            assert err <= TOL_GRAD_REL, (name, err)


MODES = {
    "dense": dict(causal=False),
    "causal": dict(causal=True),
    "window": dict(causal=False, window=(96, 40)),
    "causal_window": dict(causal=True, window=(200, -1)),
    "alibi": dict(causal=True, alibi=True),
}


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("cross", [False, True])
def test_varlen_fwd_bwd(d, dtype, mode, cross):
    H = 3
    lk = CROSS if cross else SELF
    cu_q, cu_k, q, k, v, do = inputs.make_varlen(SELF, lk, H, d, dtype, seed=d + len(mode) + 7 * cross)
    m = MODES[mode]
    slopes = inputs.alibi_slopes(H) if m.get("alibi") else None
    scale = inputs.default_scale(d)
    got = _gpu(cu_q, cu_k, q, k, v, do, m["causal"], scale, m.get("window"), slopes)
    ref = oracle.bwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                            cu_q.numpy(), cu_k.numpy(), scale, oracle.CAUSAL if m["causal"] else 0,
                            window=m.get("window"), slopes=None if slopes is None else slopes.double().numpy())
    _check(got, [ref[0], ref[1], ref[2], ref[3], ref[4]], dtype)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cross", [False, True])
def test_varlen_fwd_d256(causal, cross):
    H, d = 2, 256
    lk = CROSS if cross else SELF
    cu_q, cu_k, q, k, v, do = inputs.make_varlen(SELF, lk, H, d, "bf16", seed=11 + cross)
    scale = inputs.default_scale(d)
    got = _gpu(cu_q, cu_k, q, k, v, do, causal, scale, bwd=False)
    ref = oracle.fwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(), cu_q.numpy(),
                            cu_k.numpy(), scale, oracle.CAUSAL if causal else 0)
    _check(got, list(ref), "bf16")


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_long_mixed_lengths(d):
    """Sequences up to 2,048 rows, many tiles each, causal: every element."""
    H = 4
    lengths = [1500, 700, 2048, 33, 1024, 129]
    cu_q, cu_k, q, k, v, do = inputs.make_varlen(lengths, lengths, H, d, "bf16", seed=5)
    scale = inputs.default_scale(d)
    got = _gpu(cu_q, cu_k, q, k, v, do, True, scale)
    ref = oracle.bwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                            cu_q.numpy(), cu_k.numpy(), scale, oracle.CAUSAL)
    _check(got, list(ref), "bf16")


def test_varlen_equal_lengths_match_batched_entry_points():
    """Equal lengths: the packed call gives what the general batched forward
    gives on the [B, H, N, d] transpose of the same data, bit for bit (the
    same tiles in the same order; window (-1, -1) selects that kernel)."""
    import flash_fwd_b200 as fa
    B, N, H, d = 3, 300, 4, 128
    cu_q, cu_k, q, k, v, do = inputs.make_varlen([N] * B, [N] * B, H, d, "bf16", seed=3)
    got = _gpu(cu_q, cu_k, q, k, v, do, True, inputs.default_scale(d))
    dev = torch.device("cuda:0")
    bhnd = lambda x: x.reshape(B, N, H, d).transpose(1, 2).contiguous().to(dev)   # noqa: E731
    o, lse = fa.attention_fwd(bhnd(q), bhnd(k), bhnd(v), causal=True, window=(-1, -1))
    torch.cuda.synchronize()
    assert torch.equal(bhnd(got[0]).cpu(), o.cpu())
    assert torch.equal(got[1].reshape(H, B, N).transpose(0, 1).contiguous(), lse.cpu())


@pytest.mark.parametrize("mode", ["dense", "causal", "window", "alibi"])
@pytest.mark.parametrize("cross", [False, True])
def test_varlen_fwd_bwd_d256(mode, cross):
    H, d = 2, 256
    lk = CROSS if cross else SELF
    cu_q, cu_k, q, k, v, do = inputs.make_varlen(SELF, lk, H, d, "bf16", seed=21 + 3 * cross + len(mode))
    m = MODES[mode]
    slopes = inputs.alibi_slopes(H) if m.get("alibi") else None
    scale = inputs.default_scale(d)
    got = _gpu(cu_q, cu_k, q, k, v, do, m["causal"], scale, m.get("window"), slopes)
    ref = oracle.bwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                            cu_q.numpy(), cu_k.numpy(), scale, oracle.CAUSAL if m["causal"] else 0,
                            window=m.get("window"), slopes=None if slopes is None else slopes.double().numpy())
    _check(got, list(ref), "bf16")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("mode", ["dense", "causal", "causal_window"])
@pytest.mark.parametrize("cross", [False, True])
def test_varlen_deterministic(d, mode, cross):
    """fa_bwd_varlen_deterministic: the oracle's gradients, identical bytes on
    a repeated call, and the same dK, dV bytes as the default backward."""
    import flash_fwd_b200 as fa
    H = 2
    lk = CROSS if cross else SELF
    cu_q, cu_k, q, k, v, do = inputs.make_varlen(SELF, lk, H, d, "bf16", seed=31 + d + len(mode) + 5 * cross)
    m = MODES[mode]
    scale = inputs.default_scale(d)
    dev = torch.device("cuda:0")
    cq, ck, qd, kd, vd, dod = (t.to(dev) for t in (cu_q, cu_k, q, k, v, do))
    mq = int((cu_q[1:] - cu_q[:-1]).max())
    mk = int((cu_k[1:] - cu_k[:-1]).max())
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cq, ck, mq, mk, causal=m["causal"], scale=scale,
                                     window=m.get("window"))
    args = (qd, kd, vd, o, dod, lse, cq, ck, mq, mk)
    kw = dict(causal=m["causal"], scale=scale, window=m.get("window"))
    g1 = fa.attention_bwd_varlen(*args, deterministic=True, **kw)
    g2 = fa.attention_bwd_varlen(*args, deterministic=True, **kw)
    g0 = fa.attention_bwd_varlen(*args, **kw)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    assert torch.equal(g1[1], g0[1]) and torch.equal(g1[2], g0[2])
    ref = oracle.bwd_varlen(q.double().numpy(), k.double().numpy(), v.double().numpy(), do.double().numpy(),
                            cu_q.numpy(), cu_k.numpy(), scale, oracle.CAUSAL if m["causal"] else 0,
                            window=m.get("window"))
    _check([o.cpu(), lse.cpu()] + [t.cpu() for t in g1], list(ref), "bf16")


def test_varlen_bad_lengths_are_clamped_and_reported():
    """Cumulative lengths that decrease, or exceed max_seqlen, are clamped by
    the kernels (nothing outside the buffers is touched) and reported as
    FA_ERR_INVALID_ARG through the device status word."""
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    cu_q, cu_k, q, k, v, do = inputs.make_varlen([100, 200], [100, 200], 2, 64, "bf16")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    bad = torch.tensor([0, 250, 200], dtype=torch.int32, device=dev)       # decreasing
    fa.attention_fwd_varlen(qd, kd, vd, bad, bad, 200, 200)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 1
    fa.attention_fwd_varlen(qd, kd, vd, cu_q.to(dev), cu_k.to(dev), 150, 150)   # 200 > max_seqlen
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 1
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cu_q.to(dev), cu_k.to(dev), 200, 200)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
