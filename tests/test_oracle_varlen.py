"""Pins for the oracle's packed variable-length batches (oracle.fwd_varlen,
oracle.bwd_varlen), against a formulation that shares nothing with it: one
softmax per head over ALL packed keys, with a block-diagonal visibility mask
(query t keeps key s only when both lie in the same sequence and s is visible
from t inside it, bottom-right aligned per sequence), in plain numpy for the
forward and in torch autograd (fp64) for the gradients.  A slicing mistake
(wrong offsets, cu_q used for keys, one sequence's alignment applied to
another, a dropped empty sequence) changes which keys a row sees and fails
these comparisons.  Also: isolation (changing one sequence leaves the others
bit-identical) and the empty-sequence conventions.
"""
import numpy as np
import pytest
import torch

import oracle

rng = np.random.default_rng(2718)


def _packed_mask(cu_q, cu_k, causal, window):
    """[total_q, total_k] bool visibility and the relative key offset rel = s_pos - (t_pos + Nk_b - Nq_b)."""
    cu_q, cu_k = np.asarray(cu_q), np.asarray(cu_k)
    tq, tk = cu_q[-1], cu_k[-1]
    sq = np.searchsorted(cu_q, np.arange(tq), side="right") - 1
    sk = np.searchsorted(cu_k, np.arange(tk), side="right") - 1
    pos_q = np.arange(tq) - cu_q[sq]
    pos_k = np.arange(tk) - cu_k[sk]
    off = (cu_k[1:] - cu_k[:-1]) - (cu_q[1:] - cu_q[:-1])
    rel = pos_k[None, :] - (pos_q[:, None] + off[sq][:, None])
    keep = sq[:, None] == sk[None, :]
    if causal:
        keep &= rel <= 0
    if window is not None:
        wl, wr = window
        if wl >= 0:
            keep &= rel >= -wl
        if wr >= 0:
            keep &= rel <= wr
    return keep, rel


def _block_diag_fwd(q, k, v, cu_q, cu_k, scale, causal=False, window=None, slopes=None):
    keep, rel = _packed_mask(cu_q, cu_k, causal, window)
    s = scale * np.einsum("thd,shd->hts", q, k)
    if slopes is not None:
        s = s - np.asarray(slopes)[:, None, None] * np.abs(rel)[None]
    s = np.where(keep[None], s, -np.inf)
    m = s.max(axis=2, keepdims=True)
    seen = np.isfinite(m)
    p = np.where(keep[None], np.exp(s - np.where(seen, m, 0.0)), 0.0)
    l = p.sum(axis=2, keepdims=True)
    o = np.einsum("hts,shd->thd", p / np.where(seen, l, 1.0), v)
    lse = np.where(seen[..., 0], (m + np.log(np.where(seen, l, 1.0)))[..., 0], -np.inf)
    return o, lse


def _block_diag_grads(q, k, v, do, cu_q, cu_k, scale, causal=False, window=None, slopes=None):
    keep, rel = _packed_mask(cu_q, cu_k, causal, window)
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = scale * torch.einsum("thd,shd->hts", qt, kt)
    if slopes is not None:
        s = s - torch.tensor(np.asarray(slopes), dtype=torch.float64)[:, None, None] * torch.tensor(np.abs(rel))[None]
    kp = torch.tensor(keep)[None]
    s = torch.where(kp, s, torch.full_like(s, -1e300))
    p = torch.softmax(s, dim=2) * kp            # rows with no visible key: all zero
    o = torch.einsum("hts,shd->thd", p, vt)
    (o * torch.tensor(do)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


CASES = [
    # (q lengths, k lengths): self attention, cross attention with empty
    # sequences, longer queries than keys (rows that see nothing under causal)
    ([5, 0, 9, 1, 12], [5, 0, 9, 1, 12]),
    ([4, 7, 0, 3, 6], [9, 2, 5, 0, 6]),
    ([11, 2], [3, 8]),
]


def _make(lq, lk, H=2, d=8):
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int64)
    q = rng.standard_normal((cu_q[-1], H, d))
    k = rng.standard_normal((cu_k[-1], H, d))
    v = rng.standard_normal((cu_k[-1], H, d))
    do = rng.standard_normal((cu_q[-1], H, d))
    return cu_q, cu_k, q, k, v, do


@pytest.mark.parametrize("lq,lk", CASES)
@pytest.mark.parametrize("mode", ["dense", "causal", "window", "alibi"])
def test_fwd_matches_block_diagonal(lq, lk, mode):
    cu_q, cu_k, q, k, v, _ = _make(lq, lk)
    kw = dict(causal=mode in ("causal", "alibi"), window=(2, 1) if mode == "window" else None,
              slopes=[0.3, 0.05] if mode == "alibi" else None)
    o_ref, lse_ref = _block_diag_fwd(q, k, v, cu_q, cu_k, 0.37, **kw)
    o, lse = oracle.fwd_varlen(q, k, v, cu_q, cu_k, 0.37, oracle.CAUSAL if kw["causal"] else 0,
                               window=kw["window"], slopes=kw["slopes"])
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref))
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(lse[fin], lse_ref[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("lq,lk", CASES)
@pytest.mark.parametrize("mode", ["dense", "causal", "window", "alibi"])
def test_bwd_matches_autograd_block_diagonal(lq, lk, mode):
    cu_q, cu_k, q, k, v, do = _make(lq, lk)
    kw = dict(causal=mode in ("causal", "alibi"), window=(2, 1) if mode == "window" else None,
              slopes=[0.3, 0.05] if mode == "alibi" else None)
    dq_ref, dk_ref, dv_ref = _block_diag_grads(q, k, v, do, cu_q, cu_k, 0.37, **kw)
    o, lse, dq, dk, dv = oracle.bwd_varlen(q, k, v, do, cu_q, cu_k, 0.37, oracle.CAUSAL if kw["causal"] else 0,
                                           window=kw["window"], slopes=kw["slopes"])
    for got, want in ((dq, dq_ref), (dk, dk_ref), (dv, dv_ref)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)
    o2, lse2 = oracle.fwd_varlen(q, k, v, cu_q, cu_k, 0.37, oracle.CAUSAL if kw["causal"] else 0,
                                 window=kw["window"], slopes=kw["slopes"])
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_sequences_are_isolated():
    cu_q, cu_k, q, k, v, _ = _make([6, 10, 3], [6, 10, 3])
    o, lse = oracle.fwd_varlen(q, k, v, cu_q, cu_k, 0.5, oracle.CAUSAL)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[6:16] += 3.0
    k2[6:16] *= -2.0
    v2[6:16] += 1.0
    o2, lse2 = oracle.fwd_varlen(q2, k2, v2, cu_q, cu_k, 0.5, oracle.CAUSAL)
    for sl in (slice(0, 6), slice(16, 19)):
        np.testing.assert_array_equal(o[sl], o2[sl])
        np.testing.assert_array_equal(lse[:, sl], lse2[:, sl])
    assert not np.allclose(o[6:16], o2[6:16])


def test_sequence_without_keys_gives_zero_output_and_gradients():
    cu_q, cu_k, q, k, v, do = _make([4, 5], [0, 7])
    o, lse, dq, dk, dv = oracle.bwd_varlen(q, k, v, do, cu_q, cu_k, 0.5)
    assert np.all(o[:4] == 0) and np.all(np.isneginf(lse[:, :4])) and np.all(dq[:4] == 0)
    assert np.all(np.isfinite(lse[:, 4:]))


def test_equal_lengths_match_the_batched_layout():
    """Equal lengths: the packed batch is the [B, H, N, d] problem transposed."""
    B, N, H, d = 3, 9, 2, 8
    cu = np.arange(B + 1) * N
    q, k, v = (rng.standard_normal((B * N, H, d)) for _ in range(3))
    o, lse = oracle.fwd_varlen(q, k, v, cu, cu, 0.4, oracle.CAUSAL)
    bhnd = lambda x: np.ascontiguousarray(x.reshape(B, N, H, d).transpose(0, 2, 1, 3).reshape(B * H, N, d))  # noqa: E731
    ob, lb = _block_diag_fwd(q, k, v, cu, cu, 0.4, causal=True)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    o_dense, l_dense = oracle.fwd(bhnd(q), bhnd(k), bhnd(v), 0.4, oracle.CAUSAL)
    np.testing.assert_allclose(bhnd(o), o_dense, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse.reshape(H, B, N).transpose(1, 0, 2).reshape(B * H, N), l_dense, rtol=0,
                               atol=1e-13)
