"""Pins for the fp64 oracle, each against something other than the oracle itself.

* hand-worked cases (tests/golden/hand_cases.json, each with its citation);
* the online-softmax recurrence against the two-pass definition;
* closed forms: N = 1, Q = 0 (means of V, prefix means under causal),
  identical V rows;
* invariants: K shift, V shift, rows of P summing to one, sum_j dK_j = 0;
* central finite differences of L = sum(dO * O) against the backward;
* block-sparse consistency with dense and causal;
* PyTorch's own fp64 attention and autograd as an independent library routine;
* the sampled entry points against the full materialising one.

A plausible mistake (a dropped scale, a wrong sign in dS, a transposed operand,
a missing mask term) breaks at least one of these.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _flags(causal, sparse):
    return (oracle.CAUSAL if causal else 0) | (oracle.SPARSE if sparse else 0)


# --------------------------------------------------------------------------
# hand-worked golden cases
# --------------------------------------------------------------------------
def _golden_cases():
    with open(os.path.join(GOLDEN, "hand_cases.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_hand_cases(case):
    q, k, v = (np.array(case[x], dtype=np.float64) for x in ("q", "k", "v"))
    mask = np.array(case["mask"], dtype=np.uint8) if case["mask"] is not None else None
    flags = _flags(case["causal"], mask is not None)
    o, lse = oracle.fwd(q, k, v, case["scale"], flags, mask, case["blk"])
    np.testing.assert_allclose(o[0], np.array(case["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], np.array(case["lse"]), rtol=0, atol=1e-12)
    if case.get("dout") is not None:
        dout = np.array(case["dout"])
        o2, lse2, dq, dk, dv = oracle.bwd_full(q, k, v, dout, case["scale"], flags, mask, case["blk"])
        np.testing.assert_allclose(o2[0], np.array(case["o"]), atol=1e-12)
        np.testing.assert_allclose(dq[0], np.array(case["dq"]), atol=1e-12)
        np.testing.assert_allclose(dk[0], np.array(case["dk"]), atol=1e-12)
        np.testing.assert_allclose(dv[0], np.array(case["dv"]), atol=1e-12)


# --------------------------------------------------------------------------
# online softmax == two-pass softmax
# --------------------------------------------------------------------------
@pytest.mark.parametrize("tile", [1, 3, 7, 128])
@pytest.mark.parametrize("mode", ["dense", "causal", "sparse"])
def test_online_equals_two_pass(tile, mode):
    N, d, blk = 53, 8, 4
    q, k, v = _rand(N, d, scale=2.0), _rand(N, d, scale=2.0), _rand(N, d)
    mask = None
    if mode == "sparse":
        nb = (N + blk - 1) // blk
        mask = (rng.random((nb, nb)) < 0.4).astype(np.uint8)
        np.fill_diagonal(mask, 1)
    flags = _flags(mode == "causal", mode == "sparse")
    o2, lse2 = oracle.fwd(q, k, v, 0.3, flags, mask, blk)
    o1, lse1 = oracle.online_softmax_fwd(q, k, v, 0.3, tile, flags, mask, blk)
    np.testing.assert_allclose(o1, o2[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse1, lse2[0], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
def test_single_key_gives_v():
    d = 5
    q, k, v = _rand(1, d), _rand(1, d), _rand(1, d)
    o, lse = oracle.fwd(q, k, v, 0.7)
    np.testing.assert_allclose(o[0], v, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], 0.7 * float(q[0] @ k[0]), atol=1e-13)


def test_zero_query_gives_mean_dense():
    N, d = 37, 6
    q, k, v = np.zeros((N, d)), _rand(N, d, scale=3.0), _rand(N, d)
    o, lse = oracle.fwd(q, k, v, 0.5)
    np.testing.assert_allclose(o[0], np.broadcast_to(v.mean(0), (N, d)), atol=1e-13)
    np.testing.assert_allclose(lse[0], np.full(N, math.log(N)), atol=1e-13)


def test_zero_query_gives_prefix_mean_causal():
    N, d = 37, 6
    q, k, v = np.zeros((N, d)), _rand(N, d), _rand(N, d)
    o, lse = oracle.fwd(q, k, v, 0.5, oracle.CAUSAL)
    prefix = np.cumsum(v, axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(o[0], prefix, atol=1e-13)
    np.testing.assert_allclose(lse[0], np.log(np.arange(1, N + 1)), atol=1e-13)


def test_zero_query_gives_kept_mean_sparse():
    N, d, blk = 40, 3, 8
    nb = N // blk
    mask = (rng.random((nb, nb)) < 0.5).astype(np.uint8)
    np.fill_diagonal(mask, 1)
    q, k, v = np.zeros((N, d)), _rand(N, d), _rand(N, d)
    o, lse = oracle.fwd(q, k, v, 1.0, oracle.SPARSE, mask, blk)
    for i in range(N):
        keys = [j for j in range(N) if mask[i // blk, j // blk]]
        np.testing.assert_allclose(o[0, i], v[keys].mean(0), atol=1e-13)
        np.testing.assert_allclose(lse[0, i], math.log(len(keys)), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_v_rows(causal):
    N, d = 29, 7
    q, k = _rand(N, d, scale=4.0), _rand(N, d, scale=4.0)
    row = _rand(d)
    v = np.broadcast_to(row, (N, d)).copy()
    o, _ = oracle.fwd(q, k, v, 1.0, _flags(causal, False))
    np.testing.assert_allclose(o[0], np.broadcast_to(row, (N, d)), atol=1e-12)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_k_shift_and_v_shift(causal):
    N, d, scale = 31, 5, 0.4
    q, k, v = _rand(N, d), _rand(N, d), _rand(N, d)
    u, c = _rand(d), _rand(d)
    flags = _flags(causal, False)
    o, lse = oracle.fwd(q, k, v, scale, flags)
    o_k, lse_k = oracle.fwd(q, k + u, v, scale, flags)
    o_v, _ = oracle.fwd(q, k, v + c, scale, flags)
    np.testing.assert_allclose(o_k, o, atol=1e-12)
    np.testing.assert_allclose(lse_k[0], lse[0] + scale * (q @ u), atol=1e-12)
    np.testing.assert_allclose(o_v[0], o[0] + c, atol=1e-12)


def test_probabilities_sum_to_one_via_ones_v():
    # with V = all-ones column, O is the row sum of P
    N, d = 23, 4
    q, k = _rand(N, d), _rand(N, d)
    v = np.ones((N, 1))
    for flags in (0, oracle.CAUSAL):
        o, _ = oracle.fwd(np.pad(q, ((0, 0), (0, 0))), k, np.ones((N, d)), 1.0, flags)
        np.testing.assert_allclose(o[0], 1.0, atol=1e-13)
    del v


@pytest.mark.parametrize("causal", [False, True])
def test_dk_sums_to_zero(causal):
    N, d = 19, 4
    q, k, v, do = _rand(N, d), _rand(N, d), _rand(N, d), _rand(N, d)
    _, _, dq, dk, dv = oracle.bwd_full(q, k, v, do, 0.6, _flags(causal, False))
    np.testing.assert_allclose(dk[0].sum(0), 0.0, atol=1e-12)


# --------------------------------------------------------------------------
# backward against central finite differences of L = sum(dO * O)
# --------------------------------------------------------------------------
def _loss(q, k, v, do, scale, flags, mask, blk):
    o, _ = oracle.fwd(q, k, v, scale, flags, mask, blk, nthreads=1)
    return float((o[0] * do).sum())


@pytest.mark.parametrize("mode", ["dense", "causal", "sparse"])
def test_backward_finite_differences(mode):
    N, d, scale, blk, h = 8, 4, 0.8, 2, 1e-6
    q, k, v, do = _rand(N, d), _rand(N, d), _rand(N, d), _rand(N, d)
    mask = None
    if mode == "sparse":
        mask = np.array([[1, 0, 1, 0], [1, 1, 0, 0], [0, 1, 1, 1], [1, 0, 0, 1]], dtype=np.uint8)
    flags = _flags(mode == "causal", mode == "sparse")
    _, _, dq, dk, dv = oracle.bwd_full(q, k, v, do, scale, flags, mask, blk)
    for name, x, g in (("q", q, dq[0]), ("k", k, dk[0]), ("v", v, dv[0])):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            lp = _loss(args_p["q"], args_p["k"], args_p["v"], do, scale, flags, mask, blk)
            lm = _loss(args_m["q"], args_m["k"], args_m["v"], do, scale, flags, mask, blk)
            num[idx] = (lp - lm) / (2 * h)
        rel = np.abs(num - g).max() / max(np.abs(g).max(), 1e-30)
        assert rel <= 1e-6, (name, rel)


# --------------------------------------------------------------------------
# block-sparse consistency
# --------------------------------------------------------------------------
def test_all_ones_mask_equals_dense():
    N, d, blk = 45, 6, 8
    q, k, v, do = _rand(N, d), _rand(N, d), _rand(N, d), _rand(N, d)
    nb = (N + blk - 1) // blk
    ones = np.ones((nb, nb), dtype=np.uint8)
    a = oracle.bwd_full(q, k, v, do, 0.5, 0)
    b = oracle.bwd_full(q, k, v, do, 0.5, oracle.SPARSE, ones, blk)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-13)


def test_block_lower_triangle_with_causal_equals_causal():
    N, d, blk = 45, 6, 8
    q, k, v, do = _rand(N, d), _rand(N, d), _rand(N, d), _rand(N, d)
    nb = (N + blk - 1) // blk
    tril = np.tril(np.ones((nb, nb), dtype=np.uint8))
    a = oracle.bwd_full(q, k, v, do, 0.5, oracle.CAUSAL)
    b = oracle.bwd_full(q, k, v, do, 0.5, oracle.CAUSAL | oracle.SPARSE, tril, blk)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-13)
    # and without the causal flag it is NOT the causal result (the diagonal
    # blocks still need their element mask)
    c = oracle.fwd(q, k, v, 0.5, oracle.SPARSE, tril, blk)
    assert np.abs(c[0] - a[0]).max() > 1e-3


def test_fully_masked_row_convention():
    N, d, blk = 8, 3, 4
    mask = np.array([[0, 0], [1, 1]], dtype=np.uint8)  # first 4 rows see nothing
    q, k, v, do = _rand(N, d), _rand(N, d), _rand(N, d), _rand(N, d)
    o, lse, dq, dk, dv = oracle.bwd_full(q, k, v, do, 1.0, oracle.SPARSE, mask, blk)
    assert np.all(o[0, :4] == 0.0) and np.all(np.isneginf(lse[0, :4]))
    assert np.all(dq[0, :4] == 0.0)
    assert np.all(np.isfinite(o[0, 4:]))


# --------------------------------------------------------------------------
# an independent library routine: PyTorch fp64 attention and autograd
# --------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["dense", "causal", "sparse"])
def test_against_torch_fp64(mode):
    B, H, N, d, blk, scale = 2, 3, 70, 16, 16, 0.25
    g = torch.Generator().manual_seed(7)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(4))
    nb = (N + blk - 1) // blk
    mask_np = None
    attn_mask = None
    if mode == "sparse":
        mask_np = (np.random.default_rng(3).random((nb, nb)) < 0.4).astype(np.uint8)
        np.fill_diagonal(mask_np, 1)
        full = torch.from_numpy(np.kron(mask_np, np.ones((blk, blk), dtype=np.uint8))[:N, :N]).bool()
        attn_mask = full
    elif mode == "causal":
        attn_mask = torch.ones(N, N, dtype=torch.bool).tril()
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=attn_mask, scale=scale)
    ref.backward(do)
    flags = _flags(mode == "causal", mode == "sparse")
    o, lse, dq, dk, dv = oracle.bwd_full(q.reshape(B * H, N, d).numpy(), k.reshape(B * H, N, d).numpy(),
                                         v.reshape(B * H, N, d).numpy(), do.reshape(B * H, N, d).numpy(),
                                         scale, flags, mask_np, blk)
    np.testing.assert_allclose(o, ref.detach().reshape(B * H, N, d).numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, qq.grad.reshape(B * H, N, d).numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, kk.grad.reshape(B * H, N, d).numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, vv.grad.reshape(B * H, N, d).numpy(), atol=1e-11)
    # LSE against torch.logsumexp of the masked score matrix
    s = (q @ k.transpose(-1, -2)) * scale
    if attn_mask is not None:
        s = s.masked_fill(~attn_mask, float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).reshape(B * H, N).numpy(), atol=1e-12)


# --------------------------------------------------------------------------
# sampled entry points agree with the full one
# --------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["dense", "causal", "sparse"])
def test_sampled_entry_points(mode):
    BH, N, d, blk = 3, 50, 8, 8
    q, k, v, do = (_rand(BH, N, d) for _ in range(4))
    nb = (N + blk - 1) // blk
    mask = None
    if mode == "sparse":
        mask = (rng.random((nb, nb)) < 0.5).astype(np.uint8)
        np.fill_diagonal(mask, 1)
    flags = _flags(mode == "causal", mode == "sparse")
    o, lse, dq, dk, dv = oracle.bwd_full(q, k, v, do, 0.35, flags, mask, blk)
    rows = np.array([0, 3, 17, 49], dtype=np.int32)
    cols = np.array([1, 8, 30, 49], dtype=np.int32)
    o_r, lse_r = oracle.fwd_rows(q, k, v, 0.35, flags, mask, blk, rows)
    dq_r = oracle.bwd_dq_rows(q, k, v, do, 0.35, rows, flags, mask, blk)
    dk_c, dv_c = oracle.bwd_dkdv_cols(q, k, v, do, 0.35, cols, flags, mask, blk)
    np.testing.assert_allclose(o_r, o[:, rows], atol=1e-13)
    np.testing.assert_allclose(lse_r, lse[:, rows], atol=1e-13)
    np.testing.assert_allclose(dq_r, dq[:, rows], atol=1e-12)
    np.testing.assert_allclose(dk_c, dk[:, cols], atol=1e-12)
    np.testing.assert_allclose(dv_c, dv[:, cols], atol=1e-12)


def test_threads_do_not_change_results():
    BH, N, d = 4, 64, 8
    q, k, v = (_rand(BH, N, d) for _ in range(3))
    a = oracle.fwd(q, k, v, 0.3, oracle.CAUSAL, nthreads=1)
    b = oracle.fwd(q, k, v, 0.3, oracle.CAUSAL, nthreads=8)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
