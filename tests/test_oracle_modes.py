"""Pins for the oracle's extended modes: Nq != Nk (cross attention, bottom-right
aligned), sliding window (left, right) and ALiBi -- the built-in mask modes of
"FlashAttention 深度解析" section 五 -- each against something other than the
oracle's own formula:

* reductions to the already pinned paths: an unbounded window is dense, the
  window (unbounded, 0) is causal, ALiBi with slope 0 is no bias, Nq = Nk
  reproduces the square entry points, a single query row under a
  bottom-right causal mask sees every key;
* closed forms: window (0, 0) leaves one key per row (O = V_i, LSE = score);
  Q = 0 gives means of V over the visible keys (window, cross-attention
  causal), and a fully hidden row gets the O = 0 / LSE = -inf convention;
* ALiBi under a causal mask is linear in the key index, so it equals plain
  causal attention on Q and K augmented by one column ([q, 1], [k, slope j /
  scale]) with LSE shifted by -slope (i + Nk - Nq);
* central finite differences of L = sum(dO * O) against the backward in every
  mode, and the online recurrence against the two-pass definition.
"""
import numpy as np
import pytest

import oracle

rng = np.random.default_rng(4321)


def _r(*shape, s=1.0):
    return rng.standard_normal(shape) * s


def test_square_matches_plain_entry_points():
    q, k, v, do = _r(2, 19, 8), _r(2, 19, 8), _r(2, 19, 8), _r(2, 19, 8)
    for flags in (0, oracle.CAUSAL):
        a = oracle.bwd_full(q, k, v, do, 0.4, flags)
        b = oracle.bwd_full(q, k, v, do, 0.4, flags, window=(-1, -1))
        for x, y in zip(a, b):
            np.testing.assert_allclose(x, y, rtol=0, atol=1e-13)


@pytest.mark.parametrize("nq,nk", [(7, 13), (13, 7), (9, 9)])
def test_unbounded_window_is_dense(nq, nk):
    q, k, v = _r(1, nq, 4), _r(1, nk, 4), _r(1, nk, 4)
    o1, l1 = oracle.fwd(q, k, v, 0.5)
    o2, l2 = oracle.fwd(q, k, v, 0.5, window=(-1, -1))
    o3, l3 = oracle.fwd(q, k, v, 0.5, window=(nk + nq, nk + nq))
    for o, l in ((o2, l2), (o3, l3)):
        np.testing.assert_allclose(o, o1, atol=1e-13)
        np.testing.assert_allclose(l, l1, atol=1e-13)


@pytest.mark.parametrize("nq,nk", [(7, 13), (13, 7), (9, 9)])
def test_window_unbounded_left_zero_right_is_causal(nq, nk):
    q, k, v = _r(1, nq, 4), _r(1, nk, 4), _r(1, nk, 4)
    o1, l1 = oracle.fwd(q, k, v, 0.5, oracle.CAUSAL)
    o2, l2 = oracle.fwd(q, k, v, 0.5, window=(-1, 0))
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_array_equal(np.isinf(l1), np.isinf(l2))
    fin = np.isfinite(l1)
    np.testing.assert_allclose(l2[fin], l1[fin], atol=1e-13)


def test_window_zero_zero_keeps_the_diagonal_key():
    N, d, scale = 11, 5, 0.7
    q, k, v = _r(1, N, d), _r(1, N, d), _r(1, N, d)
    o, lse = oracle.fwd(q, k, v, scale, window=(0, 0))
    np.testing.assert_allclose(o[0], v[0], atol=1e-14)
    np.testing.assert_allclose(lse[0], scale * (q[0] * k[0]).sum(-1), atol=1e-13)


@pytest.mark.parametrize("left,right", [(2, 0), (0, 3), (3, 1)])
def test_zero_query_window_means(left, right):
    N, d = 10, 3
    v = _r(1, N, d)
    o, lse = oracle.fwd(np.zeros((1, N, d)), _r(1, N, d), v, 0.9, window=(left, right))
    for i in range(N):
        lo, hi = max(0, i - left), min(N - 1, i + right)
        np.testing.assert_allclose(o[0, i], v[0, lo:hi + 1].mean(0), atol=1e-13)
        np.testing.assert_allclose(lse[0, i], np.log(hi - lo + 1), atol=1e-13)


def test_cross_attention_causal_zero_query_prefix_means():
    Nq, Nk, d = 5, 12, 3           # query i sees keys 0 .. i + 7
    v = _r(1, Nk, d)
    o, lse = oracle.fwd(np.zeros((1, Nq, d)), _r(1, Nk, d), v, 1.0, oracle.CAUSAL)
    for i in range(Nq):
        n = i + Nk - Nq + 1
        np.testing.assert_allclose(o[0, i], v[0, :n].mean(0), atol=1e-13)
        np.testing.assert_allclose(lse[0, i], np.log(n), atol=1e-13)


def test_more_queries_than_keys_hides_the_first_rows():
    Nq, Nk, d = 9, 4, 3            # rows 0..4 see no key under the bottom-right causal mask
    q, k, v = _r(1, Nq, d), _r(1, Nk, d), _r(1, Nk, d)
    o, lse = oracle.fwd(q, k, v, 0.6, oracle.CAUSAL)
    assert np.all(o[0, :Nq - Nk] == 0) and np.all(lse[0, :Nq - Nk] == -np.inf)
    assert np.all(np.isfinite(lse[0, Nq - Nk:]))
    _, _, dq, dk, dv = oracle.bwd_full(q, k, v, _r(1, Nq, d), 0.6, oracle.CAUSAL)
    assert np.all(dq[0, :Nq - Nk] == 0)


def test_single_query_causal_sees_every_key():
    q, k, v = _r(1, 1, 6), _r(1, 17, 6), _r(1, 17, 6)
    o1, l1 = oracle.fwd(q, k, v, 0.3)
    o2, l2 = oracle.fwd(q, k, v, 0.3, oracle.CAUSAL)
    np.testing.assert_allclose(o2, o1, atol=1e-14)
    np.testing.assert_allclose(l2, l1, atol=1e-14)


def test_alibi_slope_zero_is_no_bias():
    q, k, v, do = _r(2, 9, 4), _r(2, 11, 4), _r(2, 11, 4), _r(2, 9, 4)
    a = oracle.bwd_full(q, k, v, do, 0.5, oracle.CAUSAL)
    b = oracle.bwd_full(q, k, v, do, 0.5, oracle.CAUSAL, slopes=[0.0, 0.0])
    for x, y in zip(a, b):
        np.testing.assert_array_equal(np.isinf(x), np.isinf(y))
        np.testing.assert_allclose(np.where(np.isfinite(x), x, 0), np.where(np.isfinite(y), y, 0), atol=1e-13)


@pytest.mark.parametrize("nq,nk", [(8, 8), (5, 12)])
def test_causal_alibi_is_augmented_plain_attention(nq, nk):
    # -slope (i + off - j) with j <= i + off: a key-linear bias slope j plus a
    # row constant.  Augmenting q with 1 and k with slope j / scale adds
    # exactly slope j to every score.
    d, scale, slopes = 4, 0.6, np.array([0.25, 0.9])
    q, k, v = _r(2, nq, d), _r(2, nk, d), _r(2, nk, d)
    o1, l1 = oracle.fwd(q, k, v, scale, oracle.CAUSAL, slopes=slopes)
    j = np.arange(nk, dtype=np.float64)
    qa = np.concatenate([q, np.ones((2, nq, 1))], axis=2)
    ka = np.concatenate([k, (slopes[:, None] * j[None, :] / scale)[:, :, None]], axis=2)
    va = np.concatenate([v, np.zeros((2, nk, 1))], axis=2)      # the oracle shares d across q, k, v
    o2, l2 = oracle.fwd(qa, ka, va, scale, oracle.CAUSAL)
    np.testing.assert_allclose(o1, o2[:, :, :d], atol=1e-12)
    i = np.arange(nq, dtype=np.float64)
    np.testing.assert_allclose(l1, l2 - slopes[:, None] * (i[None, :] + nk - nq), atol=1e-12)


def test_alibi_zero_query_geometric_weights():
    # Q = 0, no mask: weights exp(-s |i - j|) on V_j = j (one scalar feature)
    N, s = 9, 0.4
    v = np.arange(N, dtype=np.float64).reshape(1, N, 1)
    o, _ = oracle.fwd(np.zeros((1, N, 1)), _r(1, N, 1), v, 1.0, slopes=[s])
    r = np.exp(-s)
    for i in range(N):
        left = np.array([r ** (i - j) for j in range(i + 1)])          # j = 0 .. i
        right = np.array([r ** (j - i) for j in range(i + 1, N)])     # j = i + 1 .. N - 1
        num = (left * np.arange(i + 1)).sum() + (right * np.arange(i + 1, N)).sum()
        den = left.sum() + right.sum()
        np.testing.assert_allclose(o[0, i, 0], num / den, atol=1e-13)


MODES = {
    "cross_causal": dict(nq=5, nk=9, flags=oracle.CAUSAL),
    "cross_dense": dict(nq=9, nk=5, flags=0),
    "window": dict(nq=8, nk=8, window=(2, 1)),
    "window_cross": dict(nq=6, nk=9, window=(1, 2), flags=oracle.CAUSAL),
    "alibi": dict(nq=7, nk=7, slopes=[0.3]),
    "alibi_causal_cross": dict(nq=6, nk=8, slopes=[0.5], flags=oracle.CAUSAL),
}


def _loss(q, k, v, do, scale, kw):
    o, _ = oracle.fwd(q, k, v, scale, kw.get("flags", 0), nthreads=1, window=kw.get("window"),
                      slopes=kw.get("slopes"))
    return float((o[0] * do).sum())


@pytest.mark.parametrize("mode", sorted(MODES))
def test_backward_finite_differences_modes(mode):
    kw = MODES[mode]
    d, scale, h = 3, 0.8, 1e-6
    q, k, v, do = _r(kw["nq"], d), _r(kw["nk"], d), _r(kw["nk"], d), _r(kw["nq"], d)
    _, _, dq, dk, dv = oracle.bwd_full(q, k, v, do, scale, kw.get("flags", 0), window=kw.get("window"),
                                       slopes=kw.get("slopes"))
    for name, x, g in (("q", q, dq[0]), ("k", k, dk[0]), ("v", v, dv[0])):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p[name], args_m[name] = xp, xm
            num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], do, scale, kw)
                        - _loss(args_m["q"], args_m["k"], args_m["v"], do, scale, kw)) / (2 * h)
        rel = np.abs(num - g).max() / max(np.abs(g).max(), 1e-30)
        assert rel <= 1e-6, (mode, name, rel)


@pytest.mark.parametrize("mode", sorted(MODES))
@pytest.mark.parametrize("tile", [1, 3, 128])
def test_online_equals_two_pass_modes(mode, tile):
    kw = MODES[mode]
    q, k, v = _r(kw["nq"], 5), _r(kw["nk"], 5), _r(kw["nk"], 5)
    sl = kw.get("slopes")
    o1, l1 = oracle.fwd(q, k, v, 0.7, kw.get("flags", 0), window=kw.get("window"), slopes=sl)
    o2, l2 = oracle.online_softmax_fwd(q, k, v, 0.7, tile, kw.get("flags", 0), window=kw.get("window"),
                                       slope=None if sl is None else sl[0])
    np.testing.assert_allclose(o2, o1[0], atol=1e-12)
    np.testing.assert_array_equal(np.isinf(l2), np.isinf(l1[0]))


@pytest.mark.parametrize("mode", sorted(MODES))
def test_sampled_entry_points_modes(mode):
    kw = MODES[mode]
    q, k, v, do = _r(2, kw["nq"], 4), _r(2, kw["nk"], 4), _r(2, kw["nk"], 4), _r(2, kw["nq"], 4)
    sl = None if kw.get("slopes") is None else kw["slopes"] * 2
    args = dict(window=kw.get("window"), slopes=sl)
    o, lse, dq, dk, dv = oracle.bwd_full(q, k, v, do, 0.5, kw.get("flags", 0), **args)
    rows = np.array([0, kw["nq"] - 1, 2], dtype=np.int32)
    cols = np.array([kw["nk"] - 1, 1], dtype=np.int32)
    o_r, l_r = oracle.fwd_rows(q, k, v, 0.5, kw.get("flags", 0), rows=rows, **args)
    np.testing.assert_allclose(o_r, o[:, rows], atol=1e-13)
    dq_r = oracle.bwd_dq_rows(q, k, v, do, 0.5, rows, kw.get("flags", 0), **args)
    np.testing.assert_allclose(dq_r, dq[:, rows], atol=1e-12)
    dk_c, dv_c = oracle.bwd_dkdv_cols(q, k, v, do, 0.5, cols, kw.get("flags", 0), **args)
    np.testing.assert_allclose(dk_c, dk[:, cols], atol=1e-12)
    np.testing.assert_allclose(dv_c, dv[:, cols], atol=1e-12)
