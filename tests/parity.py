"""Shared helpers for the GPU parity tests: seeded inputs -> CUDA path (through
the C ABI binding) and -> fp64 oracle, compared element by element.

Tolerances (max absolute error unless stated):
  O   1e-2 (fp16), 2e-2 (bf16)
  LSE 1e-3
  dQ, dK, dV  5e-2 * max |oracle value| of that tensor.  Only a tensor whose
              oracle values are all exactly zero (dQ and dK at N = 1, where
              every row has one key) is held to 5e-3 absolute instead.  A
              sampled check normalises by the largest oracle value among the
              sampled elements, a lower bound of the tensor's maximum, so its
              bar is never looser than the one on the whole tensor.
"""
import numpy as np
import torch

import oracle
from flash_fwd_b200 import inputs

TOL_O = {"f16": 1e-2, "bf16": 2e-2}
TOL_LSE = 1e-3
TOL_GRAD_REL = 5e-2
GRAD_NORM_FLOOR = 0.1


def grad_norm(want_max):
    """The normaliser of the gradient bar for an oracle tensor whose largest
    magnitude is `want_max` (the floor applies only to an exactly zero tensor)."""
    return want_max if want_max > 0.0 else GRAD_NORM_FLOOR


def bh(x):
    """[B, H, N, d] -> float64 numpy [B*H, N, d]."""
    return x.reshape(-1, x.shape[-2], x.shape[-1]).double().numpy()


def flags(causal, mask):
    return (oracle.CAUSAL if causal else 0) | (oracle.SPARSE if mask is not None else 0)


def mask_np(mask):
    return None if mask is None else mask.numpy().astype(np.uint8)


def gpu_fwd(q, k, v, causal, scale, mask=None):
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    md = mask.to(dev) if mask is not None else None
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, scale=scale, block_mask=md)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return o.cpu(), lse.cpu()


def gpu_bwd(q, k, v, o, do, lse, causal, scale, mask=None):
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    args = [t.to(dev) for t in (q, k, v, o, do)]
    md = mask.to(dev) if mask is not None else None
    dq, dk, dv = fa.attention_bwd(*args, lse.to(dev), causal=causal, scale=scale, block_mask=md)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


def check_fwd(o_gpu, lse_gpu, q, k, v, causal, scale, dtype, mask=None, rows_per_head=None, seed=0):
    """Compares O and LSE with the oracle on every row, or on sampled rows per head."""
    B, H, N, d = q.shape
    Q, K, V = bh(q), bh(k), bh(v)
    og = o_gpu.reshape(B * H, N, d).double().numpy()
    lg = lse_gpu.reshape(B * H, N).double().numpy()
    worst_o, worst_l = 0.0, 0.0
    if rows_per_head is None:
        o_ref, l_ref = oracle.fwd(Q, K, V, scale, flags(causal, mask), mask_np(mask))
        worst_o = np.abs(og - o_ref).max()
        worst_l = np.abs(lg - l_ref).max()
    else:
        for h in range(B * H):
            rows = inputs.sample_rows(N, rows_per_head, seed, h).numpy()
            o_ref, l_ref = oracle.fwd_rows(Q[h:h + 1], K[h:h + 1], V[h:h + 1], scale, flags(causal, mask),
                                           mask_np(mask), 128, rows)
            worst_o = max(worst_o, np.abs(og[h, rows] - o_ref[0]).max())
            worst_l = max(worst_l, np.abs(lg[h, rows] - l_ref[0]).max())
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    assert worst_o <= TOL_O[dtype], f"O max err {worst_o}"
    assert worst_l <= TOL_LSE, f"LSE max err {worst_l}"
    return worst_o, worst_l


def check_bwd(grads_gpu, q, k, v, do, causal, scale, mask=None, dq_rows=None, kv_cols=None, heads=None, seed=0,
              kv_blocks=None):
    """Compares dQ, dK, dV with the oracle.

    Full check when dq_rows is None; otherwise dQ on `dq_rows` sampled rows per
    head and dK/dV on `kv_cols` sampled keys per head -- or, with kv_blocks, on
    every key of `kv_blocks` sampled 128-key block columns per head -- for the
    heads listed in `heads` (all when None).  Bar: max |err| <= 5e-2 * max |oracle value|.
    """
    B, H, N, d = q.shape
    Q, K, V, DO = bh(q), bh(k), bh(v), bh(do)
    dq, dk, dv = (g.reshape(B * H, N, d).double().numpy() for g in grads_gpu)
    for g in (dq, dk, dv):
        assert np.isfinite(g).all()
    fl, mk = flags(causal, mask), mask_np(mask)
    errs = {}
    if dq_rows is None:
        _, _, rdq, rdk, rdv = oracle.bwd_full(Q, K, V, DO, scale, fl, mk)
        pairs = {"dq": (dq, rdq), "dk": (dk, rdk), "dv": (dv, rdv)}
        for name, (got, want) in pairs.items():
            errs[name] = np.abs(got - want).max() / grad_norm(np.abs(want).max())
    else:
        hs = range(B * H) if heads is None else heads
        worst = {"dq": [0.0, 0.0], "dk": [0.0, 0.0], "dv": [0.0, 0.0]}
        for hh in hs:
            rows = inputs.sample_rows(N, dq_rows, seed, hh).numpy()
            if kv_blocks is None:
                cols = inputs.sample_rows(N, kv_cols, seed + 7, hh).numpy()
            else:
                blocks = inputs.sample_key_blocks((N + 127) // 128, kv_blocks, seed, hh).numpy()
                cols = np.concatenate([np.arange(b * 128, min(b * 128 + 128, N)) for b in blocks]).astype(np.int32)
            sl = slice(hh, hh + 1)
            rdq = oracle.bwd_dq_rows(Q[sl], K[sl], V[sl], DO[sl], scale, rows, fl, mk)[0]
            rdk, rdv = oracle.bwd_dkdv_cols(Q[sl], K[sl], V[sl], DO[sl], scale, cols, fl, mk)
            for name, got, want in (("dq", dq[hh, rows], rdq), ("dk", dk[hh, cols], rdk[0]),
                                    ("dv", dv[hh, cols], rdv[0])):
                worst[name][0] = max(worst[name][0], np.abs(got - want).max())
                worst[name][1] = max(worst[name][1], np.abs(want).max())
        errs = {n: e / grad_norm(m) for n, (e, m) in worst.items()}
    for name, e in errs.items():
        assert e <= TOL_GRAD_REL, f"{name} relative max err {e}"
    return errs


def oracle_all(q, k, v, do, causal, scale, mask=None, with_bwd=True):
    """The oracle's O, LSE and (with_bwd) dQ, dK, dV on every element.

    The forward runs over every query row; the gradients come from the row
    (dQ) and column (dK, dV) entry points over every row and every key, which
    give the same values as the full materialising backward (pinned on CPU)
    without its column-strided loops, so the workload shapes finish in
    seconds to about a minute on the host cores.
    """
    Q, K, V = bh(q), bh(k), bh(v)
    N = Q.shape[1]
    fl, mk = flags(causal, mask), mask_np(mask)
    ref = {}
    ref["o"], ref["lse"] = oracle.fwd(Q, K, V, scale, fl, mk)
    if with_bwd:
        DO = bh(do)
        every = np.arange(N, dtype=np.int32)
        ref["dq"] = oracle.bwd_dq_rows(Q, K, V, DO, scale, every, fl, mk)
        ref["dk"], ref["dv"] = oracle.bwd_dkdv_cols(Q, K, V, DO, scale, every, fl, mk)
    return ref


def compare_fwd(o_gpu, lse_gpu, ref, dtype):
    """Max errors of O and LSE against oracle_all's result, asserted against the bars."""
    og = o_gpu.reshape(ref["o"].shape).double().numpy()
    lg = lse_gpu.reshape(ref["lse"].shape).double().numpy()
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    worst_o = np.abs(og - ref["o"]).max()
    worst_l = np.abs(lg - ref["lse"]).max()
    assert worst_o <= TOL_O[dtype], f"O max err {worst_o}"
    assert worst_l <= TOL_LSE, f"LSE max err {worst_l}"
    return worst_o, worst_l


def compare_bwd(grads_gpu, ref):
    """Relative max errors of dQ, dK, dV against oracle_all's result, asserted."""
    errs = {}
    for name, g in zip(("dq", "dk", "dv"), grads_gpu):
        want = ref[name]
        got = g.reshape(want.shape).double().numpy()
        assert np.isfinite(got).all(), name
        errs[name] = np.abs(got - want).max() / grad_norm(np.abs(want).max())
        assert errs[name] <= TOL_GRAD_REL, f"{name} relative max err {errs[name]}"
    return errs
