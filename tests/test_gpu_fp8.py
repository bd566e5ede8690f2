"""The FP8 forward on the GPU ("FlashAttention 深度解析" section 四: FP8 block
quantisation with incoherent processing) against the oracle.

* The quantiser is compared code for code and scale for scale (bit-exact):
  the rotation and the E4M3 rounding are decisions taken in fp32 on both
  sides in the same operation order.
* The attention is compared on the GPU's own codes (identical to the
  oracle's): LSE within 1e-3.  O differs by the rounding of P to E4M3, which
  the kernel takes on fp32 P relative to its running (lazily rescaled) row
  maximum and the oracle on fp64 P relative to the exact maximum: the two
  are different roundings of the same P, each within
  u_j = min(P_j, max(2^-4 P_j, 2^-10)) for P_j <= 1.  Exactly,
      O_k - O_o = sum_j (e_j - e'_j) (v_jx - O_o) / sum_j (P_j + e_j),
  so |O_k - O_o| <= sum_j 2 u_j |v_jx - O_o| / (sum_j P_j - sum_j u_j): the
  worst-case bar.  With the errors independent and uniform the same sum has
  a standard deviation sigma_ix: the 6-sigma bar.  Every element must meet
  both (each plus the 16-bit rounding of the output, 2^-8 |O_ix| + 1e-4);
  oracle.fp8_o_bounds computes them.
* Exact cases: identical V rows give O = sv * v8 to fp32 rounding.
* Incoherent processing lowers the error of the GPU result against exact
  attention on inputs with outlier channels.
"""
import numpy as np
import pytest
import torch

import oracle
from flash_fwd_b200 import inputs

pytestmark = pytest.mark.gpu

TOL_LSE = 1e-3


def _np(t):
    return t.cpu().numpy()


def _quant(q, k, v, signs):
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    sd = None if signs is None else signs.to(dev)
    out = fa.fa_fp8_quantize_qkv(qd, kd, vd, sd)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return out


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("N", [1, 300])
def test_quantizer_bit_exact(N, rotate, dtype, d):
    B, H = 1, 3
    q, k, v, _ = inputs.make_qkv(B, H, N, d, dtype, seed=N + d, qk_std=3.0)
    signs = inputs.hadamard_signs(d, seed=1) if rotate else None
    q8, k8, v8, sq, sk, sv = _quant(q, k, v, signs)
    sn = None if signs is None else signs.numpy()
    f = lambda t: t.float().reshape(B * H, N, d).numpy()   # noqa: E731
    for name, x, c8, sc, rows, sgn in (("q", q, q8, sq, 128, sn), ("k", k, k8, sk, 128, sn),
                                       ("v", v, v8, sv, N, None)):
        rc, rs = oracle.fp8_quantize(f(x), rows, sgn)
        got_c = _np(c8).reshape(B * H, N, d)
        got_s = _np(sc).reshape(B * H, -1)
        assert np.array_equal(got_c, rc), (name, int((got_c != rc).sum()))
        if name == "v":   # one scale per head, in every block slot
            assert np.array_equal(got_s, np.repeat(rs, got_s.shape[1], axis=1)), name
        else:
            assert np.array_equal(got_s, rs), name


def _fp8_run(q, k, v, causal, signs=None):
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    sd = None if signs is None else signs.to(dev)
    q8, k8, v8, sq, sk, sv = fa.fa_fp8_quantize_qkv(qd, kd, vd, sd)
    o = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:3], dtype=torch.float32, device=dev)
    fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return [_np(t) for t in (q8, k8, v8, sq, sk, sv)], o.float().cpu().numpy(), lse.cpu().numpy()


def _oracle_on_codes(codes, causal, scale, rows=None):
    q8, k8, v8, sq, sk, sv = codes
    B, H, N, d = q8.shape
    r = lambda t: t.reshape(B * H, N, d)   # noqa: E731
    s = lambda t: t.reshape(B * H, -1)     # noqa: E731
    return oracle.fwd_fp8(r(q8), r(k8), r(v8), s(sq), s(sk), s(sv)[:, 0], scale, causal=causal, rows=rows)


def _o_bar(codes, bh, rows, causal, scale, o_ref):
    """Per-element bar on |O_gpu - O_oracle| for query rows `rows` of one (b, h):
    the smaller of the worst case and 6 sigma of oracle.fp8_o_bounds (the
    module docstring has the derivation)."""
    q8, k8, v8, sq, sk, sv = (c.reshape(-1, *c.shape[2:]) for c in codes)
    worst, six_sigma = oracle.fp8_o_bounds(q8[bh], k8[bh], v8[bh], sq[bh], sk[bh], float(sv[bh][0]), scale,
                                           causal, rows, o_ref)
    return np.minimum(worst, six_sigma)


@pytest.mark.parametrize("N", [1, 129, 300, 1000])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_fp8_forward_parity(N, causal, dtype, d):
    B, H = 1, 2
    q, k, v, _ = inputs.make_qkv(B, H, N, d, dtype, seed=7 + N, with_dout=False)
    signs = inputs.hadamard_signs(d, seed=2)
    codes, o, lse = _fp8_run(q, k, v, causal, signs)
    scale = inputs.default_scale(d)
    ro, rl = _oracle_on_codes(codes, causal, scale)
    o = o.reshape(B * H, N, d)
    lse = lse.reshape(B * H, N)
    assert np.isfinite(o).all()
    assert np.abs(lse - rl).max() <= TOL_LSE
    for bh in range(B * H):
        bar = _o_bar(codes, bh, np.arange(N), causal, scale, ro[bh])
        err = np.abs(o[bh] - ro[bh])
        assert np.all(err <= bar), (bh, float(err.max()), float((err / bar).max()))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_fp8_identical_v_rows_exact(d):
    B, H, N = 1, 2, 700
    q, k, v, _ = inputs.make_qkv(B, H, N, d, "bf16", seed=3, with_dout=False)
    v = v[:, :, :1].expand(B, H, N, d).contiguous()
    codes, o, _ = _fp8_run(q, k, v, True)
    vals = oracle.e4m3_values()
    v8, sv = codes[2], codes[5]
    want = vals[v8[:, :, 0]] * sv[:, :, :1]                       # [B, H, d]
    got = o.reshape(B, H, N, d)
    want16 = torch.from_numpy(want).to(torch.bfloat16).float().numpy()
    assert np.abs(got - want16[:, :, None, :]).max() <= 1e-2 * np.abs(want).max()


@pytest.mark.parametrize("d", [64, 128, 256])
def test_fp8_dsweep_shape_sampled(d):
    # B=4 H=16 N=4096 causal: sampled rows per head against the oracle on the GPU's codes
    B, H, N = 4, 16, 4096
    q, k, v, _ = inputs.make_qkv(B, H, N, d, "bf16", seed=0, with_dout=False)
    codes, o, lse = _fp8_run(q, k, v, True, inputs.hadamard_signs(d, seed=0))
    o = o.reshape(B * H, N, d)
    lse = lse.reshape(B * H, N)
    scale = inputs.default_scale(d)
    flat = [c.reshape(B * H, *c.shape[2:]) for c in codes]   # codes [BH, N, d], scales [BH, nb]
    for bh in (0, 21, 63):
        rows = inputs.sample_rows(N, 16, 0, bh).numpy()
        one = [x[bh:bh + 1][None] for x in flat]              # one (b, h) as [1, 1, ...]
        ro, rl = _oracle_on_codes(one, True, scale, rows=rows)
        assert np.abs(lse[bh, rows] - rl[0]).max() <= TOL_LSE
        bar = _o_bar(codes, bh, rows, True, scale, ro[0])
        assert np.all(np.abs(o[bh, rows] - ro[0]) <= bar)


def _exact(q, k, v, scale):
    q, k, v = (t.double().numpy().reshape(-1, t.shape[2], t.shape[3]) for t in (q, k, v))
    return oracle.fwd(q, k, v, scale)[0]


def test_fp8_incoherent_processing_lowers_error():
    B, H, N, d = 1, 4, 512, 128
    q, k, v = inputs.make_qkv_outliers(B, H, N, d, "bf16", seed=5)
    scale = 0.5 / np.sqrt(d)
    ref = _exact(q, k, v, scale)
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    errs = {}
    for name, signs in (("plain", None), ("incoherent", inputs.hadamard_signs(d, seed=4))):
        o, _ = fa.attention_fwd_fp8(q.to(dev), k.to(dev), v.to(dev), scale=scale,
                                    signs=None if signs is None else signs.to(dev))
        torch.cuda.synchronize()
        errs[name] = float(np.sqrt(np.mean((o.float().cpu().numpy().reshape(ref.shape) - ref) ** 2)))
    assert errs["incoherent"] * 1.5 < errs["plain"], errs
