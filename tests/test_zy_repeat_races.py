"""Repeated runs as a race detector (collected late).

compute-sanitizer is not available, so timing-dependent hazards are hunted by
repetition: each configuration below runs 50 to 100 times and every run must
return the bytes of the first wherever the path is deterministic (everything
except the default backward's dQ, which is summed with fp32 atomics).  The
configurations are the race-prone ones: CTAs with no work (a query tile that
sees no key block, a key block that no query sees), rows that see no key
(cross attention), the d = 256 backward whose two CTAs share a key block, and
the FP8 forward.
"""
import pytest
import torch

from flash_fwd_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _dev(*ts):
    return [t.to(DEV) for t in ts]


def _same(runs):
    first = runs[0]
    for r in runs[1:]:
        for a, b in zip(first, r):
            if not torch.equal(a, b):
                return False
    return True


def _empty_mask():
    m = torch.ones((3, 3), dtype=torch.uint8)
    m[:, 1] = 0     # key block 1: no query sees it
    m[1, :] = 0     # query block 1: sees no key
    return m.to(DEV)


def test_forward_with_idle_tiles_repeats_exactly():
    import flash_fwd_b200 as fa
    q, k, v = _dev(*inputs.make_qkv(1, 2, 384, 64, "bf16", seed=31, with_dout=False)[:3])
    mask = _empty_mask()
    runs = [fa.attention_fwd(q, k, v, scale=0.125, block_mask=mask) for _ in range(100)]
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert _same(runs)
    assert torch.all(runs[0][0][:, :, 128:256] == 0)


def test_cross_attention_dead_rows_repeat_exactly():
    import flash_fwd_b200 as fa
    q, k, v, _ = inputs.make_qkv_cross(1, 2, 300, 100, 128, "bf16", seed=32)
    q, k, v = _dev(q, k, v)
    runs = [fa.attention_fwd(q, k, v, causal=True, scale=0.09) for _ in range(100)]
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert _same(runs)
    o, lse = runs[0]
    assert torch.all(o[:, :, :200] == 0) and torch.all(torch.isneginf(lse[:, :, :200]))


def test_deterministic_backward_with_idle_tiles_repeats_exactly():
    import flash_fwd_b200 as fa
    q, k, v, do = _dev(*inputs.make_qkv(1, 2, 384, 128, "bf16", seed=33))
    mask = _empty_mask()
    o, lse = fa.attention_fwd(q, k, v, scale=0.1, block_mask=mask)
    runs = [fa.attention_bwd(q, k, v, o, do, lse, scale=0.1, block_mask=mask, deterministic=True)
            for _ in range(50)]
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert _same(runs)
    dq, dk, dv = runs[0]
    assert torch.all(dq[:, :, 128:256] == 0) and torch.all(dk[:, :, 128:256] == 0)
    assert torch.all(dv[:, :, 128:256] == 0)


def test_deterministic_backward_d256_repeats_exactly():
    import flash_fwd_b200 as fa
    q, k, v, do = _dev(*inputs.make_qkv(1, 2, 300, 256, "bf16", seed=34))
    o, lse = fa.attention_fwd(q, k, v, causal=True, scale=0.0625)
    runs = [fa.attention_bwd(q, k, v, o, do, lse, causal=True, scale=0.0625, deterministic=True)
            for _ in range(50)]
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert _same(runs)


def test_split_backward_dk_dv_repeat_exactly():
    # d = 256: two CTAs per key block; dK and dV involve no atomics
    import flash_fwd_b200 as fa
    q, k, v, do = _dev(*inputs.make_qkv(1, 2, 300, 256, "bf16", seed=35))
    o, lse = fa.attention_fwd(q, k, v, causal=True, scale=0.0625)
    runs = [fa.attention_bwd(q, k, v, o, do, lse, causal=True, scale=0.0625)[1:] for _ in range(50)]
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert _same(runs)


def test_fp8_forward_repeats_exactly():
    import flash_fwd_b200 as fa
    q, k, v = _dev(*inputs.make_qkv(1, 2, 300, 128, "bf16", seed=36, with_dout=False)[:3])
    signs = inputs.hadamard_signs(128, seed=3).to(DEV)
    runs = [fa.attention_fwd_fp8(q, k, v, causal=True, signs=signs) for _ in range(100)]
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert _same(runs)
