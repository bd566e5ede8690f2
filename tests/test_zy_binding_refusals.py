"""The binding refuses, with real device tensors, what the C ABI could not
check: a host tensor among device ones, a strided view, a short output, a
mismatched dtype.  Nothing is launched, so the device status stays 0, and a
well-formed call right after still runs.  (Collected next to last, before
the no-alloc tests.)
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_refusals_launch_nothing():
    import flash_fwd_b200 as fa
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 2, 200, 64
    q, k, v = (torch.randn(B, H, N, d, device=dev).to(torch.bfloat16) for _ in range(3))
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev)
    bad = [
        dict(lse=torch.empty(B, H, N)),                                                  # host memory
        dict(q=torch.randn(B, H, d, N, device=dev).to(torch.bfloat16).transpose(2, 3)),  # strided view
        dict(o=torch.empty(B, H, N - 1, d, device=dev, dtype=torch.bfloat16)),           # short output
        dict(k=k.to(torch.float16)),                                                     # dtype mismatch
        dict(lse=torch.empty(B, H, N, device=dev, dtype=torch.float16)),                 # LSE not fp32
    ]
    for change in bad:
        a = dict(q=q, k=k, v=v, o=o, lse=lse)
        a.update(change)
        with pytest.raises(ValueError):
            fa.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    fa.fa_fwd(q, k, v, o, lse, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
