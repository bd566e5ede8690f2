"""Backward parity: dQ, dK, dV of the CUDA path (forward + backward through
the C ABI) against the fp64 oracle, which recomputes everything from Q, K, V
and dO.  Small shapes cover ragged tails, every head dim, both dtypes and the
causal mask with every element checked.  The workload shapes are checked on
every element in test_gpu_workloads.py; here only the 64K block-sparse one,
on seeded sampled rows (dQ) and key blocks (dK, dV) at full size.
"""
import pytest
import torch

from flash_fwd_b200 import inputs
from parity import check_bwd, check_fwd, gpu_bwd, gpu_fwd

pytestmark = pytest.mark.gpu


def _run(q, k, v, do, causal, scale, mask=None):
    o, lse = gpu_fwd(q, k, v, causal, scale, mask)
    return o, lse, gpu_bwd(q, k, v, o, do, lse, causal, scale, mask)


@pytest.mark.parametrize("N", [1, 17, 128, 129, 300])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_small(N, d, dtype, causal):
    q, k, v, do = inputs.make_qkv(1, 2, N, d, dtype, seed=100 + N + d)
    scale = inputs.default_scale(d)
    _, _, grads = _run(q, k, v, do, causal, scale)
    check_bwd(grads, q, k, v, do, causal, scale)


def test_bwd_tiny_config():
    c = inputs.CONFIGS["tiny"]
    q, k, v, do = inputs.make_qkv(c["B"], c["H"], c["N"], c["d"], c["dtype"], seed=0)
    scale = inputs.default_scale(c["d"])
    o, lse, grads = _run(q, k, v, do, False, scale)
    check_fwd(o, lse, q, k, v, False, scale, c["dtype"])
    check_bwd(grads, q, k, v, do, False, scale)


def test_bwd_sparse64k_config_sampled():
    c = inputs.CONFIGS["sparse64k"]
    q, k, v, do = inputs.make_qkv(c["B"], c["H"], c["N"], c["d"], c["dtype"], seed=0)
    mask = inputs.make_block_mask(c["N"], 128, c["density"], seed=0)
    scale = inputs.default_scale(c["d"])
    _, _, grads = _run(q, k, v, do, False, scale, mask)
    # 256 query rows per head for dQ; dK/dV on every key of 2 key-block columns per head
    check_bwd(grads, q, k, v, do, False, scale, mask=mask, dq_rows=256, kv_blocks=2)


def test_sparse_2048_full():
    # the same mask generator at N = 2048: forward and backward checked on every element
    N, d = 2048, 64
    q, k, v, do = inputs.make_qkv(1, 4, N, d, "bf16", seed=0)
    mask = inputs.make_block_mask(N, 128, 0.2, seed=0)
    scale = inputs.default_scale(d)
    o, lse, grads = _run(q, k, v, do, False, scale, mask)
    check_fwd(o, lse, q, k, v, False, scale, "bf16", mask=mask)
    check_bwd(grads, q, k, v, do, False, scale, mask=mask)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_bwd_sparse_small(causal, d):
    N = 1000
    q, k, v, do = inputs.make_qkv(1, 2, N, d, "bf16", seed=7)
    mask = inputs.make_block_mask(N, 128, 0.3, seed=7)
    scale = inputs.default_scale(d)
    _, _, grads = _run(q, k, v, do, causal, scale, mask)
    check_bwd(grads, q, k, v, do, causal, scale, mask=mask)


def test_bwd_empty_mask_column_and_row():
    # key block 1 is seen by no query block and query block 1 sees nothing
    N, d = 384, 64
    q, k, v, do = inputs.make_qkv(1, 1, N, d, "bf16", seed=4)
    mask = torch.ones((3, 3), dtype=torch.uint8)
    mask[:, 1] = 0
    mask[1, :] = 0
    o, lse, grads = _run(q, k, v, do, False, 0.125, mask)
    dq, dk, dv = grads
    assert torch.all(dk[0, 0, 128:256] == 0) and torch.all(dv[0, 0, 128:256] == 0)
    assert torch.all(dq[0, 0, 128:256] == 0)
    check_bwd(grads, q, k, v, do, False, 0.125, mask=mask)


def test_bwd_dk_dv_deterministic():
    q, k, v, do = inputs.make_qkv(2, 3, 1500, 128, "bf16", seed=8)
    o, lse = gpu_fwd(q, k, v, True, 0.09)
    a = gpu_bwd(q, k, v, o, do, lse, True, 0.09)
    b = gpu_bwd(q, k, v, o, do, lse, True, 0.09)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dQ is reduced with fp32 atomics: equal up to summation order
    assert (a[0].float() - b[0].float()).abs().max() <= 1e-2
