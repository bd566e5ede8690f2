"""Forward parity: the CUDA path through the C ABI against the fp64 oracle.

Small shapes cover ragged tails (N = 1, 17, 129, 300, 520), every head dim,
both dtypes and the causal mask with every row checked.  The workload shapes
are checked on every element in test_gpu_workloads.py; here only the 64K
block-sparse one, on seeded sampled rows at full size.
"""
import numpy as np
import pytest
import torch

from flash_fwd_b200 import inputs
from parity import TOL_LSE, check_fwd, gpu_fwd

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N", [1, 17, 128, 129, 300, 520])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_small(N, d, dtype, causal):
    q, k, v, _ = inputs.make_qkv(1, 2, N, d, dtype, seed=N + d, with_dout=False)
    scale = inputs.default_scale(d)
    o, lse = gpu_fwd(q, k, v, causal, scale)
    check_fwd(o, lse, q, k, v, causal, scale, dtype)


def test_fwd_tiny_config():
    c = inputs.CONFIGS["tiny"]
    q, k, v, _ = inputs.make_qkv(c["B"], c["H"], c["N"], c["d"], c["dtype"], seed=0)
    scale = inputs.default_scale(c["d"])
    o, lse = gpu_fwd(q, k, v, False, scale)
    check_fwd(o, lse, q, k, v, False, scale, c["dtype"])


def test_fwd_sparse64k_config_sampled():
    c = inputs.CONFIGS["sparse64k"]
    q, k, v, _ = inputs.make_qkv(c["B"], c["H"], c["N"], c["d"], c["dtype"], seed=0, with_dout=False)
    mask = inputs.make_block_mask(c["N"], 128, c["density"], seed=0)
    scale = inputs.default_scale(c["d"])
    o, lse = gpu_fwd(q, k, v, False, scale, mask)
    check_fwd(o, lse, q, k, v, False, scale, c["dtype"], mask=mask, rows_per_head=256)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_fwd_sparse_small(causal, d):
    N = 1000
    q, k, v, _ = inputs.make_qkv(1, 3, N, d, "bf16", seed=5, with_dout=False)
    mask = inputs.make_block_mask(N, 128, 0.3, seed=5)
    scale = inputs.default_scale(d)
    o, lse = gpu_fwd(q, k, v, causal, scale, mask)
    check_fwd(o, lse, q, k, v, causal, scale, "bf16", mask=mask)


def test_fwd_sparse_all_ones_equals_dense_bitwise():
    N, d = 700, 128
    q, k, v, _ = inputs.make_qkv(2, 2, N, d, "f16", seed=9, with_dout=False)
    nb = (N + 127) // 128
    ones = torch.ones((nb, nb), dtype=torch.uint8)
    o1, l1 = gpu_fwd(q, k, v, False, 0.1, ones)
    o2, l2 = gpu_fwd(q, k, v, False, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_sparse_lower_triangle_with_causal_equals_causal_bitwise():
    N, d = 900, 64
    q, k, v, _ = inputs.make_qkv(1, 4, N, d, "bf16", seed=11, with_dout=False)
    nb = (N + 127) // 128
    tril = torch.ones((nb, nb), dtype=torch.uint8).tril().contiguous()
    o1, l1 = gpu_fwd(q, k, v, True, 0.125, tril)
    o2, l2 = gpu_fwd(q, k, v, True, 0.125)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_empty_mask_row():
    N, d = 384, 64
    q, k, v, _ = inputs.make_qkv(1, 1, N, d, "bf16", seed=2, with_dout=False)
    mask = torch.ones((3, 3), dtype=torch.uint8)
    mask[1] = 0
    o, lse = gpu_fwd(q, k, v, False, 0.125, mask)
    assert torch.all(o[0, 0, 128:256] == 0)
    assert torch.all(torch.isneginf(lse[0, 0, 128:256]))
    keep = torch.cat([torch.arange(0, 128), torch.arange(256, 384)])
    # rows of the kept block rows still match the oracle
    import oracle
    from parity import bh
    ref_o, ref_l = oracle.fwd_rows(bh(q), bh(k), bh(v), 0.125, oracle.SPARSE, mask.numpy(), 128,
                                   keep.numpy().astype(np.int32))
    assert np.abs(o[0, 0, keep].double().numpy() - ref_o[0]).max() <= 2e-2
    assert np.abs(lse[0, 0, keep].double().numpy() - ref_l[0]).max() <= TOL_LSE


def test_fwd_deterministic():
    q, k, v, _ = inputs.make_qkv(2, 4, 2000, 128, "bf16", seed=3, with_dout=False)
    a = gpu_fwd(q, k, v, True, 0.09)
    b = gpu_fwd(q, k, v, True, 0.09)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
