"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module only draws random numbers and casts them; it holds none of the
attention arithmetic.  Recipe (the same everywhere):

* one CPU ``torch.Generator`` seeded with ``seed``;
* fp32 standard-normal draws for Q, K, V, dO, in that order, shape [B, H, N, d];
* Q and K multiplied by ``qk_std`` before the cast (the stress run uses 4);
* cast to fp16 / bf16 with round-to-nearest-even (``Tensor.to``).

The block mask for block-sparse attention has one byte per 128 x 128 block,
shared by all heads: diagonal blocks kept, off-diagonal blocks kept when a
``torch.rand`` draw from its own generator (seeded with ``seed``) is below
``density``.
"""
import math

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}

# The five workloads attention is measured and checked on.  Each one is a shape
# recipe: synthetic N(0,1) data of that shape stands in for real activations.
CONFIGS = {
    "tiny": dict(B=1, H=2, N=128, d=64, dtype="f16", causal=False, bwd=True),
    "gpt2s": dict(B=8, H=12, N=1024, d=64, dtype="bf16", causal=True, bwd=True),
    "long_fwd": dict(B=1, H=8, N=8192, d=128, dtype="f16", causal=None, bwd=False),
    "dsweep": dict(B=4, H=16, N=4096, d=None, dtype="bf16", causal=True, bwd=True),
    "sparse64k": dict(B=1, H=4, N=65536, d=64, dtype="bf16", causal=False, bwd=True,
                      sparse=True, density=0.2),
}


def make_qkv(B, H, N, d, dtype="bf16", seed=0, qk_std=1.0, with_dout=True):
    """Q, K, V (and dO) as contiguous [B, H, N, d] CPU tensors of ``dtype``."""
    g = torch.Generator().manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32) if with_dout else None
    if qk_std != 1.0:
        q = q * qk_std
        k = k * qk_std
    t = DTYPES[dtype] if isinstance(dtype, str) else dtype
    out = [q.to(t).contiguous(), k.to(t).contiguous(), v.to(t).contiguous()]
    out.append(do.to(t).contiguous() if do is not None else None)
    return tuple(out)


def make_block_mask(N, blk=128, density=0.2, seed=0, keep_diagonal=True):
    """uint8 [nb, nb] block mask, nb = ceil(N / blk)."""
    nb = (N + blk - 1) // blk
    g = torch.Generator().manual_seed(int(seed))
    m = (torch.rand((nb, nb), generator=g) < density)
    if keep_diagonal:
        m |= torch.eye(nb, dtype=torch.bool)
    return m.to(torch.uint8).contiguous()


def sample_rows(N, count, seed, head):
    """The query rows checked for one head on large workloads (sorted int32)."""
    g = torch.Generator().manual_seed(int(seed) + int(head))
    idx = torch.randperm(N, generator=g)[: min(count, N)]
    return torch.sort(idx).values.to(torch.int32)


def sample_key_blocks(nb, count, seed, head):
    """Key-block columns checked for dK/dV on large workloads."""
    g = torch.Generator().manual_seed(10_000 + int(seed) + int(head))
    idx = torch.randperm(nb, generator=g)[: min(count, nb)]
    return torch.sort(idx).values.to(torch.int32)


def default_scale(d):
    return 1.0 / math.sqrt(d)


def make_qkv_cross(B, H, Nq, Nk, d, dtype="bf16", seed=0, qk_std=1.0):
    """Q, dO [B, H, Nq, d] and K, V [B, H, Nk, d] CPU tensors of ``dtype``; the
    same recipe as make_qkv (draw order Q, K, V, dO)."""
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32)
    do = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32)
    if qk_std != 1.0:
        q, k = q * qk_std, k * qk_std
    t = DTYPES[dtype]
    return q.to(t).contiguous(), k.to(t).contiguous(), v.to(t).contiguous(), do.to(t).contiguous()


def make_varlen(lengths_q, lengths_k, H, d, dtype="bf16", seed=0):
    """A packed batch: cu_seqlens_q, cu_seqlens_k (int32 [B + 1]), Q, dO
    [total_q, H, d] and K, V [total_k, H, d] CPU tensors of ``dtype`` (draw
    order Q, K, V, dO, as in make_qkv)."""
    lq = torch.tensor([0] + list(lengths_q), dtype=torch.int64)
    lk = torch.tensor([0] + list(lengths_k), dtype=torch.int64)
    assert len(lq) == len(lk) and bool((lq >= 0).all()) and bool((lk >= 0).all())
    cu_q, cu_k = torch.cumsum(lq, 0).to(torch.int32), torch.cumsum(lk, 0).to(torch.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn((tq, H, d), generator=g, dtype=torch.float32)
    k = torch.randn((tk, H, d), generator=g, dtype=torch.float32)
    v = torch.randn((tk, H, d), generator=g, dtype=torch.float32)
    do = torch.randn((tq, H, d), generator=g, dtype=torch.float32)
    t = DTYPES[dtype]
    return cu_q, cu_k, q.to(t).contiguous(), k.to(t).contiguous(), v.to(t).contiguous(), do.to(t).contiguous()


def varlen_lengths(B, lo, hi, seed=0):
    """B sequence lengths drawn uniformly from [lo, hi] (seeded): the length mix
    of a packed batch."""
    g = torch.Generator().manual_seed(int(seed) + 104729)
    return [int(x) for x in torch.randint(lo, hi + 1, (B,), generator=g)]


def alibi_slopes(H):
    """The geometric head slopes 2^(-8 (h + 1) / H) commonly used with ALiBi (fp32 [H])."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32)



def hadamard_signs(d, seed=0):
    """float32 [d] of +1/-1 (seeded): the sign flips of the FP8 path's rotation
    diag(signs) H_d / sqrt(d) (incoherent processing)."""
    g = torch.Generator().manual_seed(int(seed) + 7919)
    return (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.float32)


def make_qkv_outliers(B, H, N, d, dtype="bf16", seed=0, channels=4, magnitude=30.0):
    """Q, K, V i.i.d. N(0, 1) with `channels` outlier channels of Q and K
    scaled by `magnitude` (the case incoherent processing targets)."""
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
    q[..., :channels] *= magnitude
    k[..., :channels] *= magnitude
    t = DTYPES[dtype]
    return q.to(t).contiguous(), k.to(t).contiguous(), v.to(t).contiguous()
