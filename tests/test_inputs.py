"""The seeded input recipe (host logic shared by the CUDA path's tests, the
benchmark and the oracle's checks): reproducible, in the documented draw
order and cast, with the block-mask, ALiBi-slope and sign-flip conventions
the readings state."""
import torch

from flash_fwd_b200 import inputs


def test_qkv_follow_the_recipe_bit_for_bit():
    # one generator, fp32 standard normals in the order Q, K, V, dO, Q and K
    # scaled before a round-to-nearest-even cast
    g = torch.Generator().manual_seed(5)
    draws = [torch.randn((2, 3, 17, 8), generator=g) for _ in range(4)]
    q, k, v, do = inputs.make_qkv(2, 3, 17, 8, "bf16", seed=5, qk_std=4.0)
    assert torch.equal(q, (draws[0] * 4.0).to(torch.bfloat16))
    assert torch.equal(k, (draws[1] * 4.0).to(torch.bfloat16))
    assert torch.equal(v, draws[2].to(torch.bfloat16))
    assert torch.equal(do, draws[3].to(torch.bfloat16))
    for t in (q, k, v, do):
        assert t.is_contiguous() and t.dtype == torch.bfloat16
    # reproducible; a different seed gives different data; no dO when not asked
    assert torch.equal(inputs.make_qkv(2, 3, 17, 8, "bf16", seed=5, qk_std=4.0)[0], q)
    assert not torch.equal(inputs.make_qkv(2, 3, 17, 8, "bf16", seed=6, qk_std=4.0)[0], q)
    assert inputs.make_qkv(1, 1, 4, 8, "f16", with_dout=False)[3] is None


def test_cross_inputs_share_the_recipe():
    q, k, v, do = inputs.make_qkv_cross(1, 2, 5, 9, 8, "f16", seed=3)
    assert q.shape == do.shape == (1, 2, 5, 8) and k.shape == v.shape == (1, 2, 9, 8)
    g = torch.Generator().manual_seed(3)
    want_q = torch.randn((1, 2, 5, 8), generator=g).to(torch.float16)
    want_k = torch.randn((1, 2, 9, 8), generator=g).to(torch.float16)
    assert torch.equal(q, want_q) and torch.equal(k, want_k)
    # with Nq = Nk it is the square recipe
    a, b = inputs.make_qkv_cross(1, 2, 6, 6, 8, "bf16", seed=4), inputs.make_qkv(1, 2, 6, 8, "bf16", seed=4)
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_block_mask_of_the_64k_workload():
    # 128 x 128 blocks at N = 65536, diagonal kept, off-diagonal Bernoulli(0.2), seed 0:
    # the realised mask the block-sparse figures are quoted on
    m = inputs.make_block_mask(65536, 128, 0.2, seed=0)
    assert m.shape == (512, 512) and m.dtype == torch.uint8 and m.is_contiguous()
    assert torch.all(torch.diagonal(m) == 1)
    assert int(m.sum()) == 52834
    assert abs(int(m.sum()) / 512 ** 2 - 0.2015) < 1e-4
    assert set(torch.unique(m).tolist()) == {0, 1}
    # a ragged N rounds the block count up; keep_diagonal=False keeps only the draws
    assert inputs.make_block_mask(300, 128, 0.5, seed=1).shape == (3, 3)
    assert int(inputs.make_block_mask(1024, 128, 0.0, seed=2, keep_diagonal=False).sum()) == 0


def test_alibi_slopes_are_geometric():
    s = inputs.alibi_slopes(8)
    assert s.dtype == torch.float32
    assert s.tolist() == [2.0 ** -k for k in range(1, 9)]          # 1/2, 1/4, ..., 1/256
    s16 = inputs.alibi_slopes(16)
    assert abs(float(s16[0]) - 2.0 ** -0.5) < 1e-7 and float(s16[-1]) == 2.0 ** -8


def test_hadamard_signs_and_samples():
    s = inputs.hadamard_signs(128, seed=3)
    assert s.shape == (128,) and s.dtype == torch.float32
    assert set(s.tolist()) == {-1.0, 1.0}
    assert torch.equal(s, inputs.hadamard_signs(128, seed=3))
    rows = inputs.sample_rows(4096, 16, 0, 5)
    assert rows.dtype == torch.int32 and len(set(rows.tolist())) == 16
    assert torch.all(rows[1:] > rows[:-1]) and int(rows.min()) >= 0 and int(rows.max()) < 4096
    assert torch.equal(rows, inputs.sample_rows(4096, 16, 0, 5))
    assert len(inputs.sample_rows(10, 16, 0, 0)) == 10                # never more rows than exist
    cols = inputs.sample_key_blocks(512, 2, 0, 1)
    assert len(cols) == 2 and int(cols.max()) < 512
