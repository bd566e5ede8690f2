"""The benchmark's FLOP/byte helpers reproduce the figures the pages print."""
import json
import os

import pytest

from flash_fwd_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_arithmetic.json")
with open(GOLDEN) as f:
    ITEMS = json.load(f)["items"]

FN = {
    "S_matrix_bytes": lambda a: acc.s_matrix_bytes(a["B"], a["H"], a["N"], a["elem"]),
    "qkv_read_bytes_one_head": lambda a: acc.qkv_read_bytes(a["N"], a["d"], a["elem"]),
    "o_write_bytes_one_head": lambda a: acc.o_write_bytes(a["N"], a["d"], a["elem"]),
    "sram_tile_bytes": lambda a: acc.sram_tile_bytes(a["Br"], a["Bc"], a["d"], a["elem"]),
    "standard_S_traffic": lambda a: acc.standard_s_traffic(a["B"], a["H"], a["N"], a["elem"]),
}


@pytest.mark.parametrize("item", ITEMS, ids=lambda i: i["name"])
def test_page_figures(item):
    got = FN[item["name"]](item["args"])
    assert abs(got - item["value"]) <= item["rel_tol"] * item["value"] + 1e-9, (got, item["value"])


def test_flop_conventions():
    # 5 products backward vs 2 forward (深度解析 section 四)
    assert acc.bwd_flops(1, 1, 128, 64) == 2.5 * acc.fwd_flops(1, 1, 128, 64)
    assert acc.fwd_flops(2, 3, 256, 64, causal=True) == acc.fwd_flops(2, 3, 256, 64) / 2
    # a fully kept block mask counts the dense work
    nb = 4
    assert acc.sparse_fwd_flops(1, 2, 64, nb * nb) == acc.fwd_flops(1, 2, nb * 128, 64)


def _visible_brute(Nq, Nk, causal, window):
    # query i sees key j iff i + off - left <= j <= i + off + right (off = Nk - Nq,
    # a negative side unbounded), and j <= i + off under causal: counted pair by pair
    off = Nk - Nq
    left, right = (-1, -1) if window is None else window
    n = 0
    for i in range(Nq):
        for j in range(Nk):
            if causal and j > i + off:
                continue
            if left >= 0 and j < i + off - left:
                continue
            if right >= 0 and j > i + off + right:
                continue
            n += 1
    return n


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (7, 7), (5, 13), (13, 5), (64, 40)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("window", [None, (0, 0), (3, -1), (-1, 2), (4, 1), (0, 6)])
def test_visible_pairs_brute_force(Nq, Nk, causal, window):
    assert acc.visible_pairs(Nq, Nk, causal, window) == _visible_brute(Nq, Nk, causal, window)


def test_visible_pairs_closed_forms():
    N = 300
    assert acc.visible_pairs(N, N) == N * N
    assert acc.visible_pairs(N, N, causal=True) == N * (N + 1) // 2
    assert acc.visible_pairs(N, N, window=(0, 0)) == N                      # the diagonal only
    assert acc.visible_pairs(N, N, causal=True, window=(10, 0)) == N * 11 - 10 * 11 // 2
    # bottom-right causal with Nq < Nk: query i sees Nk - Nq + i + 1 keys
    assert acc.visible_pairs(3, 10, causal=True) == 8 + 9 + 10
    # Nq > Nk: the first Nq - Nk queries see nothing
    assert acc.visible_pairs(10, 3, causal=True) == 1 + 2 + 3
    # the general count equals the square dense convention
    assert acc.general_fwd_flops(2, 3, 256, 256, 64) == acc.fwd_flops(2, 3, 256, 64)


def test_forward_minimum_bytes_from_the_page_figures():
    # 原理概览 section 3.4 prints one head's Q/K/V read (6.3 MB) and O write (2.1 MB);
    # eight heads of that shape plus one fp32 LSE per row is the forward's minimum
    B, H, N, d = 1, 8, 8192, 128
    per_head = acc.qkv_read_bytes(N, d, 2) + acc.o_write_bytes(N, d, 2)
    assert acc.fwd_min_bytes(B, H, N, d) == B * H * (per_head + 4 * N)
