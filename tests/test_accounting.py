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
