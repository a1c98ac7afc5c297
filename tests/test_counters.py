"""The op/byte counters behind the reported TOPS, pinned to the complexity table (Table 7)."""
import os

import pytest

from quantized_gemm_moe_b200 import roofline

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "table7_complexity.txt")


def _rows():
    with open(GOLDEN) as f:
        lines = f.read().splitlines()
    for line in lines:
        line = line.strip()
        if line and not line.startswith("#"):
            yield [int(v) for v in line.split()]


@pytest.mark.parametrize("row", list(_rows()))
def test_counters_match_table7(row):
    s, d, r, nr, qe_macs, orig_macs, qe_params, orig_params = row
    assert roofline.table7_macs(s, d, r, nr) == qe_macs
    assert roofline.table7_params(d, r, nr) == qe_params
    assert s * d * d == orig_macs and d * d == orig_params
    # our counters, with d_in = d_out = d and the rank split evenly, reproduce the table
    macs = (roofline.int_ops(s, d, d) + roofline.adapter_flops(s, d, d, r // 2, nr, r // 2)) // 2
    assert macs == qe_macs
    assert roofline.layer_params(d, d, r // 2, nr, r // 2) == qe_params


def test_byte_count_terms():
    # weights dominate decode: 8192 x 29568 W4 codes + fp32 group scales (g = 128)
    b = roofline.layer_bytes(1, 8192, 29568, 128, 4, 32, 8, 4)
    codes = 8192 * 29568 // 2
    scales = 4 * 29568 * 64
    assert codes + scales < b < codes + scales + 4_000_000
    # W3 codes are 3/8 byte per weight
    assert roofline.layer_bytes(1, 8192, 29568, 128, 3, 0, 8, 0) - roofline.layer_bytes(1, 8192, 29568, 128, 4, 0, 8, 0) \
        == -(8192 * 29568) // 8
