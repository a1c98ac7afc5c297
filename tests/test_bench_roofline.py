"""bench.py's roofline bookkeeping, on CPU: which kernel a layer set's product is attributed to,
which bound applies, and that `achieved` is the algorithmic work over the measured time."""
import os
import sys

import pytest

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import qe_inputs as qi  # noqa: E402
from quantized_gemm_moe_b200 import roofline  # noqa: E402

PEAKS = {"hbm_gbs": 6553.0, "bf16_tflops": 1640.9, "source": "measured"}
INT8 = {"peak": 3281.8, "source": "2 x bf16"}


def _layers(cfg):
    return [{"proj": p} for p in cfg.projections]


@pytest.mark.parametrize("name,T", [("decode72b_w4a8", 16), ("decode72b_w3a16", 1), ("decode72b_w4a8_s16", 16)])
def test_decode_sets_are_the_decode_product_at_hbm(name, T):
    cfg = qi.CONFIGS[name]
    r = bench.product_roofline(cfg, _layers(cfg), T, 0.2, PEAKS, INT8, None)
    assert r["kernel"] == "qdec" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    wonly = cfg.a_bits == 16
    by = sum(roofline.layer_bytes(T, p.d_in, p.d_out, cfg.group, cfg.w_bits, cfg.rank_shared, cfg.n_routed,
                                  cfg.rank_routed, 2 if wonly else 1, 2, 2 if cfg.scale_fp16 else 4)
             for p in cfg.projections)
    assert r["achieved"] == pytest.approx(by / 0.2e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6553.0)
    # the three projections stream about 3 x 121 MB of 4-bit codes (3-bit: 3 x 91 MB)
    codes = sum(p.d_in * p.d_out * cfg.w_bits / 8 for p in cfg.projections)
    assert codes <= by <= 1.2 * codes


def test_prefill_is_the_int8_gemm_at_the_int8_peak():
    cfg = qi.CONFIGS["qwen2vl72b"]
    r = bench.product_roofline(cfg, _layers(cfg), cfg.T, 10.0, PEAKS, INT8, None)
    assert r["kernel"] == "qgemm" and r["bound"] == "tensor" and r["unit"] == "TOP/s"
    ints = sum(2 * cfg.T * p.d_in * p.d_out for p in cfg.projections)
    assert r["achieved"] == pytest.approx(ints / 10.0e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 3281.8)


def test_weight_only_prefill_is_the_bf16_gemm():
    cfg = qi.CONFIGS["qwen2vl2b_w3a16"]
    r = bench.product_roofline(cfg, _layers(cfg), cfg.T, 1.0, PEAKS, INT8, None)
    assert r["kernel"] == "wgemm" and r["unit"] == "TFLOP/s"
    assert r["frac"] == pytest.approx(r["achieved"] / 1640.9)
