"""Pins for the oracle's byte accounting against the pages' closed forms (CPU).

* "Asymmetric Key-Value Quantization ...", §3.1: (4 + 2) / 2 = 3 bits per
  coordinate, 5.3x versus fp16; §3.4: 2.0 average bits -> 8.0x.
* same page, §5.4: a 7B model at 262k tokens holds 137.4 GB of fp16 KV and
  25.8 GB at 3 bits (metadata ignored, as the page does).
"""
import pytest

from oracle import kvq_oracle as o


def test_average_bits_and_ratio_without_metadata():
    assert o.bits_per_coordinate(4, 2) == 3.0
    assert round(o.compression_vs_fp16(4, 2), 1) == 5.3
    assert o.compression_vs_fp16(4, 2) == pytest.approx(16 / 3)
    assert o.compression_vs_fp16(3, 1) == 8.0        # AKVQ-Aggressive row
    assert o.compression_vs_fp16(2, 2) == 8.0        # 2-bit KIVI row of the table


def test_seven_b_model_at_262k():
    fp16 = o.kv_cache_bytes_fp16(layers=32, heads=32, head_dim=128, tokens=262144)
    assert fp16 == 137_438_953_472
    assert round(fp16 / 1e9, 1) == 137.4
    three_bit = fp16 * o.bits_per_coordinate(4, 2) / 16
    assert round(three_bit / 1e9, 1) == 25.8


@pytest.mark.parametrize("kb,vb,G,ratio", [(4, 2, 32, 4.0), (2, 2, 32, 16 / 3), (4, 2, 64, 512 / 112)])
def test_ratio_with_fp16_metadata(kb, vb, G, ratio):
    """With one fp16 (scale, min) pair per group the real ratio is lower than
    the pages' figure; it must agree with the block size of LAYOUT v2."""
    assert o.compression_vs_fp16(kb, vb, G, with_metadata=True) == pytest.approx(ratio)
    cfg = o.Config(kb, vb, G, 128, 1, 1)
    assert o.fp16_bytes_per_token_head(128) / o.bytes_per_token_head(cfg) == pytest.approx(ratio)
