"""The cache-precision reading: every K/V element is rounded to fp16 (nearest
even) on entry.  The oracle does it with numpy's float32 -> float16 cast; this
pins that cast against a conversion written from the binary16 definition
(tests/fp16_rne.py) on a stratified set of fp32 patterns (every exponent,
ties at the fp16 spacing, the subnormal range, overflow) and on every bf16
pattern (bf16 inputs widen exactly to fp32 before the same rounding)."""
import numpy as np

from oracle import kvq_oracle as o
from tests.fp16_rne import fp16_bits_rne, stratified_fp32_patterns


def test_hand_values():
    u = np.array([0x3F800000, 0x3F801000, 0x3F802000, 0x3F803000,   # 1, 1+2^-11 (tie -> even), 1+2^-10, tie -> up
                  0x477FE000, 0x477FF000,                            # 65504, 65520 -> inf
                  0x33800000, 0x33000000, 0x33000001,                # 2^-24, 2^-25 (tie -> 0), just above -> 2^-24
                  0x38800000, 0x387FE000, 0x387FC000,                # 2^-14; 1023.5 * 2^-24 (tie -> 1024, even); 1023 * 2^-24
                  0x80000000, 0x7F800000], np.uint32)
    want = np.array([0x3C00, 0x3C00, 0x3C01, 0x3C02,
                     0x7BFF, 0x7C00,
                     0x0001, 0x0000, 0x0001,
                     0x0400, 0x0400, 0x03FF,
                     0x8000, 0x7C00], np.uint16)
    assert np.array_equal(fp16_bits_rne(u), want)


def test_oracle_fp16_matches_definition_fp32():
    u = stratified_fp32_patterns(np.random.default_rng(7))
    got = o.to_fp16(u.view(np.float32)).view(np.uint16)
    assert np.array_equal(got, fp16_bits_rne(u))


def test_oracle_fp16_matches_definition_all_bf16():
    b = np.arange(1 << 16, dtype=np.uint32)
    u = b << 16
    keep = ~np.isnan(u.view(np.float32))
    u = u[keep]
    got = o.to_fp16(u.view(np.float32)).view(np.uint16)
    assert np.array_equal(got, fp16_bits_rne(u))
