"""Pins for the oracle's quantizer (CPU only).

The quantizer is the uniform asymmetric min/scale reading of the KIVI-style
scheme ("[Framework] The Asymmetric Key-Value Cache Compression", §III;
per-group asymmetric quantization in the InnerQ abstract on the "WUSH-KV"
page).  Pins: hand-worked examples (tests/golden/quantizer_examples.json),
the nearest-level property checked by brute force over every code, the
half-step error bound, the per-channel / per-token grouping behaviour the
first page describes, and its absmax counter-example (§II).
"""
import json
import os

import numpy as np
import pytest

from oracle import kvq_oracle as o

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    with open(os.path.join(GOLD, "quantizer_examples.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_hand_examples(case):
    x16 = np.array(case["x"], np.float64).astype(np.float16)
    codes, s, z = o.quantize_along(x16[None, :], case["bits"], axis=1)
    assert float(s[0]) == case["scale"]
    assert float(z[0]) == case["min"]
    assert codes[0].tolist() == case["codes"]
    deq = o.dequantize(codes[0], s[0], z[0])
    np.testing.assert_array_equal(deq, np.array(case["dequant"], np.float64))


def _brute_nearest(x, s, z, Q):
    """All codes tried in float64; returns (best code, gap to second best)."""
    levels = np.arange(Q + 1, dtype=np.float64) * s[..., None] + z[..., None]
    dist = np.abs(x[..., None] - levels)
    order = np.argsort(dist, axis=-1, kind="stable")
    best = order[..., 0]
    gap = np.take_along_axis(dist, order[..., 1:2], -1)[..., 0] - \
        np.take_along_axis(dist, order[..., 0:1], -1)[..., 0]
    return best, gap


@pytest.mark.parametrize("bits", [2, 4])
def test_code_is_nearest_level(bits):
    """Every code is the level nearest to x among all 2^b levels (brute force
    in float64), except where two levels are within fp32 rounding of a tie."""
    rng = np.random.default_rng(1)
    Q = 2 ** bits - 1
    x = (rng.standard_normal((500, 32)) * np.exp(rng.standard_normal((500, 1)))).astype(np.float16)
    codes, s, z = o.quantize_along(x, bits, axis=1)
    s64 = s.astype(np.float64)[:, None]
    z64 = z.astype(np.float64)[:, None]
    x64 = x.astype(np.float64)
    best, gap = _brute_nearest(x64, s64, z64, Q)
    ok = (codes == best) | (gap <= 4 * np.abs(x64) * 2.0 ** -23 + s64 * 2.0 ** -21)
    assert ok.all()
    assert (codes == best).mean() > 0.999


@pytest.mark.parametrize("bits", [2, 4])
def test_error_within_half_step(bits):
    """|x - x_hat| <= s/2 for x inside [z, z + Q s]; outside, the error is the
    distance to the clamped end level plus at most s/2."""
    rng = np.random.default_rng(2)
    Q = 2 ** bits - 1
    x = (rng.standard_normal((400, 64)) * 3).astype(np.float16)
    codes, s, z = o.quantize_along(x, bits, axis=1)
    x64 = x.astype(np.float64)
    s64 = s.astype(np.float64)[:, None]
    z64 = z.astype(np.float64)[:, None]
    xh = o.dequantize(codes, s64, z64)
    lo, hi = z64, z64 + Q * s64
    inside = (x64 >= lo) & (x64 <= hi)
    slack = np.abs(x64) * 2.0 ** -22 + 1e-12
    err = np.abs(x64 - xh)
    assert (err <= np.where(inside, s64 / 2 + slack, np.inf)).all()
    out_err = np.maximum(lo - x64, x64 - hi)
    assert (err <= np.where(inside, np.inf, out_err + s64 / 2 + slack)).all()
    # the stored range covers the data up to fp16 rounding of s and z
    assert (np.abs(lo - x64.min(1, keepdims=True)) <= np.abs(x64).max(1, keepdims=True) * 2.0 ** -11).all()


def test_keys_grouped_per_channel_outlier_column():
    """An outlier channel in K changes only its own (scale, min); the other
    channels keep their own step (first page §III: key outliers are
    channel-wise, so K is quantized per channel)."""
    rng = np.random.default_rng(3)
    G, d = 32, 64
    k = rng.standard_normal((G, d))
    base_c, base_s, base_z = o.quantize_keys(k.astype(np.float16), 4)
    k2 = k.copy()
    k2[:, 7] = 1000.0 * (1.0 + 0.1 * k[:, 7])
    c2, s2, z2 = o.quantize_keys(k2.astype(np.float16), 4)
    others = np.arange(d) != 7
    np.testing.assert_array_equal(s2[others], base_s[others])
    np.testing.assert_array_equal(z2[others], base_z[others])
    np.testing.assert_array_equal(c2[:, others], base_c[:, others])
    assert float(s2[7]) > 50 * float(base_s[7])
    # reconstruction of the normal channels stays within their own half step
    deq = o.dequantize_keys(c2, s2, z2)
    err = np.abs(deq - k2.astype(np.float16).astype(np.float64))[:, others]
    assert (err <= s2[others].astype(np.float64) / 2 + 1e-6).all()
    # the same column quantized per token would be flattened: per-token
    # grouping of this K gives most normal channels one shared code per token
    pt_c, pt_s, _ = o.quantize_values(k2.astype(np.float16), 4, d)
    assert (pt_s.astype(np.float64) > 30).all()
    flattened = (pt_c[:, others] == np.median(pt_c[:, others], axis=1, keepdims=True)).mean()
    assert flattened > 0.9


def test_values_grouped_per_token_outlier_row():
    """An outlier token in V changes only that token's pairs (first page
    §III: value outliers are tied to tokens, so V is quantized per token)."""
    rng = np.random.default_rng(4)
    T, d, G = 32, 64, 32
    v = rng.standard_normal((T, d))
    c0, s0, z0 = o.quantize_values(v.astype(np.float16), 2, G)
    v2 = v.copy()
    v2[11] *= 500.0
    c2, s2, z2 = o.quantize_values(v2.astype(np.float16), 2, G)
    others = np.arange(T) != 11
    np.testing.assert_array_equal(s2[others], s0[others])
    np.testing.assert_array_equal(z2[others], z0[others])
    np.testing.assert_array_equal(c2[others], c0[others])
    assert (s2[11].astype(np.float64) > 100 * s0[11].astype(np.float64)).all()


def test_absmax_counter_example():
    """First page §II: symmetric absmax scaling of [0.1, 0.12, 0.08, 1e5, 0.11]
    by S = 127 / 1e5 sends the normal features to 0.  Per-channel asymmetric
    quantization of a token stream with that outlier channel keeps them.

    The outlier is 1e4 here: the cache stores fp16, whose largest finite
    value is 65504."""
    feats = np.array([0.1, 0.12, 0.08, 1e5, 0.11])
    S = 127 / 1e5
    absmax = np.rint(feats * S)
    assert absmax.tolist() == [0, 0, 0, 127, 0]
    rng = np.random.default_rng(5)
    base = np.array([0.1, 0.12, 0.08, 1e4, 0.11])
    toks = base[None, :] * (1 + 0.2 * rng.standard_normal((32, 5)))
    x16 = toks.astype(np.float16)
    codes, s, z = o.quantize_keys(x16, 4)
    normal = [0, 1, 2, 4]
    assert (codes[:, normal].max(axis=0) == 15).all()
    assert (codes[:, normal].min(axis=0) == 0).all()
    deq = o.dequantize_keys(codes, s, z)
    rel = np.abs(deq[:, normal] - x16[:, normal].astype(np.float64)) / 0.1
    assert rel.max() < 0.05
