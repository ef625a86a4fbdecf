"""Pins of the oracle's Hadamard rotation of the cache (FWHT).

"[Framework] The Asymmetric Key-Value Cache Compression", §IV stage 1:
Y = X H with an orthogonal +-1 Hadamard matrix, computed by the fast
Walsh-Hadamard transform in O(N log N); "Asymmetric Key-Value Quantization:
2-Bit Values and 4-Bit Keys under Long-Context Drift", §3.1: keys and values
quantized after an FWHT rotation.  The butterfly is pinned against the
Walsh matrix written from its closed form (entry (-1)^popcount(i & j)), the
normalized map against orthogonality, and the rotated decode against plain
attention on histories whose rotated tokens quantize exactly.
"""
import math

import numpy as np
import pytest

from oracle import kvq_oracle as o


def _walsh(d):
    i = np.arange(d)[:, None]
    j = np.arange(d)[None, :]
    bits = np.vectorize(lambda x: bin(int(x)).count("1"))(i & j)
    return np.where(bits % 2 == 0, 1.0, -1.0)


@pytest.mark.parametrize("d", [2, 16, 64, 128])
def test_butterfly_is_the_walsh_matrix(d):
    rng = np.random.default_rng(d)
    x = rng.integers(-50, 50, size=(5, d)).astype(np.float32)
    # integer inputs: every fp32 sum is exact, so the butterfly must equal
    # the matrix product exactly
    assert np.array_equal(o.fwht_fp32(x).astype(np.float64), x.astype(np.float64) @ _walsh(d))
    H = _walsh(d)
    assert np.array_equal(H @ H, d * np.eye(d))


def test_normalized_rotation_is_orthogonal_and_its_own_inverse():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((7, 128))
    y = rng.standard_normal((7, 128))
    rx, ry = o.rotate_fp64(x), o.rotate_fp64(y)
    assert np.allclose((rx * ry).sum(-1), (x * y).sum(-1), rtol=0, atol=1e-12)
    assert np.allclose(o.rotate_fp64(rx), x, rtol=0, atol=1e-13)


def test_fp16_rotation_rounds_the_scaled_butterfly():
    """fp16(butterfly * fp32(1/sqrt(d))): for d = 64 the scale is 1/8, so
    the result equals the exact rotation rounded to fp16 for integer
    inputs."""
    rng = np.random.default_rng(3)
    x = rng.integers(-300, 300, size=(4, 64)).astype(np.float32)
    want = ((x.astype(np.float64) @ _walsh(64)) / 8.0).astype(np.float16)
    assert np.array_equal(o.rotate_fp16(x).view(np.uint16), want.view(np.uint16))


def _exact_rotated_history(rng, ngroups, hkv, d, G, kb, vb):
    """Inputs x whose rotated fp16 tokens y are exactly quantizable (codes
    with 0 and Q in every group, power-of-two scales, integer mins): y is
    built first and x = y H / sqrt(d) in float64, rounded to fp32."""
    QK, QV = 2 ** kb - 1, 2 ** vb - 1
    n = ngroups * G
    y_k = np.zeros((n, hkv, d))
    for g in range(ngroups):
        for h in range(hkv):
            for c in range(d):
                codes = rng.integers(0, QK + 1, size=G)
                codes[0], codes[1] = 0, QK
                rng.shuffle(codes)
                y_k[g * G:(g + 1) * G, h, c] = float(rng.integers(-2, 2)) + 0.25 * codes
    y_v = np.zeros((n, hkv, d))
    for t in range(n):
        for h in range(hkv):
            for j in range(d // G):
                codes = rng.integers(0, QV + 1, size=G)
                codes[0], codes[1] = 0, QV
                rng.shuffle(codes)
                y_v[t, h, j * G:(j + 1) * G] = float(rng.integers(-2, 2)) + 0.5 * codes
    xk = o.rotate_fp64(y_k).astype(np.float32)
    xv = o.rotate_fp64(y_v).astype(np.float32)
    return xk, xv, y_k, y_v


def test_rotated_decode_is_plain_attention_when_rotated_tokens_quantize_exactly():
    rng = np.random.default_rng(11)
    G, d, hkv, gqa = 32, 64, 1, 2
    cfg = o.Config(4, 2, G, d, hkv * gqa, hkv, rotate=True)
    xk, xv, y_k, y_v = _exact_rotated_history(rng, 2, hkv, d, G, 4, 2)
    # the cache's fp32 rotation of the fp32 inputs lands on y exactly
    assert np.array_equal(o.rotate_fp16(xk).astype(np.float64), y_k)
    assert np.array_equal(o.rotate_fp16(xv).astype(np.float64), y_v)
    q = rng.standard_normal((hkv * gqa, d))
    got = o.decode(cfg, xk, xv, q)
    want = o.attention(q, xk.astype(np.float64), xv.astype(np.float64), gqa)
    assert np.abs(got - want).max() <= 1e-5
    # without the rotation the same inputs do not quantize exactly
    c0 = o.Config(4, 2, G, d, hkv * gqa, hkv)
    assert np.abs(o.decode(c0, xk, xv, q) - want).max() > 1e-3


def test_rotated_decode_with_everything_in_fp16_is_attention_up_to_fp16_rounding():
    rng = np.random.default_rng(12)
    n, d = 40, 128
    cfg = o.Config(4, 2, 32, d, 4, 2, window=64, rotate=True)
    k = rng.standard_normal((n, 2, d)).astype(np.float32)
    v = rng.standard_normal((n, 2, d)).astype(np.float32)
    q = rng.standard_normal((4, d))
    got = o.decode(cfg, k, v, q)
    want = o.attention(q, k.astype(np.float64), v.astype(np.float64), 2)
    err = np.abs(got - want).max()
    assert err <= 2e-3, err      # fp16 storage of the rotated tokens only
    assert err > 0
