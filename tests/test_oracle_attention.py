"""Pins for the oracle's attention and decode (CPU only).

Decode attention is out_h = sum_t alpha_t v_t with
alpha = softmax(q_h . k_t / sqrt(d)) ("Asymmetric Key-Value Quantization:
2-Bit Values and 4-Bit Keys under Long-Context Drift", §1 and §2.1).  Pins:
a hand-worked example (tests/golden/attention_example.json), a brute-force
pure-Python softmax on tiny inputs, special cases with closed forms
(one token, identical keys, q = 0, shifted keys), the GQA head mapping, the
fp16 tail being exact, and a cache whose quantization is exact by
construction so that decode must equal plain attention on the raw values.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import kvq_oracle as o

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_example():
    with open(os.path.join(GOLD, "attention_example.json")) as f:
        g = json.load(f)
    q = np.array([g["q"]])
    k = np.array(g["k"])[:, None, :]
    v = np.array(g["v"])[:, None, :]
    alpha = o.attention_weights(q[0], k[:, 0])
    np.testing.assert_allclose(alpha, g["alpha"], rtol=0, atol=1e-15)
    out = o.attention(q, k, v)
    np.testing.assert_allclose(out[0], g["out"], rtol=0, atol=1e-15)


def _brute(q, k, v):
    """Textbook softmax attention with Python floats, one term at a time."""
    d = len(q)
    logits = []
    for kt in k:
        s = 0.0
        for a, b in zip(q, kt):
            s += a * b
        logits.append(s / math.sqrt(d))
    m = max(logits)
    w = [math.exp(x - m) for x in logits]
    tot = math.fsum(w)
    return [math.fsum(wi * vt[c] for wi, vt in zip(w, v)) / tot for c in range(d)]


def test_brute_force_tiny():
    rng = np.random.default_rng(11)
    for n in (1, 2, 5, 17, 40):
        for d in (4, 8):
            q = rng.standard_normal(d) * 2
            k = rng.standard_normal((n, d)) * 2
            v = rng.standard_normal((n, d))
            ref = _brute(q.tolist(), k.tolist(), v.tolist())
            out = o.attention(q[None], k[:, None], v[:, None])[0]
            np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_weights_sum_to_one():
    rng = np.random.default_rng(12)
    for n in (1, 3, 100, 4113):
        a = o.attention_weights(rng.standard_normal(64) * 3, rng.standard_normal((n, 64)) * 3)
        assert abs(a.sum() - 1.0) < 1e-12
        assert (a >= 0).all()


def test_single_token_returns_its_value():
    rng = np.random.default_rng(13)
    v = rng.standard_normal((1, 2, 16))
    out = o.attention(rng.standard_normal((4, 16)), rng.standard_normal((1, 2, 16)), v, gqa=2)
    for h in range(4):
        np.testing.assert_array_equal(out[h], v[0, h // 2])


def test_identical_keys_or_zero_query_give_mean():
    rng = np.random.default_rng(14)
    n, d = 37, 16
    v = rng.standard_normal((n, 1, d))
    k_same = np.repeat(rng.standard_normal((1, 1, d)), n, axis=0)
    out = o.attention(rng.standard_normal((1, d)), k_same, v)
    np.testing.assert_allclose(out[0], v[:, 0].mean(0), rtol=0, atol=1e-14)
    out0 = o.attention(np.zeros((1, d)), rng.standard_normal((n, 1, d)), v)
    np.testing.assert_allclose(out0[0], v[:, 0].mean(0), rtol=0, atol=1e-14)


def test_shifting_all_keys_changes_nothing():
    """Adding one vector u to every key adds q.u to every logit."""
    rng = np.random.default_rng(15)
    n, d = 50, 32
    q = rng.standard_normal((1, d))
    k = rng.standard_normal((n, 1, d))
    v = rng.standard_normal((n, 1, d))
    u = rng.standard_normal(d) * 10
    a = o.attention(q, k, v)
    b = o.attention(q, k + u, v)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_gqa_mapping():
    """Hq = 8, Hkv = 2: heads 0-3 read kv head 0, heads 4-7 read kv head 1."""
    rng = np.random.default_rng(16)
    n, d = 9, 16
    k = np.repeat(rng.standard_normal((1, 2, d)), n, axis=0)   # identical keys per head
    v = rng.standard_normal((n, 2, d))
    out = o.attention(rng.standard_normal((8, d)), k, v, gqa=4)
    for h in range(8):
        np.testing.assert_allclose(out[h], v[:, h // 4].mean(0), atol=1e-14)


def test_empty_context_is_an_error():
    with pytest.raises(ValueError):
        o.attention(np.zeros((1, 8)), np.zeros((0, 1, 8)), np.zeros((0, 1, 8)))


def test_tail_only_context_is_exact_fp16_attention():
    """With fewer than G tokens everything sits in the fp16 tail (the FP16
    window of the first page, §III): decode equals attention on the fp16
    values."""
    cfg = o.Config(4, 2, 32, 64, 2, 1)
    rng = np.random.default_rng(17)
    n = 31
    k16 = rng.standard_normal((n, 1, 64)).astype(np.float16)
    v16 = rng.standard_normal((n, 1, 64)).astype(np.float16)
    q = rng.standard_normal((2, 64))
    out = o.decode(cfg, k16, v16, q)
    ref = o.attention(q, k16.astype(np.float64), v16.astype(np.float64), gqa=2)
    np.testing.assert_array_equal(out, ref)


def _exactly_quantizable(rng, n_groups, G, d, kb, vb):
    """Keys/values whose min/scale quantization is exact: each key channel of
    each group is z + s * code with codes covering 0..Q, s a power of two and
    z a small multiple of s; each value channel group of each token likewise."""
    Qk, Qv = 2 ** kb - 1, 2 ** vb - 1
    n = n_groups * G
    k = np.zeros((n, d))
    for g in range(n_groups):
        for c in range(d):
            s = 2.0 ** rng.integers(-6, 2)
            z = s * rng.integers(-40, 40)
            codes = rng.integers(0, Qk + 1, G)
            codes[rng.integers(0, G)] = 0
            codes[(rng.integers(1, G) + np.argmin(codes)) % G] = Qk
            k[g * G:(g + 1) * G, c] = z + s * codes
    v = np.zeros((n, d))
    J = d // G
    for t in range(n):
        for j in range(J):
            s = 2.0 ** rng.integers(-6, 2)
            z = s * rng.integers(-40, 40)
            codes = rng.integers(0, Qv + 1, G)
            codes[0], codes[-1] = 0, Qv
            v[t, j * G:(j + 1) * G] = z + s * codes
    return k, v


@pytest.mark.parametrize("kb,vb,G,d", [(4, 2, 32, 64), (2, 2, 32, 64), (4, 2, 64, 64)])
def test_exactly_quantizable_cache_decodes_exactly(kb, vb, G, d):
    """When every group is exactly representable, quantize -> pack -> unpack ->
    dequantize must reproduce the inputs bit for bit and decode must equal
    plain attention on them (a dropped min, a swapped scale, a wrong group
    axis or a GQA slip all break this)."""
    rng = np.random.default_rng(18)
    cfg = o.Config(kb, vb, G, d, 4, 2)
    n_groups = 3
    ks, vs = [], []
    for _ in range(2):
        k, v = _exactly_quantizable(rng, n_groups, G, d, kb, vb)
        ks.append(k)
        vs.append(v)
    k16 = np.stack(ks, axis=1).astype(np.float16)
    v16 = np.stack(vs, axis=1).astype(np.float16)
    assert np.array_equal(k16.astype(np.float64), np.stack(ks, 1))
    tail = 5
    k16 = np.concatenate([k16, rng.standard_normal((tail, 2, d)).astype(np.float16)])
    v16 = np.concatenate([v16, rng.standard_normal((tail, 2, d)).astype(np.float16)])
    img = o.cache_image(cfg, k16, v16)
    assert img["N"] == n_groups * G and img["T"] == tail
    back = o.unpack_blocks(cfg, img["blocks"])
    kh_, vh_ = o.dequantized_cache(cfg, k16, v16)
    np.testing.assert_array_equal(kh_, k16.astype(np.float64))
    np.testing.assert_array_equal(vh_, v16.astype(np.float64))
    for a, b in zip(back, img["groups"]):
        np.testing.assert_array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
    q = rng.standard_normal((4, d))
    out = o.decode(cfg, k16, v16, q)
    ref = o.attention(q, k16.astype(np.float64), v16.astype(np.float64), gqa=2)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_path_independence_of_groups():
    """Groups depend only on their own G tokens: the image of a prefix is a
    prefix of the image (appending tokens never rewrites earlier groups)."""
    cfg = o.Config(4, 2, 32, 64, 1, 1)
    rng = np.random.default_rng(19)
    k = rng.standard_normal((100, 1, 64)).astype(np.float16)
    v = rng.standard_normal((100, 1, 64)).astype(np.float16)
    full = o.cache_image(cfg, k, v)
    part = o.cache_image(cfg, k[:70], v[:70])
    np.testing.assert_array_equal(full["blocks"][:, :2], part["blocks"])
    np.testing.assert_array_equal(part["tail_k"][0], k[64:70, 0])
