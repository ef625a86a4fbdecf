"""Pins for the oracle's position-adaptive key bits (CPU only).

"Asymmetric Key-Value Quantization: 2-Bit Values and 4-Bit Keys under
Long-Context Drift", §3.2: bit widths by position with a window Delta
(default 1024).  Reading taken (the page's formula and its rationale
disagree on the early tokens): 4-bit keys for the early groups (positions
< Delta) and the recent ones (last position >= n - Delta), 2-bit keys in the
middle; a 4-bit group that ages into the middle is requantized from its
dequantized keys.  Pinned here: hand-worked requantization examples, the
widths after any append history against a closed form of the region sizes
derived separately, the key bytes per sequence in closed form, decode equal
to plain attention on keys exactly representable at both widths whatever
the history, the history dependence of the bytes (not of the widths), a
prefill's blocks equal to the plain 4-bit and 2-bit caches' blocks group by
group, and Delta beyond the length reducing to the plain 4-bit cache and
its decode.
"""
import dataclasses
import json
import math
import os

import numpy as np
import pytest

from oracle import kvq_oracle as o

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    with open(os.path.join(GOLD, "akvq_requantize_examples.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_requantization_hand_examples(case):
    kc = np.array(case["codes4"], np.uint8)[:, None]              # [G=4 tokens, 1 channel]
    ks = np.array([case["scale4"]], np.float64).astype(np.float16)
    kz = np.array([case["min4"]], np.float64).astype(np.float16)
    c2, s2, z2 = o.akvq_requantize_keys(ks, kz, kc)
    assert c2[:, 0].tolist() == case["codes2"]
    assert float(s2[0]) == case["scale2"] and float(z2[0]) == case["min2"]


def _cfg(G, delta, d=64, hkv=1):
    return o.Config(4, 2, G, d, hkv, hkv, akvq_delta=delta)   # the layout's head dims: 64, 128


def _histories(rng, n, G):
    yield [n]                                   # one prefill
    yield [1] * n                               # one token at a time
    chunks, left = [], n
    while left:
        c = int(min(left, rng.integers(1, 3 * G)))
        chunks.append(c)
        left -= c
    yield chunks


def _two_bit_groups_closed_form(n, G, delta):
    # middle groups: first position >= Delta (group index >= Delta / G) and
    # last position < n - Delta, i.e. (g + 1) G <= n - Delta
    ng = n // G
    hi = min(ng, max(0, (n - delta) // G)) if n >= delta else 0
    return max(0, hi - delta // G)


@pytest.mark.parametrize("G,delta", [(32, 32), (32, 128), (64, 256), (32, 1024)])
def test_widths_after_any_history(G, delta):
    cfg = _cfg(G, delta)
    rng = np.random.default_rng(G + delta)
    for n in sorted({1, G, delta, delta + G - 1, 2 * delta, 2 * delta + 5 * G + 3,
                     3 * delta + 7}):
        k = rng.standard_normal((n, 1, 64)).astype(np.float16)
        for chunks in _histories(rng, n, G):
            img = o.akvq_cache_image(cfg, k, k, chunks)
            ng = n // G
            assert img["bits"] == [o.akvq_key_bits(cfg, g, n) for g in range(ng)]
            assert sum(b == 2 for b in img["bits"]) == _two_bit_groups_closed_form(n, G, delta)
            # early groups keep 4 bits for ever
            assert all(b == 4 for b in img["bits"][:delta // G])


def test_key_bytes_closed_form():
    """Key bytes of a sequence: 4-bit groups G d / 2 + 4 d bytes, 2-bit groups
    G d / 4 + 4 d; the packed slots hold exactly that many key bytes."""
    G, delta, d = 32, 256, 64
    cfg = _cfg(G, delta, d)
    rng = np.random.default_rng(5)
    for n in (100, 600, 1500, 3000):
        k = rng.standard_normal((n, 1, d)).astype(np.float16)
        img = o.akvq_cache_image(cfg, k, k, [n])
        ng = n // G
        n2 = _two_bit_groups_closed_form(n, G, delta)
        want = (ng - n2) * (G * d // 2 + 4 * d) + n2 * (G * d // 4 + 4 * d)
        got = 0
        for b in img["bits"]:
            sec = o.block_sections(dataclasses.replace(cfg, k_bits=b))
            got += sec["kcodes"][1] + sec["kscale"][1] + sec["kmin"][1]
        assert got == want
        assert img["blocks"].shape == (1, ng, o.block_bytes(cfg))


def _exact_history(rng, n, G, d):
    """Keys whose every (group, channel) takes values z + j S, j in 0..3, with
    S = 5 u and u a power of two: exactly quantizable at 4 bits (scale u,
    codes 5 j), their dequantized values exactly quantizable at 2 bits (scale
    S, codes j); values exactly quantizable at 2 bits per token group."""
    k = np.zeros((n, 1, d))
    for g0 in range(0, n, G):
        for c in range(d):
            u = 2.0 ** int(rng.integers(-6, -2))
            z = u * round(rng.standard_normal() / u)   # a multiple of u: every level is fp16
            j = rng.integers(0, 4, size=min(G, n - g0))
            j[0], j[-1] = 0, 3          # both ends of the range present
            k[g0:g0 + len(j), 0, c] = z + j * 5 * u
    v = np.zeros((n, 1, d))
    for t in range(n):
        for j0 in range(0, d, G if G <= d else d):
            w = min(G, d)
            u = 2.0 ** int(rng.integers(-5, -1))
            z = u * round(rng.standard_normal() / u)
            j = rng.integers(0, 4, size=w)
            j[0], j[-1] = 0, 3
            v[t, 0, j0:j0 + w] = z + j * u
    return k.astype(np.float16), v.astype(np.float16)


def test_decode_equals_attention_on_exact_keys():
    G, delta, d = 32, 64, 64
    cfg = _cfg(G, delta, d)
    rng = np.random.default_rng(11)
    n = 300
    k, v = _exact_history(rng, n, G, d)
    q = rng.standard_normal((1, d))
    want = o.attention(q, k, v, 1)
    for chunks in _histories(rng, n, G):
        got = o.akvq_decode(cfg, k, v, q, chunks)
        assert np.abs(got - want).max() < 1e-12, chunks


def test_bytes_depend_on_the_history_widths_do_not():
    G, delta, d = 32, 64, 64
    cfg = _cfg(G, delta, d)
    rng = np.random.default_rng(12)
    n = 400
    k = rng.standard_normal((n, 1, d)).astype(np.float16)
    a = o.akvq_cache_image(cfg, k, k, [n])
    b = o.akvq_cache_image(cfg, k, k, [1] * n)
    assert a["bits"] == b["bits"]
    two = [g for g, bits in enumerate(a["bits"]) if bits == 2]
    assert two
    # a middle group quantized straight from fp16 keys differs from one that
    # went through 4 bits first, for some group; early / recent groups agree
    assert any(not np.array_equal(a["blocks"][:, g], b["blocks"][:, g]) for g in two)
    for g, bits in enumerate(a["bits"]):
        if bits == 4:
            assert np.array_equal(a["blocks"][:, g], b["blocks"][:, g])


def test_prefill_image_selects_plain_k4_and_k2_blocks():
    """One append (a prefill): every group is quantized from its fp16 keys at
    its width, so its block is the plain 4-bit cache's block or the plain
    2-bit cache's block (from the start of the slot), group by group."""
    G, delta, d = 32, 96, 64
    cfg = _cfg(G, delta, d)
    rng = np.random.default_rng(21)
    n = 20 * G + 11
    k = (rng.standard_normal((n, 2, d)) * np.exp(rng.standard_normal((1, 2, d)))).astype(np.float16)
    v = rng.standard_normal((n, 2, d)).astype(np.float16)
    img = o.akvq_cache_image(cfg, k, v, [n])
    c4 = o.cache_image(dataclasses.replace(cfg, akvq_delta=0), k, v)
    c2 = o.cache_image(dataclasses.replace(cfg, k_bits=2, akvq_delta=0), k, v)
    n2 = o.block_sections(dataclasses.replace(cfg, k_bits=2))["total"][1]
    assert set(img["bits"]) == {2, 4}
    for g, bits in enumerate(img["bits"]):
        if bits == 4:
            assert np.array_equal(img["blocks"][:, g], c4["blocks"][:, g])
        else:
            assert np.array_equal(img["blocks"][:, g, :n2], c2["blocks"][:, g])
            assert not img["blocks"][:, g, n2:].any()


@pytest.mark.parametrize("chunks", [[700], [1] * 700, [5, 300, 1, 1, 393]])
def test_delta_beyond_the_length_is_the_plain_4bit_cache(chunks):
    """Delta >= n: every group is early or recent, so the cache is the plain
    4-bit cache whatever the history, and so is the decode."""
    G, d = 32, 64
    n = sum(chunks)
    cfg = _cfg(G, 1024, d)
    rng = np.random.default_rng(22)
    k = rng.standard_normal((n, 1, d)).astype(np.float16)
    v = rng.standard_normal((n, 1, d)).astype(np.float16)
    q = rng.standard_normal((1, d))
    img = o.akvq_cache_image(cfg, k, v, chunks)
    plain = dataclasses.replace(cfg, akvq_delta=0)
    c4 = o.cache_image(plain, k, v)
    assert img["bits"] == [4] * (n // G)
    assert np.array_equal(img["blocks"], c4["blocks"])
    assert np.allclose(o.akvq_decode(cfg, k, v, q, chunks), o.decode(plain, k, v, q), rtol=0,
                       atol=1e-12)
