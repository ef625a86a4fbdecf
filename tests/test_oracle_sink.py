"""Pins of the oracle's sink window (the first S tokens kept in fp16).

InnerQ abstract (page "WUSH-KV: KV Cache Quantization with Data-Adaptive
Transforms", third abstract): high-precision windows for the recent tokens
and for the attention-sink tokens.  The reading: the first S tokens of a
sequence are never quantized, key groups are cut from position S on, and
the recent window R applies to the tokens after the sink.  These tests pin
the split against the process run token by token, the groups against the
sink-free oracle on the shifted history, and the decode against plain
attention on histories whose quantized part is exactly representable.
"""
import math

import numpy as np
import pytest

from oracle import kvq_oracle as o


def _process(n_max, S, G, R):
    """(Sb, Nq, T) after each appended token: the first S tokens go to the
    sink; every later one to the tail, whose oldest G become a group when it
    holds R + G tokens."""
    Sb = Nq = T = 0
    out = [(0, 0, 0)]
    for _ in range(n_max):
        if Sb < S:
            Sb += 1
        else:
            T += 1
            if T == R + G:
                Nq += G
                T -= G
        out.append((Sb, Nq, T))
    return out


@pytest.mark.parametrize("S", [0, 4, 16, 33])
@pytest.mark.parametrize("G,R", [(32, 0), (32, 64), (64, 16)])
def test_segments_match_the_process(S, G, R):
    cfg = o.Config(4, 2, G, 64, 1, 1, window=R, sink=S)
    for n, want in enumerate(_process(S + R + 4 * G + 3, S, G, R)):
        assert o.segments(cfg, n) == want, (n, S, G, R)
        if S == 0:
            assert o.segments(cfg, n)[1:] == o.split_tokens(n, G, R)


def _hist(rng, n, hkv, d):
    k = (rng.standard_normal((n, hkv, d)) * np.exp(rng.standard_normal((1, hkv, d)))).astype(np.float16)
    v = rng.standard_normal((n, hkv, d)).astype(np.float16)
    return k, v


@pytest.mark.parametrize("S,R", [(4, 0), (16, 32), (40, 64)])
def test_sink_groups_are_the_sink_free_groups_of_the_shifted_history(S, R):
    rng = np.random.default_rng(S + R)
    G = 32
    cs = o.Config(2, 2, G, 64, 2, 1, window=R, sink=S)
    c0 = o.Config(2, 2, G, 64, 2, 1, window=R)
    for n in (S - 1, S, S + R + G - 1, S + R + G, S + R + 5 * G + 7):
        if n < 0:
            continue
        k, v = _hist(rng, n, 1, 64)
        a = o.cache_image(cs, k, v)
        b = o.cache_image(c0, k[min(n, S):], v[min(n, S):])
        assert np.array_equal(a["blocks"], b["blocks"])
        assert a["Sb"] == min(n, S) and a["N"] == a["Sb"] + b["N"] and a["T"] == b["T"]
        assert np.array_equal(a["sink_k"][0], k[:a["Sb"], 0])
        assert np.array_equal(a["tail_k"][0], k[a["N"]:, 0])


def _exact_groups(rng, ngroups, hkv, d, G, kb, vb):
    """[ngroups*G, hkv, d] fp16 tokens whose key groups (G tokens x channel)
    and value groups (token x G channels) are exactly representable: codes
    in [0, Q] including 0 and Q, power-of-two scales, small integer mins."""
    QK, QV = 2 ** kb - 1, 2 ** vb - 1
    n = ngroups * G
    k = np.zeros((n, hkv, d))
    for g in range(ngroups):
        for h in range(hkv):
            for c in range(d):
                codes = rng.integers(0, QK + 1, size=G)
                codes[rng.integers(G)] = 0
                codes[(rng.integers(G - 1) + 1 + np.argmin(codes)) % G] = QK
                s = 2.0 ** rng.integers(-3, 2)
                z = float(rng.integers(-4, 4))
                k[g * G:(g + 1) * G, h, c] = z + s * codes
    v = np.zeros((n, hkv, d))
    for t in range(n):
        for h in range(hkv):
            for j in range(d // G):
                codes = rng.integers(0, QV + 1, size=G)
                codes[0], codes[1] = 0, QV
                rng.shuffle(codes)
                s = 2.0 ** rng.integers(-3, 1)
                z = float(rng.integers(-2, 2))
                v[t, h, j * G:(j + 1) * G] = z + s * codes
    return k.astype(np.float16), v.astype(np.float16)


def _plain_attention(q, k, v, gqa):
    hq, d = q.shape
    out = np.zeros((hq, d))
    for h in range(hq):
        kv = h // gqa
        logits = [sum(float(q[h, c]) * float(k[t, kv, c]) for c in range(d)) / math.sqrt(d)
                  for t in range(k.shape[0])]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = sum(w)
        for c in range(d):
            out[h, c] = sum(w[t] * float(v[t, kv, c]) for t in range(k.shape[0])) / z
    return out


@pytest.mark.parametrize("S,R", [(5, 0), (16, 32)])
def test_decode_with_sink_is_plain_attention_when_the_groups_are_exact(S, R):
    """Sink and tail tokens random (not quantizable), the groups in between
    exactly representable: the decode must equal attention on the raw
    history; quantizing a sink token, or cutting the groups elsewhere,
    breaks the equality."""
    rng = np.random.default_rng(9 + S)
    G, d, hkv, gqa = 32, 32, 1, 2
    cfg = o.Config(4, 2, G, d, hkv * gqa, hkv, window=R, sink=S)
    ks, vs = _hist(rng, S, hkv, d)
    kq, vq = _exact_groups(rng, 2, hkv, d, G, 4, 2)
    kt, vt = _hist(rng, R + 7, hkv, d)
    k = np.concatenate([ks, kq, kt])
    v = np.concatenate([vs, vq, vt])
    Sb, Nq, T = o.segments(cfg, k.shape[0])
    assert (Sb, Nq, T) == (S, 2 * G, R + 7)
    q = rng.standard_normal((hkv * gqa, d))
    got = o.decode(cfg, k, v, q)
    want = _plain_attention(q, k, v, gqa)
    assert np.abs(got - want).max() <= 1e-12
    # the same history read as sink-free: the random sink tokens land in a
    # quantized group, which is no longer exact
    c0 = o.Config(4, 2, G, d, hkv * gqa, hkv, window=R)
    assert np.abs(o.decode(c0, k, v, q) - want).max() > 1e-6


def test_sink_covering_the_context_is_plain_fp16_attention():
    rng = np.random.default_rng(21)
    n, d = 20, 16
    cfg = o.Config(4, 2, 32, d, 2, 1, sink=64)
    k, v = _hist(rng, n, 1, d)
    q = rng.standard_normal((2, d))
    assert o.segments(cfg, n) == (n, 0, 0)
    assert np.abs(o.decode(cfg, k, v, q) - _plain_attention(q, k, v, 2)).max() <= 1e-12


@pytest.mark.parametrize("S", [4, 16, 33])
def test_sink_shifts_the_tail_ring(S):
    """With a sink the tail ring holds the tokens after it exactly as the
    sink-free ring holds the shifted sequence; slots stay distinct."""
    G, R = 32, 64
    cs = o.Config(4, 2, G, 64, 1, 1, window=R, sink=S)
    c0 = o.Config(4, 2, G, 64, 1, 1, window=R)
    for n in range(S, S + R + 4 * G):
        Sb, Nq, T = o.segments(cs, n)
        slots = [o.tail_slot(cs, p) for p in range(Sb + Nq, n)]
        assert slots == [o.tail_slot(c0, p - S) for p in range(Sb + Nq, n)]
        assert len(set(slots)) == T and all(0 <= x < R + G for x in slots)
    assert o.sink_slots(cs) % 16 == 0 and S <= o.sink_slots(cs) < S + 16
