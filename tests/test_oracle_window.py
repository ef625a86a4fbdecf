"""Pins of the oracle's recent fp16 window (R tokens beyond the partial group).

"[Framework] The Asymmetric Key-Value Cache Compression", §III and §V: the
most recent tokens (32 to 128 of them) stay in FP16.  The reading: a group is
quantized once R newer tokens follow it, i.e. the tail is flushed G tokens at
a time when it reaches R + G tokens.  These tests pin the oracle's closed
form against that process run token by token, and the rest of the windowed
cache against what must not change (group contents, exact tail, plain
attention when the window covers everything).
"""
import math

import numpy as np
import pytest

from oracle import kvq_oracle as o


def _flush_process(n_max: int, G: int, R: int):
    """(N, T) after every append of one token, by the flush rule itself:
    append to the tail; when the tail holds R + G tokens, its oldest G become
    the next group."""
    N, T, out = 0, 0, [(0, 0)]
    for _ in range(n_max):
        T += 1
        if T == R + G:
            N += G
            T -= G
        out.append((N, T))
    return out


@pytest.mark.parametrize("G", [32, 64])
@pytest.mark.parametrize("R", [0, 16, 32, 64, 128])
def test_split_matches_the_flush_process(G, R):
    n_max = R + 4 * G + 7
    for n, (N, T) in enumerate(_flush_process(n_max, G, R)):
        assert o.split_tokens(n, G, R) == (N, T), (n, G, R)
        assert N % G == 0 and N + T == n
        assert min(n, R) <= T <= R + G - 1


def _hist(rng, n, hkv, d):
    k = (rng.standard_normal((n, hkv, d)) * np.exp(rng.standard_normal((1, hkv, d)))).astype(np.float16)
    v = rng.standard_normal((n, hkv, d)).astype(np.float16)
    return k, v


@pytest.mark.parametrize("R", [16, 32, 96])
def test_window_groups_are_a_prefix_of_the_unwindowed_groups(R):
    """The window changes how many groups are quantized, never their bytes."""
    rng = np.random.default_rng(7 + R)
    c0 = o.Config(4, 2, 32, 64, 2, 1)
    cw = o.Config(4, 2, 32, 64, 2, 1, window=R)
    for n in (5, R - 1, R + 31, R + 32, R + 33, 7 * 32 + R + 9):
        if n < 0:
            continue
        k, v = _hist(rng, n, 1, 64)
        a, b = o.cache_image(c0, k, v), o.cache_image(cw, k, v)
        ng = b["N"] // 32
        assert b["N"] == 32 * (max(0, n - R) // 32)
        assert np.array_equal(a["blocks"][:, :ng], b["blocks"])
        assert np.array_equal(b["tail_k"][0], k[b["N"]:, 0])
        assert np.array_equal(b["tail_v"][0], v[b["N"]:, 0])


def test_window_tail_is_exact_and_keeps_at_least_r_tokens():
    rng = np.random.default_rng(11)
    R, G = 64, 32
    cfg = o.Config(2, 2, G, 64, 4, 2, window=R)
    for n in (1, 63, 64, 95, 96, 97, 300):
        k, v = _hist(rng, n, 2, 64)
        kh, vh = o.dequantized_cache(cfg, k, v)
        N, T = o.split_tokens(n, G, R)
        assert T >= min(n, R)
        assert np.array_equal(kh[N:], k[N:].astype(np.float64))
        assert np.array_equal(vh[N:], v[N:].astype(np.float64))
        if N:   # the quantized part really is quantized (2-bit: not exact)
            assert not np.array_equal(kh[:N], k[:N].astype(np.float64))


def test_window_covering_the_context_is_plain_fp16_attention():
    """R >= n: nothing is quantized; the decode is softmax attention over the
    fp16 inputs, written out here with loops."""
    rng = np.random.default_rng(3)
    n, hkv, gqa, d = 40, 2, 2, 16
    cfg = o.Config(4, 2, 32, d, hkv * gqa, hkv, window=64)
    k, v = _hist(rng, n, hkv, d)
    q = rng.standard_normal((hkv * gqa, d))
    got = o.decode(cfg, k, v, q)
    for h in range(hkv * gqa):
        kv = h // gqa
        logits = [sum(float(q[h, c]) * float(k[t, kv, c]) for c in range(d)) / math.sqrt(d)
                  for t in range(n)]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = sum(w)
        for c in range(d):
            want = sum(w[t] * float(v[t, kv, c]) for t in range(n)) / z
            assert abs(got[h, c] - want) <= 1e-12 * max(1.0, abs(want))


@pytest.mark.parametrize("G,R", [(32, 0), (32, 32), (64, 16), (32, 128), (64, 128)])
def test_tail_ring_slots_are_distinct_and_r0_is_the_v1_tail(G, R):
    cfg = o.Config(4, 2, G, 64, 1, 1, window=R)
    W = R + G
    for n in range(0, R + 5 * G):
        N, T = o.split_tokens(n, G, R)
        slots = [o.tail_slot(cfg, p) for p in range(N, n)]
        assert len(set(slots)) == T and all(0 <= s < W for s in slots)
        if R == 0:
            assert slots == list(range(T))


def test_tail_arrays_place_each_token_in_its_ring_slot():
    rng = np.random.default_rng(5)
    G, R, d = 32, 32, 16
    cfg = o.Config(4, 2, G, d, 1, 1, window=R)
    W = R + G
    n = 3 * G + R + 13
    N, T = o.split_tokens(n, G, R)
    tk = rng.standard_normal((T, d)).astype(np.float16)
    tv = rng.standard_normal((T, d)).astype(np.float16)
    ak, av = o.tail_arrays(cfg, tk, tv, first=N)
    assert ak.shape == (W * d,) and av.shape == (W * d,)
    for i in range(T):
        s = (N + i) % W
        for c in range(d):
            assert ak[s * d + c] == tk[i, c]
            assert av[((s // 2) * d + c) * 2 + s % 2] == tv[i, c]
    used = {(N + i) % W for i in range(T)}
    for s in set(range(W)) - used:
        assert not ak[s * d:(s + 1) * d].any()
