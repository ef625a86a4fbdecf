"""GPU parity of the recent fp16 window (R tokens beyond the partial group).

"[Framework] The Asymmetric Key-Value Cache Compression", §III and §V: the
most recent tokens stay in FP16.  With a window R the append kernel keeps
between R and R + G - 1 tokens in the fp16 tail ring (token p in slot
p mod (R + G)) and quantizes the oldest G once the tail reaches R + G; the
decode kernel folds every tail token in.  Bit-exact cache bytes against the
oracle after prefill, token-by-token appends and chunks that flush several
groups out of a full tail; decode within 2e-3 of the oracle's fp64
attention, for ragged batches, every GQA size, both CTA shapes and the
128k-token context at full size.
"""
import numpy as np
import pytest
import torch

from asymmetric_kv_cache_b200 import inputs
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


def _spec(kb, vb, G, d, R, hq=4, hkv=2, seqs=4, max_tokens=1024):
    K = tl.kvq()
    return K.CacheSpec(kb, vb, G, d, hq, hkv, seqs, max_tokens, window=R)


def _history(rng, lens, hkv, d):
    ks = [inputs.keys_channel_outliers(rng, n, hkv, d).astype(np.float16) for n in lens]
    vs = [(inputs.values_token_norms(rng, n, hkv, d) * 3).astype(np.float16) for n in lens]
    return ks, vs


@pytest.mark.parametrize("kb,vb,G,d,R", [(4, 2, 32, 128, 32), (2, 2, 32, 128, 128),
                                         (4, 2, 64, 128, 16), (2, 4, 64, 64, 64),
                                         (4, 4, 32, 64, 96), (4, 2, 32, 128, 1024)])
def test_window_prefill_matches_oracle(kb, vb, G, d, R):
    K = tl.kvq()
    spec = _spec(kb, vb, G, d, R, max_tokens=R + 6 * G)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(900 + R + G + kb)
    lens = [R + 3 * G + 5, R + G - 1, R + G, min(7, R)]
    ks, vs = _history(rng, lens, 2, d)
    tl.append_chunks(cache, ks, vs, "fp16")
    tl.check_cache_against_oracle(cache, ks, vs)


@pytest.mark.parametrize("G,R", [(32, 64), (64, 32), (32, 0)])
def test_window_appends_match_oracle_after_every_call(G, R):
    """Mixed chunk sizes: single tokens through flushes, and chunks arriving
    on a full tail (R + G - 1 tokens) that quantize groups made of old tail
    tokens in several CTAs while the new tail reuses their ring slots."""
    K = tl.kvq()
    d, hkv = 128, 2
    spec = _spec(4, 2, G, d, R, hq=8, hkv=hkv, seqs=3, max_tokens=2048)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(31 + G + R)
    W = R + G
    plan = [[W - 1, 1, 5], [1, W, 0], [200, G - 1, 2 * W + 3], [3, 1, 1], [G + 1, 0, W - 1],
            [1, 7, 1], [W + 2 * G + 5, 3, G]]
    total = [sum(s[b] for s in plan) for b in range(3)]
    ks, vs = _history(rng, total, hkv, d)
    pos = [0, 0, 0]
    for step in plan:
        ck = [ks[b][pos[b]:pos[b] + step[b]] for b in range(3)]
        cv = [vs[b][pos[b]:pos[b] + step[b]] for b in range(3)]
        tl.append_chunks(cache, ck, cv, "fp16")
        pos = [pos[b] + step[b] for b in range(3)]
        tl.check_cache_against_oracle(cache, [ks[b][:pos[b]] for b in range(3)],
                                      [vs[b][:pos[b]] for b in range(3)])


def test_window_token_by_token_equals_prefill():
    K = tl.kvq()
    G, R, d = 32, 64, 64
    n = R + 3 * G + 9
    rng = np.random.default_rng(77)
    ks, vs = _history(rng, [n], 1, d)
    a = K.KVQCache(_spec(4, 2, G, d, R, hq=2, hkv=1, seqs=1, max_tokens=512))
    b = K.KVQCache(_spec(4, 2, G, d, R, hq=2, hkv=1, seqs=1, max_tokens=512))
    tl.append_chunks(a, ks, vs, "fp16")
    for t in range(n):
        tl.append_chunks(b, [ks[0][t:t + 1]], [vs[0][t:t + 1]], "fp16")
    tl.check_cache_against_oracle(a, ks, vs)
    tl.check_cache_against_oracle(b, ks, vs)
    ng = (n - R) // G
    assert torch.equal(a.block_bytes(0, 0, ng), b.block_bytes(0, 0, ng))


@pytest.mark.parametrize("kb,G,R", [(4, 32, 32), (2, 32, 128), (4, 64, 64), (2, 64, 16)])
@pytest.mark.parametrize("gqa", [1, 4, 8])
def test_window_decode_matches_oracle(kb, G, R, gqa):
    K = tl.kvq()
    hkv, d = 2, 128
    W = R + G
    lens = [1, R, R + 1, W - 1, W, W + 1, 5 * G + R + 13, 9 * G + R + G - 1]
    spec = _spec(kb, 2, G, d, R, hq=hkv * gqa, hkv=hkv, seqs=len(lens), max_tokens=1024)
    rng = np.random.default_rng(1300 + kb + G + R + gqa)
    ks, vs = _history(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), hkv * gqa, d)).astype(np.float16).astype(np.float32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    out = cache.decode(tl.to_device(q, "fp16"))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


def test_window_decode_many_units_narrow_ctas():
    """More units than SMs: the 4-warp CTAs (two tail warps walk up to ten
    16-token chunks each)."""
    K = tl.kvq()
    G, R, hkv, d = 32, 128, 8, 128
    rng = np.random.default_rng(4242)
    lens = [int(x) for x in rng.integers(1, 700, size=40)]
    spec = _spec(4, 2, G, d, R, hq=32, hkv=hkv, seqs=len(lens), max_tokens=1024)
    ks, vs = _history(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), 32, d)).astype(np.float16).astype(np.float32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    out = cache.decode(tl.to_device(q, "fp16"))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


def test_window_decode_ignores_the_tcgen05_switch(monkeypatch):
    """The tcgen05 kernel has no window: with one the mma.sync kernel runs."""
    monkeypatch.setenv("KVQ_DECODE_TC", "1")
    K = tl.kvq()
    G, R = 32, 64
    lens = [R + 4 * G + 3, R + 1]
    spec = _spec(4, 2, G, 128, R, hq=8, hkv=2, seqs=2, max_tokens=512)
    rng = np.random.default_rng(5)
    ks, vs = _history(rng, lens, 2, 128)
    q = rng.standard_normal((2, 8, 128)).astype(np.float16).astype(np.float32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    out = cache.decode(tl.to_device(q, "fp16"))
    torch.cuda.synchronize()
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


def test_window_long_context_full_size():
    """The 128k-token context (K2/V2, G32) with a 128-token window, then one
    appended token per step across a flush."""
    K = tl.kvq()
    w = inputs.WORKLOADS["long_ctx"]()
    R = 128
    spec = K.CacheSpec(w.k_bits, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                       w.batch, max(w.lens) + 64, window=R)
    cache = K.KVQCache(spec)
    hk = [x.astype(np.float16) for x in w.keys]
    hv = [x.astype(np.float16) for x in w.values]
    tl.append_chunks(cache, hk, hv, w.kv_dtype)
    out = cache.decode(tl.to_device(w.q, w.q_dtype))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    err = tl.decode_error(out, tl.oracle_decode(spec, hk, hv, w.q))
    assert err <= tl.DECODE_TOL, err
    # 40 more tokens, one per call: the tail goes 128 -> 159 -> flush -> 136
    rng = np.random.default_rng(8)
    nk, nv = _history(rng, [40], w.n_kv_heads, w.head_dim)
    for t in range(40):
        tl.append_chunks(cache, [nk[0][t:t + 1]], [nv[0][t:t + 1]], "fp16")
    hk2 = [np.concatenate([hk[0], nk[0]])]
    hv2 = [np.concatenate([hv[0], nv[0]])]
    n = hk2[0].shape[0]
    tl.check_cache_against_oracle(cache, hk2, hv2,
                                  group_sample=lambda ng: np.arange(max(0, ng - 3), ng))
    out = cache.decode(tl.to_device(w.q, w.q_dtype))
    torch.cuda.synchronize()
    err = tl.decode_error(out, tl.oracle_decode(spec, hk2, hv2, w.q))
    assert err <= tl.DECODE_TOL, (n, err)
