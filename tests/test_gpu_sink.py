"""GPU parity of the sink window (the first S tokens of a sequence in fp16).

InnerQ abstract (page "WUSH-KV: KV Cache Quantization with Data-Adaptive
Transforms", third abstract): high-precision windows for the recent tokens
and for the attention-sink tokens.  The append kernel writes the first S
tokens to an fp16 sink area and applies the group / recent-window rule to
the tokens after them; the decode kernel folds the sink in with the tail.
Bit-exact cache bytes (sink, groups, tail) against the oracle after prefill
and after appends that straddle the sink's end; decode within 2e-3 of the
oracle's fp64 attention for ragged batches (contexts shorter than the sink
included), every GQA size, both CTA shapes and the 128k-token context.
"""
import numpy as np
import pytest
import torch

from asymmetric_kv_cache_b200 import inputs
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


def _spec(kb, vb, G, d, R, S, hq=4, hkv=2, seqs=4, max_tokens=1024):
    K = tl.kvq()
    return K.CacheSpec(kb, vb, G, d, hq, hkv, seqs, max_tokens, window=R, sink=S)


def _history(rng, lens, hkv, d):
    ks = [inputs.keys_channel_outliers(rng, n, hkv, d).astype(np.float16) for n in lens]
    vs = [(inputs.values_token_norms(rng, n, hkv, d) * 3).astype(np.float16) for n in lens]
    return ks, vs


@pytest.mark.parametrize("kb,vb,G,d,R,S", [(4, 2, 32, 128, 0, 4), (2, 2, 32, 128, 64, 16),
                                           (4, 2, 64, 128, 16, 33), (2, 4, 64, 64, 0, 100),
                                           (4, 4, 32, 64, 128, 1)])
def test_sink_prefill_matches_oracle(kb, vb, G, d, R, S):
    K = tl.kvq()
    spec = _spec(kb, vb, G, d, R, S, max_tokens=S + R + 6 * G)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(700 + S + R + G + kb)
    lens = [S + R + 3 * G + 5, max(S - 1, 0), S, S + R + G]
    ks, vs = _history(rng, lens, 2, d)
    tl.append_chunks(cache, ks, vs, "fp16")
    tl.check_cache_against_oracle(cache, ks, vs)


@pytest.mark.parametrize("G,R,S", [(32, 64, 16), (64, 0, 5), (32, 32, 40)])
def test_sink_appends_match_oracle_after_every_call(G, R, S):
    """Chunks that end inside the sink, straddle its end, or arrive on a
    full tail."""
    K = tl.kvq()
    d, hkv = 128, 2
    spec = _spec(4, 2, G, d, R, S, hq=8, hkv=hkv, seqs=3, max_tokens=2048)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(61 + G + R + S)
    W = R + G
    plan = [[1, S - 1 if S > 1 else 1, S + 3], [S, 1, W - 1], [W + 5, G, 1], [1, 2 * W + 7, G - 1],
            [G + 3, 1, W + 2 * G]]
    total = [sum(st[b] for st in plan) for b in range(3)]
    ks, vs = _history(rng, total, hkv, d)
    pos = [0, 0, 0]
    for step in plan:
        ck = [ks[b][pos[b]:pos[b] + step[b]] for b in range(3)]
        cv = [vs[b][pos[b]:pos[b] + step[b]] for b in range(3)]
        tl.append_chunks(cache, ck, cv, "fp16")
        pos = [pos[b] + step[b] for b in range(3)]
        tl.check_cache_against_oracle(cache, [ks[b][:pos[b]] for b in range(3)],
                                      [vs[b][:pos[b]] for b in range(3)])


@pytest.mark.parametrize("kb,G,R,S", [(4, 32, 0, 4), (2, 32, 128, 16), (4, 64, 64, 33),
                                      (2, 64, 0, 100)])
@pytest.mark.parametrize("gqa", [1, 4, 8])
def test_sink_decode_matches_oracle(kb, G, R, S, gqa):
    K = tl.kvq()
    hkv, d = 2, 128
    W = R + G
    lens = [1, max(S - 1, 1), S, S + 1, S + W - 1, S + W, S + 5 * G + R + 13, S + 9 * G + W - 1]
    spec = _spec(kb, 2, G, d, R, S, hq=hkv * gqa, hkv=hkv, seqs=len(lens), max_tokens=1024)
    rng = np.random.default_rng(1700 + kb + G + R + S + gqa)
    ks, vs = _history(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), hkv * gqa, d)).astype(np.float16).astype(np.float32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    out = cache.decode(tl.to_device(q, "fp16"))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


def test_sink_decode_many_units_narrow_ctas():
    K = tl.kvq()
    G, R, S, hkv, d = 32, 64, 16, 8, 128
    rng = np.random.default_rng(5151)
    lens = [int(x) for x in rng.integers(1, 600, size=40)]
    spec = _spec(4, 2, G, d, R, S, hq=32, hkv=hkv, seqs=len(lens), max_tokens=1024)
    ks, vs = _history(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), 32, d)).astype(np.float16).astype(np.float32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    out = cache.decode(tl.to_device(q, "fp16"))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


def test_sink_long_context_full_size():
    """The 128k-token context (K2/V2, G32) with a 32-token sink and a
    128-token recent window."""
    K = tl.kvq()
    w = inputs.WORKLOADS["long_ctx"]()
    spec = K.CacheSpec(w.k_bits, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                       w.batch, max(w.lens), window=128, sink=32)
    cache = K.KVQCache(spec)
    hk = [x.astype(np.float16) for x in w.keys]
    hv = [x.astype(np.float16) for x in w.values]
    tl.append_chunks(cache, hk, hv, w.kv_dtype)
    tl.check_cache_against_oracle(cache, hk, hv, group_sample=lambda ng: np.r_[0:2, ng - 2:ng])
    out = cache.decode(tl.to_device(w.q, w.q_dtype))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    err = tl.decode_error(out, tl.oracle_decode(spec, hk, hv, w.q))
    assert err <= tl.DECODE_TOL, err
