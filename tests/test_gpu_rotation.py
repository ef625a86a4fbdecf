"""GPU parity of the rotating cache (kvq_config.rotate = 1).

Every K/V token entering the cache is rotated by the normalized
Walsh-Hadamard matrix ("[Framework] The Asymmetric Key-Value Cache
Compression", §IV stage 1; "Asymmetric Key-Value Quantization: 2-Bit Values
and 4-Bit Keys under Long-Context Drift", §3.1) with the fp32 butterfly in
the oracle's stage order, so the cache bytes (group blocks, tail, sink) must
equal the oracle's for the rotated tokens bit for bit; the decode rotates q
and rotates its output back, and must match the oracle's rotated decode
within the decode tolerance.  Covered: both head dims, both group sizes,
2/4-bit keys and values, fp16 / bf16 / fp32 inputs, GQA 1 / 4 / 8 / 16
(two head slices), prefill and one-token appends with flushes, the recent
and sink windows, split counts (merge in the kernel and in the combine
kernel) and the 128k-token context at full size.
"""
import numpy as np
import pytest
import torch

from asymmetric_kv_cache_b200 import inputs
from oracle import kvq_oracle as o
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


def _hist(rng, lens, hkv, d, dtype="fp16"):
    ks = [inputs.keys_channel_outliers(rng, n, hkv, d) for n in lens]
    vs = [inputs.values_token_norms(rng, n, hkv, d) * 2 for n in lens]
    if dtype == "fp16":
        ks = [x.astype(np.float16) for x in ks]
        vs = [x.astype(np.float16) for x in vs]
    elif dtype == "bf16":
        ks = [tl.bf16_values(x) for x in ks]
        vs = [tl.bf16_values(x) for x in vs]
    return ks, vs


def _check(spec, ks, vs, q, dtype, q_dtype="fp16"):
    K = tl.kvq()
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, dtype)
    cfg = tl.oracle_cfg(spec)
    # the cache holds the rotated tokens, bit for bit
    tl.check_cache_against_oracle(cache, [o.cache_tokens(cfg, x) for x in ks],
                                  [o.cache_tokens(cfg, x) for x in vs])
    out = cache.decode(tl.to_device(q, q_dtype))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    want = np.stack([o.decode(cfg, ks[b], vs[b], q[b]) for b in range(len(ks))])
    err = tl.decode_error(out, want)
    assert err <= tl.DECODE_TOL, err
    return cache, err


@pytest.mark.parametrize("kb,vb,G,d", [(4, 2, 32, 128), (2, 2, 32, 128), (4, 2, 64, 128),
                                        (2, 4, 64, 128), (4, 2, 32, 64), (2, 2, 64, 64)])
@pytest.mark.parametrize("gqa", [1, 4, 8])
def test_rotated_cache_and_decode(kb, vb, G, d, gqa):
    K = tl.kvq()
    hkv = 2
    spec = K.CacheSpec(kb, vb, G, d, hkv * gqa, hkv, 4, 1024, rotate=1)
    rng = np.random.default_rng(700 + kb + 3 * vb + G + d + gqa)
    lens = [1, G + 3, 5 * G + 13, 9 * G]
    ks, vs = _hist(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), hkv * gqa, d)).astype(np.float16).astype(np.float32)
    _check(spec, ks, vs, q, "fp16")


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_rotated_other_input_dtypes(dtype):
    """fp32 and bf16 inputs are rotated from their own values (no fp16
    rounding before the butterfly)."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 16, 4, 3, 512, rotate=1)
    rng = np.random.default_rng(7001)
    ks, vs = _hist(rng, [100, 64, 31], 4, 128, dtype)
    q = rng.standard_normal((3, 16, 128)).astype(np.float32)
    _check(spec, ks, vs, q, dtype, q_dtype="fp32")


def test_rotated_gqa16_bf16_query():
    K = tl.kvq()
    spec = K.CacheSpec(2, 4, 64, 64, 32, 2, 2, 2048, rotate=1)
    rng = np.random.default_rng(7002)
    ks, vs = _hist(rng, [1500, 333], 2, 64)
    q = tl.bf16_values(rng.standard_normal((2, 32, 64)).astype(np.float32))
    _check(spec, ks, vs, q, "fp16", q_dtype="bf16")


def test_rotated_appends_one_token_at_a_time():
    """Prefill, then one-token appends across two flushes: every token is
    rotated on entry whichever path stores it (group, tail, flush)."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 8, 2, 3, 512, rotate=1)
    rng = np.random.default_rng(7003)
    ks, vs = _hist(rng, [70, 40, 1], 2, 128)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    for _ in range(45):
        nk, nv = _hist(rng, [1, 1, 1], 2, 128)
        tl.append_chunks(cache, nk, nv, "fp16")
        ks = [np.concatenate([a, b]) for a, b in zip(ks, nk)]
        vs = [np.concatenate([a, b]) for a, b in zip(vs, nv)]
    cfg = tl.oracle_cfg(spec)
    tl.check_cache_against_oracle(cache, [o.cache_tokens(cfg, x) for x in ks],
                                  [o.cache_tokens(cfg, x) for x in vs])
    q = rng.standard_normal((3, 8, 128)).astype(np.float16).astype(np.float32)
    out = cache.decode(tl.to_device(q, "fp16"))
    want = np.stack([o.decode(cfg, ks[b], vs[b], q[b]) for b in range(3)])
    assert tl.decode_error(out, want) <= tl.DECODE_TOL


@pytest.mark.parametrize("window,sink", [(128, 0), (64, 5), (0, 33)])
def test_rotated_with_windows(window, sink):
    K = tl.kvq()
    spec = K.CacheSpec(2, 2, 32, 128, 32, 8, 2, 2048, window=window, sink=sink, rotate=1)
    rng = np.random.default_rng(7004 + window + sink)
    ks, vs = _hist(rng, [1500, 77], 8, 128)
    q = rng.standard_normal((2, 32, 128)).astype(np.float16).astype(np.float32)
    _check(spec, ks, vs, q, "fp16")


def test_rotated_split_counts(monkeypatch):
    """Outputs rotated back on every merge path: whole units, the in-kernel
    merge of split units and the combine kernel."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 32, 8, 40, 4096, rotate=1)
    rng = np.random.default_rng(7005)
    lens = [4000, 1234, 95] + [int(x) for x in rng.integers(1, 600, size=37)]
    ks, vs = _hist(rng, lens, 8, 128)
    q = rng.standard_normal((len(lens), 32, 128)).astype(np.float16).astype(np.float32)
    cfg = tl.oracle_cfg(spec)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    want = np.stack([o.decode(cfg, ks[b], vs[b], q[b]) for b in range(len(lens))])
    for cap in ("1", "7", "64", "300", None):
        if cap is None:
            monkeypatch.delenv("KVQ_DECODE_MAX_CTAS", raising=False)
        else:
            monkeypatch.setenv("KVQ_DECODE_MAX_CTAS", cap)
        out = cache.decode(tl.to_device(q, "fp16"))
        assert tl.decode_error(out, want) <= tl.DECODE_TOL, cap
    # the first three sequences alone: few units, wide CTAs, in-kernel merge
    monkeypatch.delenv("KVQ_DECODE_MAX_CTAS", raising=False)
    out = cache.decode(tl.to_device(q[:3], "fp16"))
    assert tl.decode_error(out, want[:3]) <= tl.DECODE_TOL
    assert cache.workspace_status() == 0


def test_rotated_long_context_full_size():
    K = tl.kvq()
    w = inputs.long_ctx()
    spec = K.CacheSpec(w.k_bits, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                       1, w.lens[0], rotate=1)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, w.keys, w.values, "fp16")
    cfg = tl.oracle_cfg(spec)
    tl.check_cache_against_oracle(cache, [o.cache_tokens(cfg, w.keys[0])],
                                  [o.cache_tokens(cfg, w.values[0])])
    out = cache.decode(tl.to_device(w.q, "fp16"))
    want = o.decode(cfg, w.keys[0], w.values[0], w.q[0])[None]
    assert tl.decode_error(out, want) <= tl.DECODE_TOL
