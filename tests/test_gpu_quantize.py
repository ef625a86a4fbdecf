"""GPU parity of the quantize / pack / append / flush path (bit-exact).

The CUDA append kernel must write exactly the oracle's group blocks
(codes, fp16 scales and mins in LAYOUT v2) and fp16 tails, for prefill,
per-step appends with flushes, mixed chunk sizes and every supported
(key bits, value bits, group, head_dim), from fp16, bf16 and fp32 inputs.
"""
import numpy as np
import pytest

from asymmetric_kv_cache_b200 import inputs
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu

COMBOS = [(4, 2, 32, 128), (2, 2, 32, 128), (4, 2, 64, 128), (2, 2, 64, 128),
          (4, 4, 32, 128), (2, 4, 64, 128), (4, 2, 32, 64), (2, 2, 32, 64),
          (4, 2, 64, 64), (4, 4, 64, 64)]


def _spec(kb, vb, G, d, hq=4, hkv=2, seqs=3, max_tokens=512):
    K = tl.kvq()
    return K.CacheSpec(kb, vb, G, d, hq, hkv, seqs, max_tokens)


def _history(rng, lens, hkv, d, dtype="fp16"):
    ks, vs = [], []
    for n in lens:
        ks.append(inputs.keys_channel_outliers(rng, n, hkv, d))
        vs.append(inputs.values_token_norms(rng, n, hkv, d) * 3)
    if dtype == "bf16":
        ks = [tl.bf16_values(x) for x in ks]
        vs = [tl.bf16_values(x) for x in vs]
    return ks, vs


@pytest.mark.parametrize("kb,vb,G,d", COMBOS)
def test_prefill_matches_oracle(kb, vb, G, d):
    K = tl.kvq()
    spec = _spec(kb, vb, G, d)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(100 + kb * 10 + vb + G + d)
    lens = [3 * G + 5, G, 7]
    ks, vs = _history(rng, lens, 2, d)
    tl.append_chunks(cache, ks, vs, "fp16")
    hk = [x.astype(np.float16) for x in ks]
    hv = [x.astype(np.float16) for x in vs]
    tl.check_cache_against_oracle(cache, hk, hv)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_prefill_other_input_dtypes(dtype):
    """fp32 and bf16 inputs are rounded to fp16 first (nearest even)."""
    K = tl.kvq()
    spec = _spec(4, 2, 32, 128)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(7)
    ks, vs = _history(rng, [100, 64, 31], 2, 128, dtype)
    tl.append_chunks(cache, ks, vs, dtype)
    tl.check_cache_against_oracle(cache, [x.astype(np.float16) for x in ks],
                                  [x.astype(np.float16) for x in vs])


def test_fp32_input_with_tiny_and_huge_values():
    """Values that round to fp16 subnormals, and the largest finite fp16."""
    K = tl.kvq()
    spec = _spec(4, 2, 32, 64, hq=1, hkv=1, seqs=1)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(8)
    k = rng.standard_normal((64, 1, 64)).astype(np.float32) * 1e-6
    v = rng.standard_normal((64, 1, 64)).astype(np.float32)
    k[3, 0, 5] = 60000.0
    v[40, 0, 7] = -65504.0
    k[:32, 0, 9] = 0.25        # constant channel: scale 0
    tl.append_chunks(cache, [k], [v], "fp32")
    tl.check_cache_against_oracle(cache, [k.astype(np.float16)], [v.astype(np.float16)])


@pytest.mark.parametrize("kb,vb,G,d", [(4, 2, 32, 128), (2, 2, 64, 64)])
def test_token_by_token_equals_prefill(kb, vb, G, d):
    """Appending one token at a time (flushes every G steps) writes the same
    bytes as one prefill of the same tokens."""
    K = tl.kvq()
    spec = _spec(kb, vb, G, d, seqs=2)
    rng = np.random.default_rng(9)
    n = 3 * G + 11
    ks, vs = _history(rng, [n, n], 2, d)
    a = K.KVQCache(spec)
    tl.append_chunks(a, ks, vs, "fp16")
    b = K.KVQCache(spec)
    for t in range(n):
        tl.append_chunks(b, [ks[0][t:t + 1], ks[1][t:t + 1]], [vs[0][t:t + 1], vs[1][t:t + 1]], "fp16")
    hk = [x.astype(np.float16) for x in ks]
    hv = [x.astype(np.float16) for x in vs]
    tl.check_cache_against_oracle(a, hk, hv)
    tl.check_cache_against_oracle(b, hk, hv)


def test_mixed_chunks_and_idle_sequences():
    """Random chunk sizes per sequence per call, including 0 and chunks that
    complete several groups at once starting from a partial tail."""
    K = tl.kvq()
    spec = _spec(4, 2, 32, 128, hq=8, hkv=4, seqs=5, max_tokens=1024)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(10)
    hist_k = [np.zeros((0, 4, 128), np.float32) for _ in range(5)]
    hist_v = [np.zeros((0, 4, 128), np.float32) for _ in range(5)]
    for step in range(12):
        sizes = rng.choice([0, 1, 2, 5, 31, 32, 33, 70], size=5)
        ck, cv = _history(rng, sizes, 4, 128)
        tl.append_chunks(cache, ck, cv, "fp16")
        hist_k = [np.concatenate([h, c]) for h, c in zip(hist_k, ck)]
        hist_v = [np.concatenate([h, c]) for h, c in zip(hist_v, cv)]
    tl.check_cache_against_oracle(cache, [x.astype(np.float16) for x in hist_k],
                                  [x.astype(np.float16) for x in hist_v])


def test_capacity_error_leaves_cache_unchanged():
    K = tl.kvq()
    spec = _spec(4, 2, 32, 64, hq=1, hkv=1, seqs=2, max_tokens=40)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(11)
    ks, vs = _history(rng, [30, 10], 1, 64)
    tl.append_chunks(cache, ks, vs, "fp16")
    more_k, more_v = _history(rng, [11, 1], 1, 64)
    with pytest.raises(K.KvqError) as ei:
        tl.append_chunks(cache, more_k, more_v, "fp16")
    assert ei.value.status == 4
    assert cache.lengths() == [30, 10]
    tl.check_cache_against_oracle(cache, [x.astype(np.float16) for x in ks],
                                  [x.astype(np.float16) for x in vs])


def test_append_stream_workload_full_size():
    """64 sequences, 8 kv heads, d=128, K4/V2, G=32: 256 decode steps of one
    token each (a flush every 32 steps), then every group and tail checked."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 8, 8, 64, 256)
    cache = K.KVQCache(spec)
    ks, vs = inputs.append_stream(inputs.SEED_BASE + 3, 64, 256, 8, 128)
    for t in range(256):
        cache.append(tl.to_device(ks[t], "fp16"), tl.to_device(vs[t], "fp16"), [1] * 64)
    hk = [np.stack([ks[t][b] for t in range(256)]) for b in range(64)]
    hv = [np.stack([vs[t][b] for t in range(256)]) for b in range(64)]
    tl.check_cache_against_oracle(cache, hk, hv)


def test_prefill_workload_full_size():
    """Prefill of 4 sequences x 32768 tokens x 8 kv heads x d=128 (fp16,
    K4/V2, G=32) in one call: every group of the first sequence (all 8 kv
    heads, 8192 blocks), every 7th group of the others, and the lengths."""
    K = tl.kvq()
    w = inputs.quant_append()
    spec = K.CacheSpec(4, 2, 32, 128, 8, 8, 4, 32768)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, w.keys, w.values, "fp16")
    tl.check_cache_against_oracle(cache, w.keys, w.values, seqs=[0])
    tl.check_cache_against_oracle(cache, w.keys, w.values, seqs=[1, 2, 3],
                                  group_sample=lambda ng: np.arange(0, ng, 7))


def test_division_rule_case():
    """The hand-worked golden case that pins IEEE division (quantizer
    examples, '2-bit, IEEE division not reciprocal multiply'): a key channel
    and a value group holding 0, 37.5 and 45 must get code 2 for 37.5 (the
    quotient 37.5 / 15 = 2.5 ties to even); multiplying by fp32(1/15) would
    give 3."""
    K = tl.kvq()
    G, d = 32, 64
    spec = K.CacheSpec(2, 2, G, d, 1, 1, 1, 64)
    k = np.zeros((G, 1, d), np.float16)
    v = np.zeros((G, 1, d), np.float16)
    k[3, 0, 5] = 37.5
    k[7, 0, 5] = 45.0
    v[4, 0, 1] = 37.5
    v[4, 0, 2] = 45.0
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, [k], [v], "fp16")
    tl.check_cache_against_oracle(cache, [k], [v])
    from oracle import kvq_oracle as o
    kc, ks, _ = o.quantize_keys(k[:, 0, :], 2)
    assert float(ks[5]) == 15.0 and int(kc[3, 5]) == 2 and int(kc[7, 5]) == 3


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_tail_conversion_is_rne_on_every_pattern(dtype):
    """The cache's fp16 rounding on entry, bit for bit: stratified fp32 bit
    patterns (every exponent, ties at the fp16 spacing, the subnormal range,
    overflow; tests/fp16_rne.py) or every bf16 pattern go through appends
    that stay in the fp16 tails; the stored halves must equal the binary16
    round-to-nearest-even written from the format's definition."""
    import torch
    from tests.fp16_rne import fp16_bits_rne, stratified_fp32_patterns
    K = tl.kvq()
    G, d, T = 32, 128, 31   # 31 tokens per sequence: no group completes
    if dtype == "fp32":
        u = stratified_fp32_patterns(np.random.default_rng(11))
    else:
        b = np.arange(1 << 16, dtype=np.uint32) << 16
        u = b[~np.isnan(b.view(np.float32))]
    per_seq = 2 * T * d                    # K and V elements per sequence
    n_seq = -(-len(u) // per_seq)
    pad = n_seq * per_seq - len(u)
    u = np.concatenate([u, np.zeros(pad, np.uint32)])
    vals = u.view(np.float32).reshape(n_seq, 2, T, 1, d)
    spec = K.CacheSpec(4, 2, G, d, 1, 1, n_seq, 64)
    cache = K.KVQCache(spec)
    ks = [vals[i, 0] for i in range(n_seq)]
    vs = [vals[i, 1] for i in range(n_seq)]
    if dtype == "fp32":
        kd = torch.from_numpy(np.ascontiguousarray(np.concatenate(ks))).cuda()
        vd = torch.from_numpy(np.ascontiguousarray(np.concatenate(vs))).cuda()
    else:   # exact bf16 values: the high halves of the fp32 patterns
        kd = torch.from_numpy(np.ascontiguousarray(np.concatenate(ks))).cuda().to(torch.bfloat16)
        vd = torch.from_numpy(np.ascontiguousarray(np.concatenate(vs))).cuda().to(torch.bfloat16)
    cache.append(kd, vd, [T] * n_seq)
    torch.cuda.synchronize()
    from oracle import kvq_oracle as o
    want = fp16_bits_rne(u).reshape(n_seq, 2, T, d)
    kidx = np.array([[o.tail_key_index(t, c, d) for c in range(d)] for t in range(T)])
    vidx = np.array([[o.tail_value_index(t, c, d) for c in range(d)] for t in range(T)])
    bad = 0
    for i in range(n_seq):
        tk, tv = cache.tail_halves(i, 0)
        hk = tk.cpu().view(torch.int16).numpy().view(np.uint16)
        hv = tv.cpu().view(torch.int16).numpy().view(np.uint16)
        bad += int((hk[kidx] != want[i, 0]).sum()) + int((hv[vidx] != want[i, 1]).sum())
    assert bad == 0, bad
