"""GPU parity of position-adaptive key bits (kvq_config.akvq_delta = Delta).

"Asymmetric Key-Value Quantization: 2-Bit Values and 4-Bit Keys under
Long-Context Drift", §3.2, read as: 4-bit keys for the early groups (all
positions < Delta) and the recent ones (last position >= n - Delta), 2-bit
keys in between; a group that ages into the middle is requantized from its
dequantized 4-bit keys.  The bytes therefore depend on the append history,
so every case appends in chunks and the oracle replays the same chunks
(oracle.akvq_cache_image): 4-bit groups must equal the oracle's blocks bit
for bit, 2-bit groups the first akvq_block_bytes of theirs, the fp16 tail
its defined slots; the decode (each group read at its own width) must match
oracle.akvq_decode within the decode tolerance.  Covered: both head dims,
both group sizes, 2/4-bit values, GQA 1 / 4 / 8 / 16 (packed, plain and two
head slices), prefill, one-token appends across many group boundaries,
mixed chunk sizes, several sequences per append, every decode split path,
and the 128k-token context at full size (sampled groups).
"""
import numpy as np
import pytest
import torch

from asymmetric_kv_cache_b200 import inputs
from oracle import kvq_oracle as o
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


def _hist(rng, lens, hkv, d):
    ks = [inputs.keys_channel_outliers(rng, n, hkv, d).astype(np.float16) for n in lens]
    vs = [(inputs.values_token_norms(rng, n, hkv, d) * 2).astype(np.float16) for n in lens]
    return ks, vs


def _append_schedule(cache, ks, vs, schedules):
    """Round r appends chunk r of every sequence's schedule (0 past its end)."""
    rounds = max(len(s) for s in schedules)
    off = [0] * len(ks)
    for r in range(rounds):
        ck, cv = [], []
        for b, s in enumerate(schedules):
            n = s[r] if r < len(s) else 0
            ck.append(ks[b][off[b]:off[b] + n])
            cv.append(vs[b][off[b]:off[b] + n])
            off[b] += n
        tl.append_chunks(cache, ck, cv, "fp16")
    return [[n for n in s] for s in schedules]


def _check_bytes(cache, cfg, k, v, chunks, b, group_sample=None):
    img = o.akvq_cache_image(cfg, k, v, chunks)
    lay = cache.layout
    a2 = lay["akvq_block_bytes"]
    ng = len(img["bits"])
    gsel = range(ng) if group_sample is None else group_sample(ng)
    for h in range(cfg.n_kv_heads):
        got = cache.block_bytes(b, h, ng).cpu().numpy()
        for g in gsel:
            n = lay["block_bytes"] if img["bits"][g] == cfg.k_bits else a2
            if not np.array_equal(got[g, :n], img["blocks"][h, g, :n]):
                bad = np.flatnonzero(got[g, :n] != img["blocks"][h, g, :n])
                raise AssertionError(f"seq {b} head {h} group {g} ({img['bits'][g]}-bit keys): "
                                     f"{len(bad)} bytes differ, first at {bad[0]}")
    N, T = img["N"], img["T"]
    if T:
        mk, mv = tl.expected_tail_mask(cfg, N, T)
        for h in range(cfg.n_kv_heads):
            tk, tv = o.tail_arrays(cfg, k[N:, h], v[N:, h], first=N)
            gk, gv = cache.tail_halves(b, h)
            assert np.array_equal(gk.cpu().numpy()[mk].view(np.uint16), tk[mk].view(np.uint16))
            assert np.array_equal(gv.cpu().numpy()[mv].view(np.uint16), tv[mv].view(np.uint16))
    return img


def _case(spec, lens, schedules, seed, caps=(None,), monkeypatch=None):
    K = tl.kvq()
    rng = np.random.default_rng(seed)
    ks, vs = _hist(rng, lens, spec.n_kv_heads, spec.head_dim)
    cache = K.KVQCache(spec)
    _append_schedule(cache, ks, vs, schedules)
    cfg = tl.oracle_cfg(spec)
    assert cache.lengths() == list(lens)
    bits_seen = set()
    for b in range(len(lens)):
        img = _check_bytes(cache, cfg, ks[b], vs[b], schedules[b], b)
        bits_seen.update(img["bits"])
    q = rng.standard_normal((len(lens), spec.n_q_heads, spec.head_dim)).astype(np.float16)
    q = q.astype(np.float32)
    want = np.stack([o.akvq_decode(cfg, ks[b], vs[b], q[b], schedules[b])
                     for b in range(len(lens))])
    for cap in caps:
        if monkeypatch is not None:
            if cap is None:
                monkeypatch.delenv("KVQ_DECODE_MAX_CTAS", raising=False)
            else:
                monkeypatch.setenv("KVQ_DECODE_MAX_CTAS", cap)
        out = cache.decode(tl.to_device(q, "fp16"))
        torch.cuda.synchronize()
        err = tl.decode_error(out, want)
        assert err <= tl.DECODE_TOL, (cap, err)
    assert cache.workspace_status() == 0
    return bits_seen


@pytest.mark.parametrize("vb,G,d", [(2, 32, 128), (2, 64, 128), (4, 32, 128), (2, 32, 64),
                                    (4, 64, 64)])
@pytest.mark.parametrize("gqa", [1, 4, 8, 16])
def test_prefill_and_one_token_appends(vb, G, d, gqa):
    """Prefills (the middle groups go to 2 bits from fp16), then one-token
    appends: every G-th one ages a group into the middle (requantized)."""
    K = tl.kvq()
    hkv = 2
    delta = 2 * G
    spec = K.CacheSpec(4, vb, G, d, hkv * gqa, hkv, 4, 16 * G, akvq_delta=delta)
    pre = [1, G - 1, 5 * G + 3, 9 * G]
    steps = 2 * G + 5
    lens = [p + steps for p in pre]
    schedules = [[p] + [1] * steps for p in pre]
    bits = _case(spec, lens, schedules, seed=900 + vb + G + d + gqa)
    assert bits == {2, 4}


@pytest.mark.parametrize("gqa", [1, 4, 8])
def test_mixed_chunks(gqa):
    """Chunks shorter and longer than a group, several groups aging in one
    append, sequences at different phases in the same launch."""
    K = tl.kvq()
    G, d, hkv = 32, 128, 2
    spec = K.CacheSpec(4, 2, G, d, hkv * gqa, hkv, 5, 1024, akvq_delta=3 * G)
    schedules = [[5, G + 3, 2 * G, 1, 1, 3 * G + 1, 7, 4 * G, 9],
                 [3 * G, 1, G - 1, 5 * G + 17, 2, 33],
                 [0, 0, 7 * G, 2 * G + 1],
                 [1] * 40 + [6 * G],
                 [8 * G + 31, 1, 1, 1]]
    lens = [sum(s) for s in schedules]
    bits = _case(spec, lens, schedules, seed=950 + gqa)
    assert bits == {2, 4}


def test_split_counts_mixed_widths(monkeypatch):
    """Split counts (whole units, in-kernel merge, combine kernel) over a
    cache holding both widths."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 32, 8, 40, 4096, akvq_delta=256)
    rng = np.random.default_rng(977)
    lens = [4000, 1234, 95] + [int(x) for x in rng.integers(1, 900, size=37)]
    schedules = []
    for n in lens:
        a = int(rng.integers(0, n + 1))
        rest = n - a
        mid = []
        for x in rng.integers(1, 40, size=3):
            if int(x) <= rest:
                mid.append(int(x))
                rest -= int(x)
        schedules.append([a] + mid + [rest])
    _case(spec, lens, schedules, seed=978, caps=("1", "7", "64", "300", None),
          monkeypatch=monkeypatch)


def test_long_context_full_size():
    """The 128k-token context with Delta = 1024: prefill of all but 40
    tokens, then 40 one-token appends (each group passing n - Delta is
    requantized); sampled groups bit-exact, the decode against the oracle."""
    K = tl.kvq()
    w = inputs.long_ctx()
    n = w.lens[0]
    spec = K.CacheSpec(4, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                       1, n, akvq_delta=1024)
    cache = K.KVQCache(spec)
    sched = [n - 40] + [1] * 40
    _append_schedule(cache, w.keys, w.values, [sched])
    cfg = tl.oracle_cfg(spec)
    rng = np.random.default_rng(981)

    def sample(ng):
        ends = list(range(0, 40)) + list(range(ng - 40, ng))
        return sorted(set(ends + [int(x) for x in rng.integers(0, ng, size=60)]))

    _check_bytes(cache, cfg, w.keys[0], w.values[0], sched, 0, group_sample=sample)
    out = cache.decode(tl.to_device(w.q, "fp16"))
    want = o.akvq_decode(cfg, w.keys[0], w.values[0], w.q[0], sched)[None]
    assert tl.decode_error(out, want) <= tl.DECODE_TOL
    assert cache.workspace_status() == 0


@pytest.mark.parametrize("gqa", [4, 8])
def test_rotated_adaptive_cache(gqa):
    """Rotation and position-adaptive widths together: the cache holds the
    rotated tokens (fp32 butterfly, fp16), the widths and requantizations
    act on them, the decode rotates q and its output back.  Expected values:
    the oracle's adaptive image and decode of the rotated tokens, with the
    query rotated in and the output rotated back (the steps of its rotated
    decode)."""
    K = tl.kvq()
    G, d, hkv = 32, 128, 2
    spec = K.CacheSpec(4, 2, G, d, hkv * gqa, hkv, 3, 1024, rotate=1, akvq_delta=2 * G)
    schedules = [[5 * G + 3] + [1] * 40, [1] * 70 + [3 * G], [9 * G + 1, G, 7]]
    lens = [sum(s) for s in schedules]
    rng = np.random.default_rng(990 + gqa)
    ks, vs = _hist(rng, lens, hkv, d)
    cache = K.KVQCache(spec)
    _append_schedule(cache, ks, vs, schedules)
    cfg = tl.oracle_cfg(spec)
    plain = o.Config(cfg.k_bits, cfg.v_bits, cfg.group, cfg.head_dim, cfg.n_q_heads,
                     cfg.n_kv_heads, akvq_delta=cfg.akvq_delta)
    kr = [o.cache_tokens(cfg, x) for x in ks]
    vr = [o.cache_tokens(cfg, x) for x in vs]
    for b in range(len(lens)):
        _check_bytes(cache, plain, kr[b], vr[b], schedules[b], b)
    q = rng.standard_normal((len(lens), hkv * gqa, d)).astype(np.float16).astype(np.float32)
    out = cache.decode(tl.to_device(q, "fp16"))
    want = np.stack([o.rotate_fp64(o.akvq_decode(plain, kr[b], vr[b], o.rotate_fp64(q[b]),
                                                 schedules[b])) for b in range(len(lens))])
    assert tl.decode_error(out, want) <= tl.DECODE_TOL
    assert cache.workspace_status() == 0
