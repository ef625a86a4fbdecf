"""GPU parity of split-K decode attention over the quantized cache.

Every output must be within 2e-3 (max abs) of the oracle's fp64 attention on
the dequantized cache.  Covered: all supported (key bits, value bits, group,
head_dim), GQA 1 / 4 / 8 / 16 (two head slices), fp16 / bf16 / fp32
queries, contexts shorter than a group (tail only), exact multiples of G
(no tail), one token, ragged batches, the five benchmark workloads at full
size, different split counts, repeated calls and the error paths.
"""
import os

import numpy as np
import pytest
import torch

from asymmetric_kv_cache_b200 import inputs
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


def _run(spec, hist_k, hist_v, q, q_dtype, kv_dtype="fp16"):
    K = tl.kvq()
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, hist_k, hist_v, kv_dtype)
    out = cache.decode(tl.to_device(q, q_dtype))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    return cache, out


def _workload_arrays(rng, lens, hkv, d, hq, q_dtype="fp16", vscale=1.0):
    ks = [inputs.keys_channel_outliers(rng, n, hkv, d).astype(np.float16) for n in lens]
    vs = [(inputs.values_token_norms(rng, n, hkv, d) * vscale).astype(np.float16) for n in lens]
    q = rng.standard_normal((len(lens), hq, d)).astype(np.float32)
    if q_dtype == "fp16":
        q = q.astype(np.float16).astype(np.float32)
    elif q_dtype == "bf16":
        q = tl.bf16_values(q)
    return ks, vs, q


@pytest.mark.parametrize("kb,vb,G,d", [(4, 2, 32, 128), (2, 2, 32, 128), (4, 2, 64, 128),
                                        (2, 2, 64, 128), (4, 4, 32, 128), (2, 4, 64, 128),
                                        (4, 2, 32, 64), (2, 2, 64, 64), (4, 4, 64, 64)])
@pytest.mark.parametrize("gqa", [1, 4, 8])
def test_decode_small(kb, vb, G, d, gqa):
    K = tl.kvq()
    hkv = 2
    spec = K.CacheSpec(kb, vb, G, d, hkv * gqa, hkv, 5, 1024)
    rng = np.random.default_rng(1000 + kb + vb * 3 + G + d + gqa)
    lens = [1, G - 1, G, 5 * G + 13, 9 * G]
    ks, vs, q = _workload_arrays(rng, lens, hkv, d, hkv * gqa, vscale=2.0)
    _, out = _run(spec, ks, vs, q, "fp16")
    want = tl.oracle_decode(spec, ks, vs, q)
    err = tl.decode_error(out, want)
    assert err <= tl.DECODE_TOL, err


@pytest.mark.parametrize("q_dtype", ["fp16", "bf16", "fp32"])
def test_decode_query_dtypes(q_dtype):
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 16, 4, 3, 2048)
    rng = np.random.default_rng(21)
    ks, vs, q = _workload_arrays(rng, [700, 1500, 33], 4, 128, 16, q_dtype)
    _, out = _run(spec, ks, vs, q, q_dtype)
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


def test_decode_gqa16_two_slices():
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 32, 2, 2, 1024)
    rng = np.random.default_rng(22)
    ks, vs, q = _workload_arrays(rng, [900, 77], 2, 128, 32)
    _, out = _run(spec, ks, vs, q, "fp16")
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


def test_identical_keys_give_mean_of_values():
    """All keys equal: the weights are uniform, the output is the mean of the
    dequantized values (an exact property of softmax attention)."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 64, 4, 1, 1, 256)
    rng = np.random.default_rng(23)
    n = 150
    k = np.repeat(rng.standard_normal((1, 1, 64)), n, axis=0).astype(np.float16)
    v = rng.standard_normal((n, 1, 64)).astype(np.float16)
    q = rng.standard_normal((1, 4, 64)).astype(np.float16).astype(np.float32)
    _, out = _run(spec, [k], [v], q, "fp16")
    from oracle import kvq_oracle as o
    _, vh = o.dequantized_cache(tl.oracle_cfg(spec), k, v)
    mean = vh[:, 0].mean(0)
    g = out.float().cpu().numpy()[0]
    assert np.abs(g - mean[None, :]).max() <= tl.DECODE_TOL


@pytest.mark.parametrize("name", ["tiny", "llama3_8b", "long_ctx", "llama70b_conc"])
def test_decode_workloads_full_size(name):
    """The benchmark workloads at their full sizes: every byte of every group
    block and tail of the cache compared with the oracle's (bit-exact), then
    the decode compared element by element with the oracle (every output)."""
    K = tl.kvq()
    w = inputs.WORKLOADS[name]()
    spec = K.CacheSpec(w.k_bits, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                       w.batch, max(w.lens))
    kv_dtype = w.kv_dtype
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, w.keys, w.values, kv_dtype)
    if w.q_dtype == "bf16":
        import torch as _t
        qd = _t.from_numpy(w.q_bits.view(np.int16)).view(_t.bfloat16).cuda()
    else:
        qd = tl.to_device(w.q, w.q_dtype)
    out = cache.decode(qd)
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    hk = [x.astype(np.float16) for x in w.keys]
    hv = [x.astype(np.float16) for x in w.values]
    tl.check_cache_against_oracle(cache, hk, hv)
    want = tl.oracle_decode(spec, hk, hv, w.q)
    err = tl.decode_error(out, want)
    assert err <= tl.DECODE_TOL, (name, err)


def test_split_count_does_not_change_results(monkeypatch):
    """The same cache decoded with 1, 7, 64 and the default number of CTAs."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 32, 8, 3, 4096)
    rng = np.random.default_rng(24)
    ks, vs, q = _workload_arrays(rng, [4000, 1234, 95], 8, 128, 32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    qd = tl.to_device(q, "fp16")
    outs = []
    for cap in ("1", "7", "64", None):
        if cap is None:
            monkeypatch.delenv("KVQ_DECODE_MAX_CTAS", raising=False)
        else:
            monkeypatch.setenv("KVQ_DECODE_MAX_CTAS", cap)
        outs.append(cache.decode(qd).float().cpu().numpy())
    want = tl.oracle_decode(spec, ks, vs, q)
    # Split counts only reorder the work: every attention weight p is still
    # rounded to fp16 once (relative error <= 2^-11), but relative to a
    # running max that depends on the order, so two orders can round each
    # p differently by up to 2^-10 relative; through o = sum p v / sum p
    # that moves each output by at most about 2^-9 * max_t |v_t| of its
    # sequence (the fp32 accumulation order adds far less).
    from oracle import kvq_oracle as o
    cfg = tl.oracle_cfg(spec)
    vmax = np.array([np.abs(o.dequantized_cache(cfg, k, v)[1]).max() for k, v in zip(ks, vs)])
    bound = 2.0 ** -9 * vmax[:, None, None]
    for o_ in outs:
        assert np.abs(o_ - want).max() <= tl.DECODE_TOL
        assert (np.abs(o_ - outs[-1]) <= bound).all(), np.abs(o_ - outs[-1]).max()
    assert cache.workspace_status() == 0


def test_repeated_decode_is_stable():
    """Many calls on one cache agree to rounding level and leave the
    workspace clean (no state leaks between calls).  They need not agree bit for bit:
    inside a CTA the warps claim groups dynamically, so the order in which a
    warp accumulates its groups varies from call to call."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 32, 8, 8, 4224)
    rng = np.random.default_rng(25)
    ks, vs, q = _workload_arrays(rng, [4113] * 8, 8, 128, 32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    qd = tl.to_device(q, "fp16")
    first = cache.decode(qd).float().clone()
    for _ in range(20):
        again = cache.decode(qd).float()
        assert torch.isfinite(again).all()
        # the weights p are rounded to fp16 relative to the running max, which
        # depends on the order a warp meets its groups: outputs move by a
        # fraction of that rounding (measured <= 5e-5); 1e-4 is 20x below
        # the decode tolerance
        assert ((again - first).abs() <= first.abs() * 2.0 ** -10 + 1e-4).all()
    assert cache.workspace_status() == 0


def test_decode_after_appends_tracks_tail():
    """Decode between single-token appends (tail lengths 0..G-1 and flushes)."""
    K = tl.kvq()
    spec = K.CacheSpec(2, 2, 32, 128, 32, 8, 2, 512)
    rng = np.random.default_rng(26)
    ks, vs, q = _workload_arrays(rng, [60, 45], 8, 128, 32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, [ks[0][:40], ks[1][:20]], [vs[0][:40], vs[1][:20]], "fp16")
    qd = tl.to_device(q, "fp16")
    for t in range(25):
        a, b = 40 + t, 20 + t
        tl.append_chunks(cache, [ks[0][a:a + 1], ks[1][b:b + 1]], [vs[0][a:a + 1], vs[1][b:b + 1]],
                         "fp16")
        out = cache.decode(qd)
        want = tl.oracle_decode(spec, [ks[0][:a + 1], ks[1][:b + 1]], [vs[0][:a + 1], vs[1][:b + 1]], q)
        assert tl.decode_error(out, want) <= tl.DECODE_TOL, t


def test_decode_errors_are_reported_before_launch():
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 64, 1, 1, 2, 64)
    cache = K.KVQCache(spec)
    rng = np.random.default_rng(27)
    ks, vs, q = _workload_arrays(rng, [10, 0], 1, 64, 1)
    tl.append_chunks(cache, ks, vs, "fp16")
    qd = tl.to_device(q, "fp16")
    with pytest.raises(K.KvqError) as ei:
        cache.decode(qd)                 # sequence 1 is empty
    assert ei.value.status == 5
    out = cache.decode(qd[:1])           # the first sequence alone is fine
    torch.cuda.synchronize()
    assert out.shape == (1, 1, 64)
    with pytest.raises(K.KvqError) as ei:
        cache.decode(tl.to_device(np.zeros((3, 1, 64), np.float32), "fp16"))
    assert ei.value.status == 4          # more sequences than the cache holds
    with pytest.raises(ValueError):
        cache.decode(qd[:, :, :32].contiguous())   # wrong head_dim


def test_graph_replay_of_append_and_decode():
    """A captured (append 1 token, decode) pair replayed several times gives
    the same outputs as eager calls and keeps the device lengths right."""
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 32, 8, 4, 512)
    rng = np.random.default_rng(28)
    ks, vs, q = _workload_arrays(rng, [100, 63, 31, 200], 8, 128, 32)
    steps = 40
    nk, nv, _ = _workload_arrays(rng, [steps] * 4, 8, 128, 32)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    qd = tl.to_device(q, "fp16")
    slot_k = torch.zeros((4, 8, 128), dtype=torch.float16, device="cuda")
    slot_v = torch.zeros_like(slot_k)
    out = torch.empty((4, 32, 128), dtype=torch.float16, device="cuda")
    cache.decode(qd, out=out)   # warm the launch configuration before capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        cache.append(slot_k, slot_v, [1, 1, 1, 1], stream=s)
        cache.decode(qd, out=out, stream=s)
    # capture does not run the kernels; the host mirror advanced once
    cache.sync_lengths()
    assert cache.lengths()[:4] == [100, 63, 31, 200]
    for t in range(steps):
        slot_k.copy_(tl.to_device(np.stack([nk[b][t] for b in range(4)]), "fp16"))
        slot_v.copy_(tl.to_device(np.stack([nv[b][t] for b in range(4)]), "fp16"))
        graph.replay()
        torch.cuda.synchronize()
        hk = [np.concatenate([ks[b], nk[b][:t + 1]]) for b in range(4)]
        hv = [np.concatenate([vs[b], nv[b][:t + 1]]) for b in range(4)]
        if t % 9 == 0 or t == steps - 1:
            want = tl.oracle_decode(spec, hk, hv, q)
            assert tl.decode_error(out, want) <= tl.DECODE_TOL, t
    cache.sync_lengths()
    assert cache.lengths()[:4] == [100 + steps, 63 + steps, 31 + steps, 200 + steps]
    tl.check_cache_against_oracle(cache, hk, hv)
