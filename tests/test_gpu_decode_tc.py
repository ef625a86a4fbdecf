"""GPU parity of the tcgen05 decode kernel (opt-in, KVQ_DECODE_TC=1).

The kernel covers d = 128, 32-token groups, 2-bit values and GQA groups of
at most 4 heads, with one CTA per SM (calls with at most one unit per SM).
Its outputs must be within 2e-3 (max abs) of the oracle's fp64 attention on
the dequantized cache, like the mma.sync kernel's: ragged batches with tails
shorter than a group, one token, exact multiples of G, every query dtype,
and the two benchmark workloads it covers at full size.
"""
import numpy as np
import pytest
import torch

from asymmetric_kv_cache_b200 import inputs
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _tc_path(monkeypatch):
    monkeypatch.setenv("KVQ_DECODE_TC", "1")


def _arrays(rng, lens, hkv, d, hq, q_dtype="fp16"):
    ks = [inputs.keys_channel_outliers(rng, n, hkv, d).astype(np.float16) for n in lens]
    vs = [(inputs.values_token_norms(rng, n, hkv, d) * 2.0).astype(np.float16) for n in lens]
    q = rng.standard_normal((len(lens), hq, d)).astype(np.float32)
    if q_dtype == "fp16":
        q = q.astype(np.float16).astype(np.float32)
    elif q_dtype == "bf16":
        q = tl.bf16_values(q)
    return ks, vs, q


def _decode(spec, ks, vs, q, q_dtype):
    K = tl.kvq()
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    out = cache.decode(tl.to_device(q, q_dtype))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    return cache, out


@pytest.mark.parametrize("kb", [4, 2])
@pytest.mark.parametrize("gqa", [1, 2, 4])
def test_tc_decode_ragged(kb, gqa):
    K = tl.kvq()
    hkv = 2
    lens = [1, 31, 32, 33, 5 * 32 + 13, 9 * 32, 640 + 7]
    spec = K.CacheSpec(kb, 2, 32, 128, hkv * gqa, hkv, len(lens), 1024)
    rng = np.random.default_rng(500 + kb * 7 + gqa)
    ks, vs, q = _arrays(rng, lens, hkv, 128, hkv * gqa)
    _, out = _decode(spec, ks, vs, q, "fp16")
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


@pytest.mark.parametrize("q_dtype", ["fp16", "bf16", "fp32"])
def test_tc_decode_query_dtypes(q_dtype):
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 8, 2, 3, 2048)
    rng = np.random.default_rng(31)
    ks, vs, q = _arrays(rng, [700, 1500, 33], 2, 128, 8, q_dtype)
    _, out = _decode(spec, ks, vs, q, q_dtype)
    err = tl.decode_error(out, tl.oracle_decode(spec, ks, vs, q))
    assert err <= tl.DECODE_TOL, err


@pytest.mark.parametrize("name", ["llama3_8b", "long_ctx"])
def test_tc_decode_workloads_full_size(name):
    K = tl.kvq()
    w = inputs.WORKLOADS[name]()
    spec = K.CacheSpec(w.k_bits, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                       w.batch, max(w.lens))
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, w.keys, w.values, w.kv_dtype)
    out = cache.decode(tl.to_device(w.q, w.q_dtype))
    torch.cuda.synchronize()
    assert cache.workspace_status() == 0
    hk = [x.astype(np.float16) for x in w.keys]
    hv = [x.astype(np.float16) for x in w.values]
    err = tl.decode_error(out, tl.oracle_decode(spec, hk, hv, w.q))
    assert err <= tl.DECODE_TOL, (name, err)


def test_tc_and_mma_kernels_agree(monkeypatch):
    """Both kernels on the same cache: the same attention up to rounding."""
    K = tl.kvq()
    spec = K.CacheSpec(2, 2, 32, 128, 16, 4, 2, 8192)
    rng = np.random.default_rng(41)
    ks, vs, q = _arrays(rng, [8191, 4100], 4, 128, 16)
    cache, out_tc = _decode(spec, ks, vs, q, "fp16")
    monkeypatch.setenv("KVQ_DECODE_TC", "0")
    out_mma = cache.decode(tl.to_device(q, "fp16"))
    torch.cuda.synchronize()
    d = (out_tc.float() - out_mma.float()).abs().max().item()
    assert d <= 2e-3, d
