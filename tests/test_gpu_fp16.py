"""fp16 decode baseline (comparison kernel) against the oracle's exact
attention on the same fp16 keys and values, element by element."""
import numpy as np
import pytest
import torch

from oracle import kvq_oracle as o
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


def _run(lens, hq, hkv, d, max_tokens, seed, q_dtype="fp16"):
    K = tl.kvq()
    rng = np.random.default_rng(seed)
    n_seq = len(lens)
    k = np.zeros((n_seq, hkv, max_tokens, d), np.float16)
    v = np.zeros((n_seq, hkv, max_tokens, d), np.float16)
    for b, n in enumerate(lens):
        from asymmetric_kv_cache_b200 import inputs
        k[b, :, :n] = inputs.keys_channel_outliers(rng, n, hkv, d).transpose(1, 0, 2)
        v[b, :, :n] = inputs.values_token_norms(rng, n, hkv, d).transpose(1, 0, 2)
    q = rng.standard_normal((n_seq, hq, d)).astype(np.float32)
    if q_dtype == "fp16":
        q = q.astype(np.float16).astype(np.float32)
    qd = tl.to_device(q, q_dtype)
    out = K.decode_fp16(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(),
                        torch.tensor(lens, dtype=torch.int32, device="cuda"), qd)
    torch.cuda.synchronize()
    want = np.stack([o.attention(q[b], k[b, :, :n].transpose(1, 0, 2).astype(np.float64),
                                 v[b, :, :n].transpose(1, 0, 2).astype(np.float64), hq // hkv)
                     for b, n in enumerate(lens)])
    return tl.decode_error(out, want)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("gqa", [1, 4, 8, 16])
def test_fp16_decode_small(d, gqa):
    hkv = 2
    lens = [1, 15, 16, 17, 100, 333]
    err = _run(lens, hkv * gqa, hkv, d, 352, 500 + d + gqa)
    assert err <= tl.DECODE_TOL, err


@pytest.mark.parametrize("q_dtype", ["bf16", "fp32"])
def test_fp16_decode_query_dtypes(q_dtype):
    err = _run([700, 33, 1500], 32, 8, 128, 1536, 77, q_dtype)
    assert err <= tl.DECODE_TOL, err


def test_fp16_decode_llama3_8b_shape():
    """The bench's layer shape: 8 sequences x 4113 tokens, 32q / 8kv, d 128."""
    err = _run([4113] * 8, 32, 8, 128, 4128, 78)
    assert err <= tl.DECODE_TOL, err


def test_fp16_decode_more_sequences_than_one_launch():
    """2100 sequences: two launches of the decode + combine pair."""
    lens = [1 + (7 * b) % 40 for b in range(2100)]
    err = _run(lens, 4, 1, 64, 48, 79)
    assert err <= tl.DECODE_TOL, err
