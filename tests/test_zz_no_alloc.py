"""kvq_decode_noalloc: decode for callers that cannot allocate device memory
(plugins whose host framework owns all device memory, deployments with no
allocation after start-up).  It uses the library's fixed device scratch
instead of a caller workspace; its outputs must match kvq_decode's within the
decode tolerance, on two calls in a row (the second call finds the array as
the first one left it).  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from asymmetric_kv_cache_b200 import inputs
from tests import kvq_testlib as tl

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode():
    K = tl.kvq()
    spec = K.CacheSpec(4, 2, 32, 128, 32, 8, 4, 2048)
    rng = np.random.default_rng(4242)
    lens = [1500, 777, 33, 2000]
    ks = [inputs.keys_channel_outliers(rng, n, 8, 128).astype(np.float16) for n in lens]
    vs = [inputs.values_token_norms(rng, n, 8, 128).astype(np.float16) for n in lens]
    q = rng.standard_normal((4, 32, 128)).astype(np.float16)
    cache = K.KVQCache(spec)
    tl.append_chunks(cache, ks, vs, "fp16")
    qd = torch.from_numpy(q).cuda()
    ref = cache.decode(qd).clone()
    torch.cuda.synchronize()
    assert K.kvq_noalloc_scratch_bytes() == 8 << 20
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        # through the C ABI directly
        st = K.kvq_decode_noalloc(cache._h, qd.data_ptr(), 0, out.data_ptr(), 4,
                                  torch.cuda.current_stream().cuda_stream)
        assert st == 0, K.kvq_last_error()
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.isfinite(got).all(), call
        diff = np.abs(got - ref.float().cpu().numpy()).max()
        assert diff <= tl.DECODE_TOL, (call, diff)
    want = tl.oracle_decode(spec, ks, vs, q.astype(np.float32))
    assert tl.decode_error(out, want) <= tl.DECODE_TOL


def test_noalloc_small_call_on_a_large_cache():
    """A one-sequence call on a cache built for 4096 sequences x 64 kv heads x
    8 head slices: only the units of the call's own launch need split
    records, so it fits the fixed scratch and matches kvq_decode."""
    K = tl.kvq()
    cfg = K.make_config(4, 2, 32, 64, 64 * 64, 64, 4096, 32)
    cache_bytes, ws_bytes = K.required_bytes(cfg)
    assert cache_bytes < 3 << 30
    buf = torch.empty(cache_bytes, dtype=torch.uint8, device="cuda")
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    h = ctypes.c_void_p()
    assert K.kvq_cache_create(ctypes.byref(cfg), buf.data_ptr(), cache_bytes, ctypes.byref(h)) == 0
    stream = torch.cuda.current_stream().cuda_stream
    rng = np.random.default_rng(99)
    k = torch.from_numpy(rng.standard_normal((20, 64, 64)).astype(np.float16)).cuda()
    v = torch.from_numpy(rng.standard_normal((20, 64, 64)).astype(np.float16)).cuda()
    n_new = (ctypes.c_int32 * 1)(20)
    assert K.kvq_append(h, k.data_ptr(), v.data_ptr(), 0, n_new, 1, stream) == 0
    q = torch.from_numpy(rng.standard_normal((1, 64 * 64, 64)).astype(np.float16)).cuda()
    ref = torch.empty_like(q)
    assert K.kvq_decode(h, q.data_ptr(), 0, ref.data_ptr(), 1, ws.data_ptr(), ws_bytes, stream) == 0
    out = torch.full_like(q, float("nan"))
    st = K.kvq_decode_noalloc(h, q.data_ptr(), 0, out.data_ptr(), 1, stream)
    assert st == 0, K.kvq_last_error()
    torch.cuda.synchronize()
    diff = (out.float() - ref.float()).abs().max().item()
    assert diff <= tl.DECODE_TOL, diff
    K.kvq_cache_destroy(h)


def test_noalloc_rejects_a_call_beyond_the_scratch():
    """2048 sequences x 64 kv heads x 8 head slices = 2^20 units in one
    launch: their split records and tickets (12 bytes each) alone exceed the
    8 MiB scratch, so the call must refuse on the host with a clear error
    and launch nothing (q and out are never touched, so small buffers do)."""
    K = tl.kvq()
    S = 2048
    cfg = K.make_config(4, 2, 32, 64, 64 * 64, 64, S, 32)
    cache_bytes, _ = K.required_bytes(cfg)
    assert cache_bytes < 3 << 30
    buf = torch.empty(cache_bytes, dtype=torch.uint8, device="cuda")
    h = ctypes.c_void_p()
    assert K.kvq_cache_create(ctypes.byref(cfg), buf.data_ptr(), cache_bytes, ctypes.byref(h)) == 0
    stream = torch.cuda.current_stream().cuda_stream
    k = torch.zeros((S, 64, 64), dtype=torch.float16, device="cuda")
    n_new = (ctypes.c_int32 * S)(*([1] * S))
    assert K.kvq_append(h, k.data_ptr(), k.data_ptr(), 0, n_new, S, stream) == 0
    small = torch.zeros(1024, dtype=torch.float16, device="cuda")
    st = K.kvq_decode_noalloc(h, small.data_ptr(), 0, small.data_ptr(), S, stream)
    assert st == 4 and b"fixed scratch" in K.kvq_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(small).item() == 0
    K.kvq_cache_destroy(h)
