"""kvq_decode_noalloc: decode for callers that cannot allocate device memory
(inside a CUDA-graph capture, plugins whose framework owns all device memory,
no allocation after start-up).  It uses the library's fixed device scratch
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


def test_noalloc_rejects_too_many_units():
    """4096 sequences x 64 kv heads x 8 head slices = 2^21 units: their
    tickets alone fill the fixed scratch, so the call must refuse (clear
    error, nothing launched) rather than overrun it."""
    K = tl.kvq()
    cfg = K.make_config(4, 2, 32, 64, 64 * 64, 64, 4096, 32)
    cache_bytes, _ = K.required_bytes(cfg)
    assert cache_bytes < 3 << 30
    buf = torch.empty(cache_bytes, dtype=torch.uint8, device="cuda")
    h = ctypes.c_void_p()
    assert K.kvq_cache_create(ctypes.byref(cfg), buf.data_ptr(), cache_bytes, ctypes.byref(h)) == 0
    stream = torch.cuda.current_stream().cuda_stream
    k = torch.zeros((1, 64, 64), dtype=torch.float16, device="cuda")
    n_new = (ctypes.c_int32 * 1)(1)
    assert K.kvq_append(h, k.data_ptr(), k.data_ptr(), 0, n_new, 1, stream) == 0
    q = torch.zeros((1, 64 * 64, 64), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    st = K.kvq_decode_noalloc(h, q.data_ptr(), 0, out.data_ptr(), 1, stream)
    assert st == 4 and b"fixed scratch" in K.kvq_last_error()
    torch.cuda.synchronize()
    K.kvq_cache_destroy(h)
