"""The roofline numerators of bench.py against independent sources: the
library's own layout (block sizes from kvq_layout_for, on CPU) and the
oracle's widths and segments.  The bench divides these bytes by the
measured time, so a wrong byte model would misstate every fraction."""
import os
import sys
from types import SimpleNamespace

import pytest

from oracle import kvq_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.fixture(scope="module")
def kvq():
    from asymmetric_kv_cache_b200 import kvq as mod
    return mod


def _layout_bytes(kvq, kb, vb, G, d, hq, hkv, n, window=0, sink=0, akvq_delta=0):
    """Bytes one decode reads by the library's layout and the oracle's
    segments and widths."""
    cfg = kvq.make_config(kb, vb, G, d, hq, hkv, 1, max(n, 1), window=window, sink=sink,
                          akvq_delta=akvq_delta)
    lay = kvq.layout_for(cfg)
    ocfg = o.Config(kb, vb, G, d, hq, hkv, window=window, sink=sink, akvq_delta=akvq_delta)
    S, Nq, T = o.segments(ocfg, n)
    groups = Nq // G
    if akvq_delta:
        qb = sum(lay["block_bytes"] if o.akvq_key_bits(ocfg, g, n) == kb else lay["akvq_block_bytes"]
                 for g in range(groups))
    else:
        qb = groups * lay["block_bytes"]
    return hkv * (qb + (S + T) * 4 * d) + hq * d * 2


@pytest.mark.parametrize("n", [1, 31, 32, 4113, 131072])
@pytest.mark.parametrize("kb,vb,G", [(4, 2, 32), (2, 2, 32), (4, 2, 64), (2, 4, 32)])
def test_decode_byte_model(kvq, n, kb, vb, G):
    import bench
    got, _ = bench.decode_bytes_one_seq(n, G, 128, kb, vb, 8, 32)
    assert got == _layout_bytes(kvq, kb, vb, G, 128, 32, 8, n)


@pytest.mark.parametrize("n,window,sink", [(131072, 128, 0), (131072, 128, 32), (5000, 64, 5),
                                           (100, 128, 32), (20, 0, 32)])
def test_decode_byte_model_windows(kvq, n, window, sink):
    import bench
    got, _ = bench.decode_bytes_one_seq(n, 32, 128, 2, 2, 8, 32, window=window, sink=sink)
    assert got == _layout_bytes(kvq, 2, 2, 32, 128, 32, 8, n, window=window, sink=sink)


@pytest.mark.parametrize("n,delta", [(131072, 1024), (5000, 256), (3000, 1024), (700, 64)])
def test_decode_byte_model_adaptive(kvq, n, delta):
    import bench
    got, _ = bench.decode_bytes_one_seq(n, 32, 128, 4, 2, 8, 32, akvq_delta=delta)
    assert got == _layout_bytes(kvq, 4, 2, 32, 128, 32, 8, n, akvq_delta=delta)


def test_step_byte_model(kvq):
    """The llama3_8b step's numerator (Workload.algorithmic_bytes)."""
    import bench
    args = SimpleNamespace(workload="llama3_8b", steps=20, warmup=5, copies=0, e2e_steps=8)
    wl = bench.Workload(args, 0)
    lens = [4113, 4096, 4127, 1, 33, 4113, 4100, 4200]
    want = sum(_layout_bytes(kvq, 4, 2, 32, 128, 32, 8, n) - 32 * 128 * 2 for n in lens)
    assert wl.algorithmic_bytes(lens) == want + 8 * 32 * 128 * 2
