"""The C ABI without a GPU: the library loads, exports every function that
include/kvq.h declares, reports sizes that agree with the oracle's byte
accounting, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from oracle import kvq_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq():
    from asymmetric_kv_cache_b200 import build
    build.build()
    from asymmetric_kv_cache_b200 import kvq as mod
    return mod


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(kvq):
    lib = ctypes.CDLL(kvq.LIB_PATH)
    names = _declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(kvq.EXPORTED) == names


def _cfg(kvq, **kw):
    base = dict(k_bits=4, v_bits=2, group=32, head_dim=128, n_q_heads=32, n_kv_heads=8,
                max_seqs=8, max_tokens=4224)
    base.update(kw)
    return kvq.make_config(**base)


@pytest.mark.parametrize("kb,vb,G,d", [(4, 2, 32, 128), (2, 2, 32, 128), (4, 2, 64, 128),
                                        (4, 2, 32, 64), (2, 4, 64, 64)])
def test_layout_matches_oracle_sections(kvq, kb, vb, G, d):
    cfg = _cfg(kvq, k_bits=kb, v_bits=vb, group=G, head_dim=d)
    lay = kvq.layout_for(cfg)
    sec = o.block_sections(o.Config(kb, vb, G, d, 32, 8))
    assert lay["block_bytes"] == sec["total"][1]
    for name in ("kcodes", "kscale", "kmin", "vcodes", "vscale", "vmin"):
        assert lay[name + "_offset"] == sec[name][0]
    assert lay["max_groups"] == 4224 // G
    assert lay["tail_bytes"] == 4 * G * d
    for k in ("lens_offset", "blocks_offset", "tails_offset", "total_bytes"):
        assert lay[k] % 256 == 0
    assert lay["blocks_offset"] >= 4 * 8
    assert lay["tails_offset"] >= lay["blocks_offset"] + 8 * 8 * lay["max_groups"] * lay["block_bytes"]
    assert lay["total_bytes"] >= lay["tails_offset"] + 8 * 8 * lay["tail_bytes"]
    cache, ws = kvq.required_bytes(cfg)
    assert cache == lay["total_bytes"]
    assert ws > 0


@pytest.mark.parametrize("G,R", [(32, 0), (32, 32), (32, 128), (64, 16), (64, 1024)])
def test_tail_ring_size_from_library(kvq, G, R):
    """The tail is a ring of R + G token slots (K and V fp16)."""
    lay = kvq.layout_for(_cfg(kvq, group=G, window=R))
    assert lay["tail_slots"] == o.Config(4, 2, G, 128, 32, 8, window=R).tail_slots == R + G
    assert lay["tail_bytes"] == 4 * (R + G) * 128
    assert lay["total_bytes"] >= lay["tails_offset"] + 8 * 8 * lay["tail_bytes"]


@pytest.mark.parametrize("S", [0, 4, 16, 33, 1024])
def test_sink_area_size_from_library(kvq, S):
    """The sink area holds S rounded up to 16 token slots (K and V fp16)."""
    lay = kvq.layout_for(_cfg(kvq, sink=S, window=64))
    sw = o.sink_slots(o.Config(4, 2, 32, 128, 32, 8, window=64, sink=S))
    assert lay["sink_slots"] == sw and lay["sink_bytes"] == 4 * sw * 128
    assert lay["sinks_offset"] % 256 == 0
    assert lay["sinks_offset"] >= lay["tails_offset"] + 8 * 8 * lay["tail_bytes"]
    assert lay["total_bytes"] >= lay["sinks_offset"] + 8 * 8 * lay["sink_bytes"]


def test_bytes_per_token_head_from_library(kvq):
    """128 B per token-head for K4/V2 G=32, 96 for K2/V2, 112 for K4/V2 G=64."""
    for kb, G, expect in ((4, 32, 128), (2, 32, 96), (4, 64, 112)):
        lay = kvq.layout_for(_cfg(kvq, k_bits=kb, group=G))
        assert lay["block_bytes"] / G == expect


@pytest.mark.parametrize("field,value", [
    ("k_bits", 3), ("k_bits", 8), ("v_bits", 1), ("group", 16), ("group", 128),
    ("head_dim", 96), ("head_dim", 256), ("n_q_heads", 30), ("n_kv_heads", 0),
    ("max_seqs", 0), ("max_tokens", 0), ("layout_version", 1), ("layout_version", 3),
    ("window", -16), ("window", 24), ("window", 1040), ("sink", -1), ("sink", 1025),
])
def test_bad_config_rejected(kvq, field, value):
    cfg = _cfg(kvq)
    setattr(cfg, field, value)
    s = kvq.kvq_cache_required_bytes(ctypes.byref(cfg), None, None)
    assert s == 2  # KVQ_ERR_CONFIG
    assert kvq.kvq_last_error()
    h = ctypes.c_void_p()
    assert kvq.kvq_cache_create(ctypes.byref(cfg), 256, 1 << 30, ctypes.byref(h)) == 2
    assert not h.value


@pytest.mark.parametrize("kw", [dict(akvq_delta=48), dict(akvq_delta=-32),
                                dict(akvq_delta=(1 << 20) + 32), dict(akvq_delta=64, k_bits=2),
                                dict(akvq_delta=64, window=32), dict(akvq_delta=64, sink=4)])
def test_bad_position_adaptive_config_rejected(kvq, kw):
    """Delta: a multiple of the group size in [0, 2^20], with 4-bit keys and
    neither a recent window nor a sink window."""
    cfg = _cfg(kvq, **kw)
    assert kvq.kvq_cache_required_bytes(ctypes.byref(cfg), None, None) == 2
    assert "akvq_delta" in kvq.kvq_last_error().decode()


@pytest.mark.parametrize("vb,G,d", [(2, 32, 128), (4, 64, 128), (2, 32, 64), (2, 64, 64)])
def test_position_adaptive_block_sections(kvq, vb, G, d):
    """The 2-bit-key block of a position-adaptive cache has the sections of a
    plain 2-bit-key block and sits at the start of the 4-bit slot."""
    cfg = _cfg(kvq, v_bits=vb, group=G, head_dim=d, akvq_delta=4 * G)
    assert kvq.kvq_cache_required_bytes(ctypes.byref(cfg), None, None) == 0
    lay = kvq.layout_for(cfg)
    sec2 = o.block_sections(o.Config(2, vb, G, d, 32, 8))
    assert lay["akvq_block_bytes"] == sec2["total"][1]
    for name in ("kscale", "kmin", "vcodes", "vscale", "vmin"):
        assert lay["akvq_" + name + "_offset"] == sec2[name][0]
    assert lay["block_bytes"] == o.block_sections(o.Config(4, vb, G, d, 32, 8))["total"][1]
    assert lay["akvq_block_bytes"] < lay["block_bytes"] and lay["akvq_block_bytes"] % 16 == 0


def test_head_dim_64_with_group_64_is_valid(kvq):
    cfg = _cfg(kvq, head_dim=64, group=64)
    assert kvq.kvq_cache_required_bytes(ctypes.byref(cfg), None, None) == 0


def test_too_many_slots_rejected(kvq):
    cfg = _cfg(kvq, max_seqs=100000, max_tokens=1 << 20, group=32)
    assert kvq.kvq_cache_required_bytes(ctypes.byref(cfg), None, None) == 2


def test_create_checks_buffer_before_touching_the_device(kvq):
    cfg = _cfg(kvq)
    cache, _ = kvq.required_bytes(cfg)
    h = ctypes.c_void_p()
    assert kvq.kvq_cache_create(ctypes.byref(cfg), None, cache, ctypes.byref(h)) == 1
    assert kvq.kvq_cache_create(ctypes.byref(cfg), 256, cache - 1, ctypes.byref(h)) == 3
    assert kvq.kvq_cache_create(ctypes.byref(cfg), 256 + 16, cache, ctypes.byref(h)) == 8
    assert kvq.kvq_cache_create(None, 256, cache, ctypes.byref(h)) == 1
    assert kvq.kvq_cache_create(ctypes.byref(cfg), 256, cache, None) == 1


def test_null_handle_calls(kvq):
    n = (ctypes.c_int32 * 1)(1)
    assert kvq.kvq_append(None, 16, 16, 0, n, 1, None) == 1
    assert kvq.kvq_decode(None, 16, 0, 16, 1, 256, 1 << 20, None) == 1
    assert kvq.kvq_reset(None, None) == 1
    assert kvq.kvq_get_lengths(None, None, 0) == 1
    assert kvq.kvq_workspace_init(None, 16, None) == 1
    assert kvq.kvq_cache_destroy(None) == 0
    assert kvq.kvq_status_string(5).startswith(b"KVQ_ERR_EMPTY")
    assert kvq.kvq_status_string(0) == b"KVQ_OK"


def test_fp16_baseline_argument_checks(kvq):
    """The fp16 comparison entry point validates on the host (no GPU use)."""
    import ctypes
    n = ctypes.c_size_t()
    assert kvq.kvq_fp16_workspace_bytes(8, 32, 8, 128, ctypes.byref(n)) == 0
    assert n.value > 0 and n.value % 256 == 0
    CONFIG, ARG, CAP, NULL, ALIGN, SMALL = 2, 9, 4, 1, 8, 3
    assert kvq.kvq_fp16_workspace_bytes(8, 32, 8, 96, ctypes.byref(n)) == CONFIG
    assert kvq.kvq_fp16_workspace_bytes(8, 30, 8, 128, ctypes.byref(n)) == CONFIG
    assert kvq.kvq_fp16_workspace_bytes(0, 32, 8, 128, ctypes.byref(n)) == ARG
    assert kvq.kvq_fp16_workspace_bytes(9000, 32, 8, 128, ctypes.byref(n)) == CAP
    p = 1 << 20   # never dereferenced: every call below fails its checks first
    assert kvq.kvq_decode_fp16(None, p, p, 64, 1, 4, 1, 64, p, 0, p, p, 1 << 30, None) == NULL
    assert kvq.kvq_decode_fp16(p + 2, p, p, 64, 1, 4, 1, 64, p, 0, p, p, 1 << 30, None) == ALIGN
    assert kvq.kvq_decode_fp16(p, p, p, 64, 1, 4, 1, 64, p, 0, p, p, 16, None) == SMALL
    assert kvq.kvq_decode_fp16(p, p, p, 0, 1, 4, 1, 64, p, 0, p, p, 1 << 30, None) == ARG
    assert kvq.kvq_decode_fp16(p, p, p, 64, 1, 4, 1, 64, p, 7, p, p, 1 << 30, None) != 0
