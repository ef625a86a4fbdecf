"""Pins for LAYOUT v2 as the oracle states it (CPU only).

The pages only ask for a fixed-width layout ("avoids irregular memory
layouts", summary page; "a fixed per-token bit count", NOVA-KV abstract on
the "WUSH-KV" page); the exact permutation is this library's definition.
Pins: hand-worked positions (tests/golden/layout_positions.json), section
sizes equal to the closed-form bytes per token, bijection, and round trip.
"""
import json
import os

import numpy as np
import pytest

from oracle import kvq_oracle as o

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold():
    with open(os.path.join(GOLD, "layout_positions.json")) as f:
        return json.load(f)


def test_hand_positions():
    g = _gold()
    for e in g["key"]:
        assert o.key_code_position(e["t"], e["c"], e["d"], e["bits"]) == (e["byte"], e["bit"]), e
    for e in g["value"]:
        assert o.value_code_position(e["t"], e["c"], e["d"], e["bits"]) == (e["byte"], e["bit"]), e
    for e in g["key_meta"]:
        assert o.key_meta_index(e["c"], e["d"]) == e["slot"], e
    for e in g["value_meta"]:
        assert o.value_meta_index(e["t"], e["j"], e["J"]) == e["slot"], e
    for e in g["tail"]:
        assert o.tail_key_index(e["t"], e["c"], e["d"]) == e["key_index"]
        assert o.tail_value_index(e["t"], e["c"], e["d"]) == e["value_index"]


@pytest.mark.parametrize("kb,vb,G,d,expect", [
    (4, 2, 32, 128, 128),   # K4/V2, G=32: 64 + 16 + 32 + 16 bytes per token-head
    (2, 2, 32, 128, 96),    # K2/V2
    (4, 2, 64, 128, 112),   # K4/V2, G=64
    (4, 2, 32, 64, 64),     # d=64: 32 + 8 + 16 + 8
    (4, 4, 32, 128, 160),
    (2, 4, 64, 64, 56),
])
def test_bytes_per_token_head(kb, vb, G, d, expect):
    cfg = o.Config(kb, vb, G, d, 1, 1)
    # closed form: codes d*(kb+vb)/8 + key pair 4d/G + value pairs 4d/G
    assert d * (kb + vb) / 8 + 4 * d / G + 4 * d / G == expect
    assert o.bytes_per_token_head(cfg) == expect
    sec = o.block_sections(cfg)
    for name, (off, size) in sec.items():
        if name != "total":
            assert off % 16 == 0 and size % 16 == 0


@pytest.mark.parametrize("kb,vb,G,d", [(4, 2, 32, 128), (2, 2, 32, 128),
                                        (4, 2, 64, 128), (4, 2, 32, 64),
                                        (4, 4, 64, 64), (2, 4, 32, 128)])
def test_pack_is_bijective_and_round_trips(kb, vb, G, d):
    cfg = o.Config(kb, vb, G, d, 1, 1)
    # every code slot is hit exactly once (asserted while tabulating)
    o._slot_table("k", G, d, kb)
    o._slot_table("v", G, d, vb)
    rng = np.random.default_rng(7)
    J = d // G
    kc = rng.integers(0, 2 ** kb, (3, G, d)).astype(np.uint8)
    vc = rng.integers(0, 2 ** vb, (3, G, d)).astype(np.uint8)
    ks = rng.standard_normal((3, d)).astype(np.float16)
    kz = rng.standard_normal((3, d)).astype(np.float16)
    vs = rng.standard_normal((3, G, J)).astype(np.float16)
    vz = rng.standard_normal((3, G, J)).astype(np.float16)
    blk = o.pack_blocks(cfg, kc, ks, kz, vc, vs, vz)
    assert blk.shape == (3, o.block_bytes(cfg))
    back = o.unpack_blocks(cfg, blk)
    for a, b in zip(back, (kc, ks, kz, vc, vs, vz)):
        np.testing.assert_array_equal(a.view(np.uint8), np.asarray(b).view(np.uint8))


def test_single_code_lands_where_stated():
    """A block with one non-zero key code and one non-zero value code has
    exactly those bits set, at the hand-worked positions."""
    cfg = o.Config(4, 2, 32, 128, 1, 1)
    kc = np.zeros((32, 128), np.uint8)
    vc = np.zeros((32, 128), np.uint8)
    kc[9, 19] = 0xB
    vc[9, 19] = 0x2
    z = np.zeros(128, np.float16)
    zz = np.zeros((32, 4), np.float16)
    blk = o.pack_block(cfg, kc, z, z, vc, zz, zz)
    nz = np.nonzero(blk)[0].tolist()
    sec = o.block_sections(cfg)
    assert nz == [595, sec["vcodes"][0] + 195]
    assert blk[595] == 0xB
    assert blk[sec["vcodes"][0] + 195] == 0x2 << 4


def test_tail_arrays_placement():
    cfg = o.Config(4, 2, 32, 128, 1, 1)
    rng = np.random.default_rng(8)
    tk = rng.standard_normal((5, 128)).astype(np.float16)
    tv = rng.standard_normal((5, 128)).astype(np.float16)
    ak, av = o.tail_arrays(cfg, tk, tv)
    # hand-worked slots: key t*d + c; value ((t//2)*d + c)*2 + t%2
    assert ak[4 * 128 + 3] == tk[4, 3]
    assert av[(2 * 128 + 3) * 2 + 0] == tv[4, 3]
    assert av[(1 * 128 + 7) * 2 + 1] == tv[3, 7]
    assert np.count_nonzero(ak[5 * 128:]) == 0
