"""Shared helpers of the GPU parity tests: drive the CUDA library through its
C ABI (asymmetric_kv_cache_b200.kvq) and compare what it wrote with the CPU
oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import kvq_oracle as o

DECODE_TOL = 2e-3   # max |out_gpu - out_oracle|, fp16 outputs


def kvq():
    from asymmetric_kv_cache_b200 import kvq as mod
    return mod


def oracle_cfg(spec) -> o.Config:
    return o.Config(spec.k_bits, spec.v_bits, spec.group, spec.head_dim, spec.n_q_heads,
                    spec.n_kv_heads, window=getattr(spec, "window", 0),
                    sink=getattr(spec, "sink", 0), rotate=bool(getattr(spec, "rotate", 0)),
                    akvq_delta=getattr(spec, "akvq_delta", 0))


def to_device(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Host array -> CUDA tensor of the named dtype (values already exactly
    representable for fp16/bf16 inputs made by the generators)."""
    if dtype == "fp16":
        return torch.from_numpy(np.ascontiguousarray(x, np.float16)).cuda()
    if dtype == "fp32":
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).cuda()
    raise ValueError(dtype)


def bf16_values(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to bf16 (what the device will see)."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def append_chunks(cache, chunks_k, chunks_v, dtype: str):
    """Append per-sequence chunks (lists of [n_b, hkv, d] arrays, n_b may be 0)."""
    n_new = [c.shape[0] for c in chunks_k]
    hkv, d = cache.spec.n_kv_heads, cache.spec.head_dim
    if sum(n_new):
        k = np.concatenate([c.reshape(-1, hkv, d) for c in chunks_k])
        v = np.concatenate([c.reshape(-1, hkv, d) for c in chunks_v])
    else:
        k = np.zeros((0, hkv, d), np.float32)
        v = np.zeros((0, hkv, d), np.float32)
    cache.append(to_device(k, dtype), to_device(v, dtype), n_new)


def expected_tail_mask(cfg: o.Config, N: int, T: int):
    """Element masks of the defined slots of the fp16 tail rings: the slots of
    positions N .. N + T - 1."""
    W, d = cfg.tail_slots, cfg.head_dim
    mk = np.zeros(W * d, bool)
    mv = np.zeros(W * d, bool)
    for p in range(N, N + T):
        t = o.tail_slot(cfg, p)
        for c in range(d):
            mk[o.tail_key_index(t, c, d)] = True
            mv[o.tail_value_index(t, c, d)] = True
    return mk, mv


def check_cache_against_oracle(cache, hist_k, hist_v, seqs=None, group_sample=None):
    """Bytes of every full group and the defined tail slots of each sequence
    must equal the oracle's (bit-exact).  hist_k[b]: [n_b, hkv, d] fp16 token
    history of sequence b.  group_sample: optional function (n_groups) ->
    indices of the groups to compare."""
    cfg = oracle_cfg(cache.spec)
    seqs = range(len(hist_k)) if seqs is None else seqs
    lens = cache.lengths()
    dev_lens = cache.device_lengths().cpu().numpy()
    for b in seqs:
        n = hist_k[b].shape[0]
        assert lens[b] == n, (b, lens[b], n)
        assert dev_lens[b] == n, (b, dev_lens[b], n)
        Sb, Nq, T = o.segments(cfg, n)
        N = Sb + Nq                      # first tail position
        ng = Nq // cfg.group
        gsel = np.arange(ng) if group_sample is None else np.asarray(group_sample(ng), np.int64)
        if len(gsel):
            toks = (Sb + gsel[:, None] * cfg.group + np.arange(cfg.group)[None, :]).reshape(-1)
            kk = hist_k[b][toks].reshape(len(gsel), cfg.group, cfg.n_kv_heads, cfg.head_dim)
            vv = hist_v[b][toks].reshape(len(gsel), cfg.group, cfg.n_kv_heads, cfg.head_dim)
            q = o.quantize_group(cfg, kk.transpose(2, 0, 1, 3), vv.transpose(2, 0, 1, 3))
            want = o.pack_blocks(cfg, *q)                       # [hkv, len(gsel), bytes]
            for h in range(cfg.n_kv_heads):
                got = cache.block_bytes(b, h, ng).cpu().numpy()[gsel]
                if not np.array_equal(got, want[h]):
                    bad = np.argwhere(got != want[h])
                    g0, byte0 = bad[0]
                    raise AssertionError(
                        f"seq {b} head {h}: {len(bad)} bytes differ; first at group "
                        f"{gsel[g0]} byte {byte0}: got {got[g0, byte0]:#04x} want {want[h][g0, byte0]:#04x}")
        if T:
            mk, mv = expected_tail_mask(cfg, N, T)
            for h in range(cfg.n_kv_heads):
                tk, tv = o.tail_arrays(cfg, hist_k[b][N:, h], hist_v[b][N:, h], first=N)
                gk, gv = cache.tail_halves(b, h)
                gk = gk.cpu().numpy()
                gv = gv.cpu().numpy()
                assert np.array_equal(gk[mk].view(np.uint16), tk[mk].view(np.uint16)), (b, h, "tail K")
                assert np.array_equal(gv[mv].view(np.uint16), tv[mv].view(np.uint16)), (b, h, "tail V")
        if Sb:
            d = cfg.head_dim
            mk = np.zeros(o.sink_slots(cfg) * d, bool)
            mv = np.zeros(o.sink_slots(cfg) * d, bool)
            for t in range(Sb):
                for c in range(d):
                    mk[o.tail_key_index(t, c, d)] = True
                    mv[o.tail_value_index(t, c, d)] = True
            for h in range(cfg.n_kv_heads):
                sk, sv = o.sink_arrays(cfg, hist_k[b][:Sb, h], hist_v[b][:Sb, h])
                gk, gv = cache.sink_halves(b, h)
                gk = gk.cpu().numpy()
                gv = gv.cpu().numpy()
                assert np.array_equal(gk[mk].view(np.uint16), sk[mk].view(np.uint16)), (b, h, "sink K")
                assert np.array_equal(gv[mv].view(np.uint16), sv[mv].view(np.uint16)), (b, h, "sink V")


def oracle_decode(spec, hist_k, hist_v, q: np.ndarray) -> np.ndarray:
    cfg = oracle_cfg(spec)
    return np.stack([o.decode(cfg, hist_k[b], hist_v[b], q[b]) for b in range(len(hist_k))])


def decode_error(got: torch.Tensor, want: np.ndarray) -> float:
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all()
    return float(np.abs(g - want).max())
