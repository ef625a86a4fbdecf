"""Seeded synthetic inputs for the quantized-KV decode path.

This module only draws random numbers and shapes them; it holds none of the
quantization or attention arithmetic, so both the CPU oracle's tests and the
CUDA path's tests/benchmark take their inputs from here.

Workloads (shapes and value distributions) follow the long-context decode
settings that the pages' experiments talk about; no dataset or model weights
are involved:

* keys: per-channel outliers.  "[Framework] The Asymmetric Key-Value Cache
  Compression", §III, says key outliers sit in fixed channels across the whole
  sequence; we draw each channel's standard deviation sigma_c = exp(N(0, 1))
  once per (sequence, kv-head, channel) and keys as sigma_c * N(0, 1).
* values: per-token magnitude spikes (same page, same section: value outliers
  are tied to individual tokens); each token's L2 norm is exp(N(0, 0.5^2)) and
  its direction is uniform on the sphere.
* queries: N(0, 1).

All generators use numpy's PCG64 (``numpy.random.default_rng``) seeded with
0x4B5651 + workload index unless a seed is given.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 0x4B5651


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even).

    Returns (values as float32, raw uint16 bit patterns).  Used to hand the
    same bf16 query to the GPU (as bits) and to the oracle (as exact floats).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    bits = u.astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    return vals, bits


def keys_channel_outliers(rng, n: int, hkv: int, d: int) -> np.ndarray:
    """Keys [n, hkv, d] float32 with a log-normal(0, 1) std per channel."""
    sigma = np.exp(rng.standard_normal((1, hkv, d)))
    return (sigma * rng.standard_normal((n, hkv, d))).astype(np.float32)


def values_token_norms(rng, n: int, hkv: int, d: int, sigma: float = 0.5) -> np.ndarray:
    """Values [n, hkv, d] float32: token norm exp(N(0, sigma^2)), uniform direction."""
    g = rng.standard_normal((n, hkv, d))
    g /= np.linalg.norm(g, axis=-1, keepdims=True)
    r = np.exp(sigma * rng.standard_normal((n, hkv, 1)))
    return (r * g).astype(np.float32)


@dataclass
class Workload:
    """One synthetic decode workload.

    ``keys[b]``/``values[b]`` are [n_b, hkv, d] arrays in ``kv_dtype``
    (numpy float16 or float32); ``q`` is [batch, hq, d] float32 holding values
    exactly representable in ``q_dtype``; ``q_bits`` holds the raw uint16 bits
    for bf16 queries.
    """

    name: str
    k_bits: int
    v_bits: int
    group: int
    head_dim: int
    n_q_heads: int
    n_kv_heads: int
    lens: list
    kv_dtype: str
    q_dtype: str
    keys: list = field(default_factory=list)
    values: list = field(default_factory=list)
    q: np.ndarray | None = None
    q_bits: np.ndarray | None = None
    seed: int = 0

    @property
    def batch(self) -> int:
        return len(self.lens)


def _cast(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "fp16":
        return x.astype(np.float16)
    if dtype == "fp32":
        return x.astype(np.float32)
    raise ValueError(dtype)


def _queries(rng, batch, hq, d, q_dtype):
    q = rng.standard_normal((batch, hq, d)).astype(np.float32)
    if q_dtype == "fp16":
        return q.astype(np.float16).astype(np.float32), None
    if q_dtype == "bf16":
        return bf16_round(q)
    return q, None


def tiny(seed: int | None = None, n: int = 256) -> Workload:
    """Tiny decode: B=1, Hq=Hkv=1, d=64, context 256, fp32 K/V ~ N(0,1),
    4 of 64 key channels scaled x10, K4/V2, G=32, fp32 query."""
    seed = SEED_BASE + 0 if seed is None else seed
    rng = np.random.default_rng(seed)
    d = 64
    k = rng.standard_normal((n, 1, d)).astype(np.float32)
    v = rng.standard_normal((n, 1, d)).astype(np.float32)
    outl = rng.permutation(d)[:4]
    k[:, :, outl] *= 10.0
    q, qb = _queries(rng, 1, 1, d, "fp32")
    return Workload("tiny", 4, 2, 32, d, 1, 1, [n], "fp32", "fp32", [k], [v], q, qb, seed)


def _lognormal_workload(name, seed, lens, hq, hkv, d, kb, vb, g, q_dtype):
    rng = np.random.default_rng(seed)
    keys, values = [], []
    for n in lens:
        keys.append(keys_channel_outliers(rng, n, hkv, d).astype(np.float16))
        values.append(values_token_norms(rng, n, hkv, d).astype(np.float16))
    q, qb = _queries(rng, len(lens), hq, d, q_dtype)
    return Workload(name, kb, vb, g, d, hq, hkv, list(lens), "fp16", q_dtype,
                    keys, values, q, qb, seed)


def llama3_8b(seed: int | None = None, batch: int = 8, n: int = 4096 + 17) -> Workload:
    """Llama-3-8B-shaped layer: B=8, 32q/8kv, d=128, context 4096+17, K4/V2, G=32."""
    seed = SEED_BASE + 1 if seed is None else seed
    return _lognormal_workload("llama3_8b", seed, [n] * batch, 32, 8, 128, 4, 2, 32, "fp16")


def long_ctx(seed: int | None = None, n: int = 131072) -> Workload:
    """Long context: B=1, 32q/8kv, d=128, context 131072, K2/V2, G=32."""
    seed = SEED_BASE + 2 if seed is None else seed
    return _lognormal_workload("long_ctx", seed, [n], 32, 8, 128, 2, 2, 32, "fp16")


def llama70b_conc(seed: int | None = None, batch: int = 64, lo: int = 1024,
                  hi: int = 8192) -> Workload:
    """70B-shaped high concurrency: B=64, 64q/8kv, d=128, contexts ~ U{lo..hi},
    bf16 queries, K4/V2, G=64."""
    seed = SEED_BASE + 4 if seed is None else seed
    rng = np.random.default_rng(seed ^ 0x5EED)
    lens = [int(x) for x in rng.integers(lo, hi + 1, size=batch)]
    return _lognormal_workload("llama70b_conc", seed, lens, 64, 8, 128, 4, 2, 64, "bf16")


def quant_append(seed: int | None = None, batch: int = 4, n: int = 32768,
                 hkv: int = 8, d: int = 128) -> Workload:
    """Prefill-quantize workload: B=4 x 32768 tokens x 8 kv-heads x d=128, fp16,
    K4/V2, G=32 (queries unused)."""
    seed = SEED_BASE + 3 if seed is None else seed
    return _lognormal_workload("quant_append", seed, [n] * batch, hkv, hkv, d, 4, 2, 32, "fp16")


def append_stream(seed: int, n_seq: int, steps: int, hkv: int, d: int):
    """Per-step decode appends: ``steps`` arrays of one token per sequence,
    each [n_seq, hkv, d] fp16 (same distributions as above)."""
    rng = np.random.default_rng(seed)
    ks, vs = [], []
    for _ in range(steps):
        ks.append(keys_channel_outliers(rng, n_seq, hkv, d).astype(np.float16))
        vs.append(values_token_norms(rng, n_seq, hkv, d).astype(np.float16))
    return ks, vs


WORKLOADS = {
    "tiny": tiny,
    "llama3_8b": llama3_8b,
    "long_ctx": long_ctx,
    "quant_append": quant_append,
    "llama70b_conc": llama70b_conc,
}
