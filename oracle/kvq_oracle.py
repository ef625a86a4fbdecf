"""CPU oracle for decode attention over an asymmetrically quantized KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this file:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm use it.  It shares no code with the CUDA library; it is a plain,
slow restatement of what the method computes, in numpy.

What it follows
---------------
* "[Framework] The Asymmetric Key-Value Cache Compression", §III (Pillar I,
  KIVI partitioning): keys are quantized per channel, values per token, and
  the most recent tokens stay in an FP16 window.
* "Asymmetric Key-Value Quantization: 2-Bit Values and 4-Bit Keys under
  Long-Context Drift", §1: attn(Q, K, V) = softmax(Q K^T / sqrt(d)) V;
  §2.1: the output is sum_j alpha_j v_j; §3.1: keys at 4 bits, values at
  2 bits (K2/V2 is the 2-bit KIVI setting of the first page, §III).
* InnerQ abstract (page "WUSH-KV: KV Cache Quantization with Data-Adaptive
  Transforms", third abstract): per-group asymmetric quantization.

Readings where the pages are silent (each is listed in the design notes):
* quantizer: uniform asymmetric min/scale with Q = 2^b - 1 levels;
  s = fp16(fp32(max - min) / Q), z = fp16(min),
  code = clamp(rne(fp32(fp32(x - z) / s)), 0, Q), computed with the STORED
  fp16 s and z widened to fp32; s == 0 gives code 0 everywhere.
* every K/V value entering the cache is first rounded to fp16 (the cache's
  precision, the FP16 window of §III); quantization acts on those values, so
  a token quantized at prefill and one that passed through the fp16 tail give
  the same bytes.
* key groups: G consecutive tokens from position 0 of each sequence; value
  groups: G consecutive channels of one token; the tail holds the n mod G
  newest tokens of both K and V.
* recent window R (same page, §III and §V: the most recent tokens, 32 to
  128 of them, stay in FP16): with R > 0 a group is quantized only once R
  newer tokens follow it, so the tail holds between R and R + G - 1 tokens
  (all n tokens while n < R); R = 0 is the n mod G tail above.  The tail is a
  ring of R + G token slots: token p sits in slot (p - S) mod (R + G), S the
  sink window below, so tokens never move while they wait (our layout; the
  pages do not store it).
* rotation (optional; "[Framework] The Asymmetric Key-Value Cache
  Compression", §IV stage 1: Y = X H with an orthogonal +-1 Hadamard matrix
  computed by the fast Walsh-Hadamard transform; "Asymmetric Key-Value
  Quantization ...", §3.1: keys and values quantized after an FWHT
  rotation): every K and V token entering the cache is rotated over its d
  channels - converted to fp32, the radix-2 butterfly in fp32 in the fixed
  order of ``fwht_fp32``, times fp32(1/sqrt(d)) - and then rounded to
  fp16, so the whole cache (groups, tail, sink) holds rotated tokens; the
  decode rotates q the same way (in fp64 here) and rotates its output
  back (H is symmetric and H H = d I).
* sink window S (InnerQ abstract, page "WUSH-KV: KV Cache Quantization with
  Data-Adaptive Transforms", third abstract: high-precision windows for the
  recent tokens and for the attention-sink tokens): the first S tokens of a
  sequence stay in fp16; key groups are cut from position S on, and the
  recent window applies to the tokens after the sink.
* GQA: query head h reads kv head floor(h / (Hq / Hkv)).
* attention is evaluated in float64 on the dequantized cache
  x_hat = code * s + z (tail tokens exactly as stored in fp16).

The byte layout (``LAYOUT v2``) is a fixed per-group permutation of the codes
and metadata; ``key_code_position``/``value_code_position`` and the
``*_meta_index`` functions state it element by element.

Parity is pinned for every function here (see tests/test_oracle_*.py); no
function is "parity unpinned".
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np

LAYOUT_VERSION = 2


# ---------------------------------------------------------------------------
# configuration and byte accounting
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class Config:
    k_bits: int
    v_bits: int
    group: int
    head_dim: int
    n_q_heads: int
    n_kv_heads: int
    max_seqs: int = 1
    max_tokens: int = 0
    window: int = 0      # R: recent tokens kept in fp16 beyond the partial group
    sink: int = 0        # S: first tokens of a sequence kept in fp16
    rotate: bool = False # cache holds Hadamard-rotated tokens
    akvq_delta: int = 0  # position-adaptive key bits: region size Delta (0 = off)

    @property
    def tail_slots(self) -> int:   # W = R + G slots of the fp16 tail ring
        return self.window + self.group

    @property
    def gqa(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def value_groups(self) -> int:  # J: value channel groups per token
        return self.head_dim // self.group


def block_sections(cfg: Config) -> dict:
    """Byte offsets and sizes of the sections of one group block (LAYOUT v2).

    Order: key codes, key scales, key mins, value codes, value scales,
    value mins.  All scales/mins are IEEE binary16.
    """
    G, d = cfg.group, cfg.head_dim
    J = cfg.value_groups
    sizes = [
        ("kcodes", G * d * cfg.k_bits // 8),
        ("kscale", 2 * d),
        ("kmin", 2 * d),
        ("vcodes", G * d * cfg.v_bits // 8),
        ("vscale", 2 * G * J),
        ("vmin", 2 * G * J),
    ]
    out, off = {}, 0
    for name, sz in sizes:
        out[name] = (off, sz)
        off += sz
    out["total"] = (0, off)
    return out


def block_bytes(cfg: Config) -> int:
    return block_sections(cfg)["total"][1]


def bytes_per_token_head(cfg: Config) -> float:
    """Packed bytes per (token, kv-head) in a full group: codes + fp16 pairs."""
    return block_bytes(cfg) / cfg.group


def fp16_bytes_per_token_head(d: int) -> int:
    """Unquantized fp16 K and V: 2 tensors x d x 2 bytes."""
    return 2 * d * 2


def bits_per_coordinate(k_bits: int, v_bits: int, group: int = 0,
                        with_metadata: bool = False) -> float:
    """Average stored bits per K/V coordinate.

    Without metadata this is the pages' (b_K + b_V) / 2 (second page §3.1:
    (4 + 2) / 2 = 3).  With metadata, each group of ``group`` elements carries
    one fp16 (scale, min) pair = 32 bits, for keys and for values.
    """
    avg = (k_bits + v_bits) / 2.0
    if with_metadata:
        avg += 32.0 / group
    return avg


def compression_vs_fp16(k_bits, v_bits, group=0, with_metadata=False) -> float:
    return 16.0 / bits_per_coordinate(k_bits, v_bits, group, with_metadata)


def kv_cache_bytes_fp16(layers: int, heads: int, head_dim: int, tokens: int) -> int:
    """Bytes of an unquantized fp16 KV cache: K and V, 2 bytes per element."""
    return 2 * layers * heads * head_dim * 2 * tokens


# ---------------------------------------------------------------------------
# quantizer (uniform asymmetric min/scale), fp32 arithmetic
# ---------------------------------------------------------------------------
def to_fp16(x) -> np.ndarray:
    """Round to IEEE binary16, nearest-even (the cache's storage precision)."""
    return np.asarray(x).astype(np.float16)


def quantize_along(x16: np.ndarray, bits: int, axis: int):
    """Quantize fp16 values with one (scale, min) per slice along ``axis``.

    Returns (codes uint8 same shape as x16, scale fp16, min fp16) where scale
    and min have ``axis`` removed.  Steps, all in IEEE fp32 with
    round-to-nearest-even and no fused multiply-add:
      mn, mx = exact min / max over the group
      s32 = (mx - mn) / Q          ; Q = 2^bits - 1 levels
      s = fp16(s32), z = fp16(mn)  ; the stored pair
      code = clamp(rne((x - z) / s), 0, Q) using fp32(s), fp32(z);
      code = 0 for every element when s == 0.
    """
    Q = np.float32(2 ** bits - 1)
    x32 = np.asarray(x16, dtype=np.float16).astype(np.float32)
    mn = x32.min(axis=axis)
    mx = x32.max(axis=axis)
    s32 = (mx - mn) / Q                      # fp32 subtract, fp32 IEEE divide
    s16 = s32.astype(np.float16)
    z16 = mn.astype(np.float16)
    s_w = np.expand_dims(s16.astype(np.float32), axis)
    z_w = np.expand_dims(z16.astype(np.float32), axis)
    diff = x32 - z_w                         # fp32
    safe = np.where(s_w == 0, np.float32(1), s_w)
    t = diff / safe                          # fp32 IEEE divide
    codes = np.clip(np.rint(t), 0, Q)        # rint: ties to even
    codes = np.where(s_w == 0, np.float32(0), codes)
    return codes.astype(np.uint8), s16, z16


def quantize_keys(k16: np.ndarray, bits: int):
    """Per-channel key quantization of key groups.

    k16: [..., G, d] fp16 (G tokens of one kv-head per group).  One
    (scale, min) per channel, shared by the G tokens ("[Framework] The
    Asymmetric Key-Value Cache Compression", §III: quantize K per channel).
    Returns codes [..., G, d], scale [..., d], min [..., d].
    """
    return quantize_along(k16, bits, axis=-2)


def quantize_values(v16: np.ndarray, bits: int, group: int):
    """Per-token value quantization.

    v16: [..., T, d] fp16.  Each token's channels are cut into d / group
    groups of ``group`` consecutive channels, one (scale, min) per
    (token, channel group) (same page, §III: quantize V per token).
    Returns codes [..., T, d], scale [..., T, d/group], min [..., T, d/group].
    """
    d = v16.shape[-1]
    J = d // group
    shp = v16.shape[:-1] + (J, group)
    codes, s, z = quantize_along(np.asarray(v16).reshape(shp), bits, axis=-1)
    return codes.reshape(v16.shape), s, z


def dequantize(codes, scale, mn) -> np.ndarray:
    """x_hat = code * s + z in float64 (scale/min broadcast by the caller)."""
    return codes.astype(np.float64) * np.asarray(scale, np.float64) + np.asarray(mn, np.float64)


def dequantize_keys(codes, s16, z16) -> np.ndarray:
    """codes [..., G, d], s16/z16 [..., d] -> [..., G, d] float64."""
    return dequantize(codes, np.asarray(s16)[..., None, :], np.asarray(z16)[..., None, :])


def dequantize_values(codes, s16, z16, group) -> np.ndarray:
    """codes [..., T, d], s16/z16 [..., T, d/group] -> [..., T, d] float64."""
    d = codes.shape[-1]
    J = d // group
    c = codes.reshape(codes.shape[:-1] + (J, group))
    x = dequantize(c, np.asarray(s16)[..., None], np.asarray(z16)[..., None])
    return x.reshape(codes.shape)


# ---------------------------------------------------------------------------
# LAYOUT v2: element positions inside a group block
# ---------------------------------------------------------------------------
def key_code_position(t: int, c: int, d: int, bits: int):
    """(byte, bit) of key code (token t, channel c) inside the key-code section.

    Tokens are cut into tiles of 8 (nt = t // 8, r = t % 8) and channels into
    tiles of 16 (kt = c // 16, cc = c % 16 -> v = cc // 8, i = (cc % 8) // 2,
    e = cc % 2).  Lane = 4 r + i; operand p = 2 kt + v; each lane owns
    d * bits / 32 bytes per token tile, read as 32-bit words holding
    F = 16 / bits code pairs: word p // F, field (p % F) + F e, i.e. bit
    bits * field of that little-endian word.
    """
    nt, r = divmod(t, 8)
    kt, cc = divmod(c, 16)
    v, rem = divmod(cc, 8)
    i, e = divmod(rem, 2)
    lane = 4 * r + i
    p = 2 * kt + v
    F = 16 // bits
    w, f = divmod(p, F)
    bit = bits * (f + F * e)
    lane_bytes = d * bits // 32
    byte = nt * 32 * lane_bytes + lane * lane_bytes + 4 * w + bit // 8
    return byte, bit % 8


def value_code_position(t: int, c: int, d: int, bits: int):
    """(byte, bit) of value code (token t, channel c) inside the value-code section.

    Tokens are cut into tiles of 16 (kv = t // 16, tk = t % 16 ->
    kh = tk // 8, i = (tk % 8) // 2, e = tk % 2) and channels into tiles of
    16 (mt = c // 16, cm = c % 16 -> hr = cm // 8, g = cm % 8).
    Lane = 4 g + i; each lane owns d * bits / 16 bytes per token tile, read
    as 32-bit words holding F = 16 / bits code pairs; a word covers
    F / 4 channel tiles: word mt // (F/4), u = mt % (F/4),
    field 2 u + hr + (F/2) kh + F e, i.e. bit bits * field.
    """
    kv, tk = divmod(t, 16)
    kh, rem = divmod(tk, 8)
    i, e = divmod(rem, 2)
    mt, cm = divmod(c, 16)
    hr, g = divmod(cm, 8)
    lane = 4 * g + i
    F = 16 // bits
    w, u = divmod(mt, F // 4)
    bit = bits * (2 * u + hr + (F // 2) * kh + F * e)
    lane_bytes = d * bits // 16
    byte = kv * 32 * lane_bytes + lane * lane_bytes + 4 * w + bit // 8
    return byte, bit % 8


def key_meta_index(c: int, d: int) -> int:
    """Slot of channel c in the key scale (and key min) arrays of a block:
    i (d/4) + 4 kt + 2 v + e with kt = c // 16, v = (c % 16) // 8,
    i = (c % 8) // 2, e = c % 2."""
    kt, cc = divmod(c, 16)
    v, rem = divmod(cc, 8)
    i, e = divmod(rem, 2)
    return i * (d // 4) + 4 * kt + 2 * v + e


def value_meta_index(t: int, j: int, J: int) -> int:
    """Slot of (token t, channel group j) in the value scale (and min) arrays:
    ((4 kv + i) J + j) 4 + 2 kh + e with kv = t // 16, kh = (t % 16) // 8,
    i = (t % 8) // 2, e = t % 2."""
    kv, tk = divmod(t, 16)
    kh, rem = divmod(tk, 8)
    i, e = divmod(rem, 2)
    return ((4 * kv + i) * J + j) * 4 + 2 * kh + e


def tail_key_index(t: int, c: int, d: int) -> int:
    """Element index of the fp16 key-tail slot (t, c): token-major."""
    return t * d + c


def tail_value_index(t: int, c: int, d: int) -> int:
    """Element index of the fp16 value-tail slot (t, c): token pairs
    interleaved, ((t // 2) d + c) 2 + t % 2."""
    return ((t // 2) * d + c) * 2 + (t % 2)


def _code_slot_table(T: int, d: int, bits: int, pos_fn) -> np.ndarray:
    """Invert a code-position function: for every (byte, slot) of a packed
    code section, the flat index t * d + c of the code stored there.

    Slot s of a byte holds bits [s * bits, (s + 1) * bits).  Asserts that the
    position function is a bijection onto the section.
    """
    per = 8 // bits
    nbytes = T * d * bits // 8
    table = np.full((nbytes, per), -1, dtype=np.int64)
    for t in range(T):
        for c in range(d):
            byte, bit = pos_fn(t, c, d, bits)
            assert bit % bits == 0 and table[byte, bit // bits] == -1
            table[byte, bit // bits] = t * d + c
    assert (table >= 0).all()
    return table


_TABLES: dict = {}


def _slot_table(kind: str, T: int, d: int, bits: int) -> np.ndarray:
    key = (kind, T, d, bits)
    if key not in _TABLES:
        fn = key_code_position if kind == "k" else value_code_position
        _TABLES[key] = _code_slot_table(T, d, bits, fn)
    return _TABLES[key]


def pack_codes(codes: np.ndarray, bits: int, kind: str) -> np.ndarray:
    """Pack codes [..., T, d] (kind "k" or "v") into [..., T*d*bits/8] bytes."""
    T, d = codes.shape[-2:]
    table = _slot_table(kind, T, d, bits)
    flat = codes.reshape(codes.shape[:-2] + (T * d,)).astype(np.uint32)
    gathered = flat[..., table]                      # [..., nbytes, per]
    shifts = (np.arange(table.shape[1], dtype=np.uint32) * bits)
    return (gathered << shifts).sum(axis=-1).astype(np.uint8)


def unpack_codes(buf: np.ndarray, T: int, d: int, bits: int, kind: str) -> np.ndarray:
    """Inverse of ``pack_codes``: bytes [..., nbytes] -> codes [..., T, d]."""
    table = _slot_table(kind, T, d, bits)
    per = table.shape[1]
    buf = np.asarray(buf, np.uint8).astype(np.uint32)
    shifts = np.arange(per, dtype=np.uint32) * bits
    vals = (buf[..., :, None] >> shifts) & ((1 << bits) - 1)     # [..., nbytes, per]
    out = np.zeros(buf.shape[:-1] + (T * d,), dtype=np.uint8)
    out[..., table.reshape(-1)] = vals.reshape(buf.shape[:-1] + (-1,))
    return out.reshape(buf.shape[:-1] + (T, d))


def _key_meta_perm(d: int) -> np.ndarray:
    """perm[slot] = channel stored at that slot of the key scale/min arrays."""
    perm = np.full(d, -1, np.int64)
    for c in range(d):
        perm[key_meta_index(c, d)] = c
    assert (perm >= 0).all()
    return perm


def _value_meta_perm(G: int, J: int) -> np.ndarray:
    """perm[slot] = t * J + j stored at that slot of the value scale/min arrays."""
    perm = np.full(G * J, -1, np.int64)
    for t in range(G):
        for j in range(J):
            perm[value_meta_index(t, j, J)] = t * J + j
    assert (perm >= 0).all()
    return perm


def pack_blocks(cfg: Config, kc, ks, kz, vc, vs, vz) -> np.ndarray:
    """Assemble group blocks (uint8 [..., block_bytes]) from codes and fp16
    metadata: kc [..., G, d] key codes, ks/kz [..., d] fp16,
    vc [..., G, d] value codes, vs/vz [..., G, J] fp16."""
    sec = block_sections(cfg)
    G, d, J = cfg.group, cfg.head_dim, cfg.value_groups
    lead = kc.shape[:-2]
    blk = np.zeros(lead + (block_bytes(cfg),), dtype=np.uint8)
    o, n = sec["kcodes"]
    blk[..., o:o + n] = pack_codes(kc, cfg.k_bits, "k")
    o, n = sec["vcodes"]
    blk[..., o:o + n] = pack_codes(vc, cfg.v_bits, "v")
    kp, vp = _key_meta_perm(d), _value_meta_perm(G, J)
    metas = (("kscale", np.asarray(ks, np.float16)[..., kp]),
             ("kmin", np.asarray(kz, np.float16)[..., kp]),
             ("vscale", np.asarray(vs, np.float16).reshape(lead + (G * J,))[..., vp]),
             ("vmin", np.asarray(vz, np.float16).reshape(lead + (G * J,))[..., vp]))
    for name, arr in metas:
        o, n = sec[name]
        blk[..., o:o + n] = np.ascontiguousarray(arr).view(np.uint8)
    return blk


def pack_block(cfg: Config, kc, ks, kz, vc, vs, vz) -> np.ndarray:
    """One group block (see ``pack_blocks``)."""
    return pack_blocks(cfg, kc, ks, kz, vc, vs, vz)


def unpack_blocks(cfg: Config, blk: np.ndarray):
    """Inverse of ``pack_blocks``: returns (kc, ks, kz, vc, vs, vz)."""
    sec = block_sections(cfg)
    G, d, J = cfg.group, cfg.head_dim, cfg.value_groups
    blk = np.asarray(blk, dtype=np.uint8)
    lead = blk.shape[:-1]
    o, n = sec["kcodes"]
    kc = unpack_codes(blk[..., o:o + n], G, d, cfg.k_bits, "k")
    o, n = sec["vcodes"]
    vc = unpack_codes(blk[..., o:o + n], G, d, cfg.v_bits, "v")

    def half(name):
        o, n = sec[name]
        return np.ascontiguousarray(blk[..., o:o + n]).view(np.float16)

    kp, vp = _key_meta_perm(d), _value_meta_perm(G, J)
    ks = np.zeros(lead + (d,), np.float16)
    kz = np.zeros(lead + (d,), np.float16)
    ks[..., kp] = half("kscale")
    kz[..., kp] = half("kmin")
    vs = np.zeros(lead + (G * J,), np.float16)
    vz = np.zeros(lead + (G * J,), np.float16)
    vs[..., vp] = half("vscale")
    vz[..., vp] = half("vmin")
    return kc, ks, kz, vc, vs.reshape(lead + (G, J)), vz.reshape(lead + (G, J))


def unpack_block(cfg: Config, blk: np.ndarray):
    return unpack_blocks(cfg, blk)


# ---------------------------------------------------------------------------
# Hadamard rotation (fast Walsh-Hadamard transform)
# ---------------------------------------------------------------------------
def fwht_fp32(x) -> np.ndarray:
    """Unnormalized Walsh-Hadamard transform over the last axis (a power of
    two), in IEEE fp32: stages h = 1, 2, 4, ..., d/2; in each, every pair
    (j, j + h) of a block of 2h entries becomes (a + b, a - b).  Equals
    x H with H[i, j] = (-1)^popcount(i & j) (Sylvester order)."""
    y = np.array(x, dtype=np.float32)
    d = y.shape[-1]
    h = 1
    while h < d:
        y = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a, b = y[..., 0, :], y[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).reshape(y.shape[:-3] + (d,))
        h *= 2
    return y


def rotate_fp16(x) -> np.ndarray:
    """The cache's rotation of tokens x [..., d] (fp16, bf16 or fp32 values):
    fp16( fwht_fp32(x) * fp32(1 / sqrt(d)) ), every step rounded to nearest
    even."""
    x32 = np.asarray(x, dtype=np.float32)
    d = x32.shape[-1]
    scale = np.float32(1.0 / math.sqrt(d))
    return (fwht_fp32(x32) * scale).astype(np.float16)


def rotate_fp64(x) -> np.ndarray:
    """x H / sqrt(d) over the last axis in float64 (the query's rotation,
    and the inverse rotation of the output: the map is its own inverse)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    y = x.copy()
    h = 1
    while h < d:
        y = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a, b = y[..., 0, :], y[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).reshape(y.shape[:-3] + (d,))
        h *= 2
    return y / math.sqrt(d)


def cache_tokens(cfg: Config, x) -> np.ndarray:
    """What the cache stores for input tokens x [n, Hkv, d]: the fp16
    values, rotated first when ``cfg.rotate``."""
    return rotate_fp16(x) if cfg.rotate else np.asarray(x).astype(np.float16)


# ---------------------------------------------------------------------------
# the cache: groups + fp16 tail, as a function of the token history
# ---------------------------------------------------------------------------
def split_tokens(n: int, group: int, window: int = 0):
    """(N, T): tokens in quantized key groups, tokens in the fp16 tail.

    Groups are cut from position 0 and one is quantized once ``window`` (R)
    newer tokens follow it: N = G floor(max(0, n - R) / G), T = n - N, so T is
    n mod G for R = 0 and lies in [R, R + G - 1] once n >= R ("[Framework] The
    Asymmetric Key-Value Cache Compression", §III and §V).
    """
    N = group * (max(0, n - window) // group)
    return N, n - N


def segments(cfg: Config, n: int):
    """(Sb, Nq, T) for a sequence of n tokens: Sb = min(n, S) sink tokens
    (positions 0 .. Sb-1, fp16), Nq quantized tokens (positions Sb ..
    Sb+Nq-1, whole groups cut from position S), T tail tokens (the rest,
    fp16).  The tokens after the sink split as in ``split_tokens``."""
    Sb = min(n, cfg.sink)
    Nq, T = split_tokens(n - Sb, cfg.group, cfg.window)
    return Sb, Nq, T


def tail_slot(cfg: Config, p: int) -> int:
    """Slot of the fp16 tail ring that token position p (>= S) occupies
    while it is in the tail: (p - S) mod (R + G)."""
    return (p - cfg.sink) % cfg.tail_slots


def sink_slots(cfg: Config) -> int:
    """Token slots of the fp16 sink area: S rounded up to a multiple of 16
    (token s < S in slot s)."""
    return (cfg.sink + 15) // 16 * 16


def quantize_group(cfg: Config, k16: np.ndarray, v16: np.ndarray):
    """Quantize key groups and their values: k16, v16 [..., G, d] fp16.
    Returns (kc, ks, kz, vc, vs, vz)."""
    kc, ks, kz = quantize_keys(k16, cfg.k_bits)
    vc, vs, vz = quantize_values(v16, cfg.v_bits, cfg.group)
    return kc, ks, kz, vc, vs, vz


def grouped(cfg: Config, x16: np.ndarray) -> np.ndarray:
    """[n, Hkv, d] token history -> [Hkv, Nq/G, G, d] quantized groups."""
    G = cfg.group
    Sb, Nq, _ = segments(cfg, x16.shape[0])
    x = np.asarray(x16[Sb:Sb + Nq], np.float16).reshape(Nq // G, G, x16.shape[1], x16.shape[2])
    return x.transpose(2, 0, 1, 3)


def cache_image(cfg: Config, k16: np.ndarray, v16: np.ndarray, pack: bool = True):
    """Expected cache contents for one sequence.

    k16, v16: [n, Hkv, d] fp16 tokens as the cache stores them (for a
    rotating cache, ``cache_tokens(cfg, x)`` of the inputs).  Returns a dict with
    ``groups``: (kc, ks, kz, vc, vs, vz) with a leading [Hkv, n_groups] shape,
    ``blocks``: [Hkv, n_groups, block_bytes] uint8 (if ``pack``),
    ``tail_k``/``tail_v``: [Hkv, T, d] fp16 tail tokens (positions N .. n-1 in
    order), ``sink_k``/``sink_v``: [Hkv, Sb, d] fp16 sink tokens (positions
    0 .. Sb-1), N (the first tail position, Sb + Nq), T, Sb and Nq.
    """
    n = k16.shape[0]
    Sb, Nq, T = segments(cfg, n)
    N = Sb + Nq
    q = quantize_group(cfg, grouped(cfg, k16), grouped(cfg, v16))
    out = {"N": N, "T": T, "Sb": Sb, "Nq": Nq, "groups": q}
    if pack:
        out["blocks"] = pack_blocks(cfg, *q)
    out["tail_k"] = np.ascontiguousarray(np.asarray(k16[N:], np.float16).transpose(1, 0, 2))
    out["tail_v"] = np.ascontiguousarray(np.asarray(v16[N:], np.float16).transpose(1, 0, 2))
    out["sink_k"] = np.ascontiguousarray(np.asarray(k16[:Sb], np.float16).transpose(1, 0, 2))
    out["sink_v"] = np.ascontiguousarray(np.asarray(v16[:Sb], np.float16).transpose(1, 0, 2))
    return out


def tail_arrays(cfg: Config, tail_k: np.ndarray, tail_v: np.ndarray, first: int = 0):
    """Place T tail tokens [T, d], the first at sequence position ``first``,
    into the (R + G)-slot tail arrays (flat fp16, LAYOUT v2): token
    first + i goes to slot tail_slot(first + i).  Slots holding no tail token
    are zero here (their device contents are unspecified)."""
    W, d = cfg.tail_slots, cfg.head_dim
    tk = np.zeros(W * d, np.float16)
    tv = np.zeros(W * d, np.float16)
    for i in range(tail_k.shape[0]):
        t = tail_slot(cfg, first + i)
        for c in range(d):
            tk[tail_key_index(t, c, d)] = tail_k[i, c]
            tv[tail_value_index(t, c, d)] = tail_v[i, c]
    return tk, tv


def sink_arrays(cfg: Config, sink_k: np.ndarray, sink_v: np.ndarray):
    """Place the Sb sink tokens [Sb, d] into the sink arrays (flat fp16 of
    sink_slots(cfg) token slots, the tail's element order): token s in slot
    s.  Slots past Sb are zero here (their device contents are unspecified)."""
    SW, d = sink_slots(cfg), cfg.head_dim
    sk = np.zeros(SW * d, np.float16)
    sv = np.zeros(SW * d, np.float16)
    for t in range(sink_k.shape[0]):
        for c in range(d):
            sk[tail_key_index(t, c, d)] = sink_k[t, c]
            sv[tail_value_index(t, c, d)] = sink_v[t, c]
    return sk, sv


def dequantized_cache(cfg: Config, k16: np.ndarray, v16: np.ndarray):
    """K_hat, V_hat [n, Hkv, d] float64: quantized groups dequantized, the
    sink and the tail exactly as stored (fp16)."""
    n, hkv, d = k16.shape
    img = cache_image(cfg, k16, v16, pack=False)
    Sb, Nq, N = img["Sb"], img["Nq"], img["N"]
    kc, ks, kz, vc, vs, vz = img["groups"]
    kh = np.asarray(k16, np.float64).copy()   # sink and tail: the fp16 values
    vh = np.asarray(v16, np.float64).copy()
    # [Hkv, ng, G, d] -> [Nq, Hkv, d]
    kh[Sb:N] = dequantize_keys(kc, ks, kz).transpose(1, 2, 0, 3).reshape(Nq, hkv, d)
    vh[Sb:N] = dequantize_values(vc, vs, vz, cfg.group).transpose(1, 2, 0, 3).reshape(Nq, hkv, d)
    return kh, vh


# ---------------------------------------------------------------------------
# Position-adaptive key bits ("Asymmetric Key-Value Quantization: 2-Bit
# Values and 4-Bit Keys under Long-Context Drift", §3.2)
# ---------------------------------------------------------------------------
# The page gives b(p) = b_high for the recent tokens (p > n - Delta), b_mid in
# the middle and b_low for the early tokens (p <= Delta), default Delta =
# 1024, but its rationale gives the middle tokens the lowest precision and
# the early ones (attention sinks) a moderate one.  Reading taken, with the
# two key widths of this cache: the high width cfg.k_bits (4) for the early
# and the recent key groups, 2 bits in the middle; values keep cfg.v_bits.
# A group's region follows from its position and the current length n, so
# a group quantized while recent ages into the middle as the sequence grows;
# it is then requantized to 2 bits from its dequantized keys (the fp16 keys
# are gone by then).  Groups that are already in the middle when they are
# quantized (a long prefill) go to 2 bits from their fp16 keys directly, so
# the bytes depend on the append history, the widths do not.
AKVQ_LOW_BITS = 2


def akvq_key_bits(cfg: Config, g: int, n: int) -> int:
    """Key bits of quantized group g (positions gG .. gG + G - 1, counted
    from 0) in a sequence of n tokens: cfg.k_bits when all its positions
    are early (< Delta) or its last position is recent (>= n - Delta), else
    2."""
    G, D = cfg.group, cfg.akvq_delta
    if (g + 1) * G <= D or (g + 1) * G > n - D:
        return cfg.k_bits
    return AKVQ_LOW_BITS


def akvq_requantize_keys(ks: np.ndarray, kz: np.ndarray, kc: np.ndarray):
    """A high-width key group requantized to 2 bits from its dequantized keys:
    x = fp16( fp32(s) * code + fp32(z) ) (the product is exact in fp32, the
    sum rounded to nearest even, then rounded to fp16), then the quantizer
    of ``quantize_keys``.  kc [..., G, d], ks/kz [..., d] fp16."""
    s32 = np.asarray(ks, np.float16).astype(np.float32)[..., None, :]
    z32 = np.asarray(kz, np.float16).astype(np.float32)[..., None, :]
    x = (s32 * np.asarray(kc).astype(np.float32) + z32).astype(np.float16)
    return quantize_keys(x, AKVQ_LOW_BITS)


def akvq_cache_image(cfg: Config, k16: np.ndarray, v16: np.ndarray, chunks):
    """Cache contents of a position-adaptive cache after appending the token
    history [n, Hkv, d] (fp16, as stored) in chunks of the given sizes, one
    append per chunk.  At each append from n0 to n1 tokens: the groups that
    complete are quantized at their width for length n1 (keys from their
    fp16 tokens), then every group quantized earlier whose width for n1 is
    2 while it holds high-width codes is requantized (akvq_requantize_keys).
    Returns ``bits`` [ng], ``groups`` (one (kc, ks, kz, vc, vs, vz) tuple per
    group, leading [Hkv]), ``blocks`` [Hkv, ng, slot] uint8 with slot = the
    high-width block size and a 2-bit group's block packed from the start of
    its slot (the rest zero here, unspecified in the cache), and the tail as
    ``cache_image`` gives it."""
    G = cfg.group
    n_all = k16.shape[0]
    if sum(chunks) != n_all:
        raise ValueError("chunks must add up to the history length")
    if cfg.window or cfg.sink:
        raise ValueError("position-adaptive bits are defined without window and sink")
    groups, bits = [], []
    n = 0
    for nn in chunks:
        n0, n1 = n, n + nn
        for g in range(n0 // G, n1 // G):
            kk = np.asarray(k16[g * G:(g + 1) * G], np.float16).transpose(1, 0, 2)
            vv = np.asarray(v16[g * G:(g + 1) * G], np.float16).transpose(1, 0, 2)
            b = akvq_key_bits(cfg, g, n1)
            kc, ks, kz = quantize_keys(kk, b)
            vc, vs, vz = quantize_values(vv, cfg.v_bits, G)
            groups.append((kc, ks, kz, vc, vs, vz))
            bits.append(b)
        for g in range(n0 // G):
            if bits[g] == cfg.k_bits and akvq_key_bits(cfg, g, n1) == AKVQ_LOW_BITS:
                kc, ks, kz, vc, vs, vz = groups[g]
                kc2, ks2, kz2 = akvq_requantize_keys(ks, kz, kc)
                groups[g] = (kc2, ks2, kz2, vc, vs, vz)
                bits[g] = AKVQ_LOW_BITS
        n = n1
    hkv = k16.shape[1]
    slot = block_bytes(cfg)
    blocks = np.zeros((hkv, len(groups), slot), np.uint8)
    for g, (q, b) in enumerate(zip(groups, bits)):
        cb = dataclasses.replace(cfg, k_bits=b)
        blocks[:, g, :block_bytes(cb)] = pack_blocks(cb, *q)
    N = G * (n_all // G)
    return {"bits": bits, "groups": groups, "blocks": blocks, "N": N, "T": n_all - N,
            "tail_k": np.ascontiguousarray(np.asarray(k16[N:], np.float16).transpose(1, 0, 2)),
            "tail_v": np.ascontiguousarray(np.asarray(v16[N:], np.float16).transpose(1, 0, 2))}


def akvq_decode(cfg: Config, k16: np.ndarray, v16: np.ndarray, q: np.ndarray, chunks) -> np.ndarray:
    """Decode output [Hq, d] (float64) on the position-adaptive cache built by
    appending k16, v16 (fp16) in the given chunks: every group dequantized at
    its own key width, the tail as stored."""
    img = akvq_cache_image(cfg, k16, v16, chunks)
    kh = np.asarray(k16, np.float64).copy()
    vh = np.asarray(v16, np.float64).copy()
    G = cfg.group
    for g, (kc, ks, kz, vc, vs, vz) in enumerate(img["groups"]):
        kh[g * G:(g + 1) * G] = dequantize_keys(kc, ks, kz).transpose(1, 0, 2)
        vh[g * G:(g + 1) * G] = dequantize_values(vc, vs, vz, G).transpose(1, 0, 2)
    return attention(q, kh, vh, cfg.gqa)


# ---------------------------------------------------------------------------
# attention (fp64), the quantity the cache approximates
# ---------------------------------------------------------------------------
def softmax(x: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(x, axis=axis, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, gqa: int = 1) -> np.ndarray:
    """Decode attention for one sequence, float64.

    q [Hq, d]; k, v [n, Hkv, d].  Query head h attends with kv head
    h // gqa: out_h = sum_t alpha_t v_t, alpha = softmax(q_h . k_t / sqrt(d))
    ("Asymmetric Key-Value Quantization ...", §1 and §2.1).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n = k.shape[0]
    if n == 0:
        raise ValueError("attention over an empty context is undefined")
    hq, d = q.shape
    out = np.zeros((hq, d))
    for h in range(hq):
        kv = h // gqa
        logits = (k[:, kv, :] @ q[h]) / math.sqrt(d)
        alpha = softmax(logits)
        out[h] = alpha @ v[:, kv, :]
    return out


def attention_weights(q_h: np.ndarray, k_kv: np.ndarray) -> np.ndarray:
    """alpha for one query head against [n, d] keys (float64)."""
    d = q_h.shape[-1]
    return softmax((np.asarray(k_kv, np.float64) @ np.asarray(q_h, np.float64)) / math.sqrt(d))


def decode(cfg: Config, k16: np.ndarray, v16: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Decode output for one sequence on the quantized cache, float64 [Hq, d].

    k16, v16: the input token history [n, Hkv, d] (fp16 values; with
    ``cfg.rotate`` any fp16/bf16/fp32 values, rotated as the cache stores
    them).  With rotation the attention runs in the rotated domain on the
    rotated query (dot products are preserved) and its output is rotated
    back."""
    if cfg.rotate:
        kh, vh = dequantized_cache(cfg, rotate_fp16(k16), rotate_fp16(v16))
        return rotate_fp64(attention(rotate_fp64(q), kh, vh, cfg.gqa))
    kh, vh = dequantized_cache(cfg, k16, v16)
    return attention(q, kh, vh, cfg.gqa)
