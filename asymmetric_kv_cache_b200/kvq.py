"""Python binding of libkvq (ctypes): argument marshalling only.

Every step of the quantize / append / decode path runs in the CUDA library;
PyTorch supplies device memory and the current stream.  The library must be
built (``python -m asymmetric_kv_cache_b200.build``); importing this module
without it raises ImportError, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# KVQ_LIBRARY=debug selects libkvq_debug.so, the same library with the
# decode kernels' range checks compiled in (a failed check is reported by
# kvq_workspace_status instead of faulting)
_NAME = "libkvq_debug.so" if os.environ.get("KVQ_LIBRARY") == "debug" else "libkvq.so"
LIB_PATH = os.path.join(_HERE, _NAME)

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{_NAME} not found at {LIB_PATH}; build it with "
                      "`python -m asymmetric_kv_cache_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

KVQ_OK = 0
STATUS_NAMES = {
    0: "KVQ_OK", 1: "KVQ_ERR_NULL", 2: "KVQ_ERR_CONFIG", 3: "KVQ_ERR_BUFFER_TOO_SMALL",
    4: "KVQ_ERR_CAPACITY", 5: "KVQ_ERR_EMPTY", 6: "KVQ_ERR_DTYPE", 7: "KVQ_ERR_CUDA",
    8: "KVQ_ERR_ALIGN", 9: "KVQ_ERR_ARG", 10: "KVQ_ERR_DEVICE",
}
DTYPE_CODES = {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2}
LAYOUT_VERSION = 2


class KvqConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "k_bits", "v_bits", "group", "head_dim", "n_q_heads", "n_kv_heads",
        "max_seqs", "max_tokens", "layout_version", "window", "sink", "rotate", "akvq_delta")]


class KvqLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "total_bytes", "lens_offset", "counters_offset", "blocks_offset", "block_bytes", "max_groups",
        "tails_offset", "tail_bytes", "kcodes_offset", "kscale_offset", "kmin_offset",
        "vcodes_offset", "vscale_offset", "vmin_offset", "tail_slots", "sinks_offset",
        "sink_bytes", "sink_slots", "akvq_block_bytes", "akvq_kscale_offset", "akvq_kmin_offset",
        "akvq_vcodes_offset", "akvq_vscale_offset", "akvq_vmin_offset")]


_c_status = ctypes.c_int32
_vp = ctypes.c_void_p
_P = ctypes.POINTER


def _sig(name, args, res=_c_status):
    fn = getattr(_lib, name)
    fn.argtypes = args
    fn.restype = res
    return fn


kvq_status_string = _sig("kvq_status_string", [_c_status], ctypes.c_char_p)
kvq_last_error = _sig("kvq_last_error", [], ctypes.c_char_p)
kvq_layout_for = _sig("kvq_layout_for", [_P(KvqConfig), _P(KvqLayout)])
kvq_cache_required_bytes = _sig("kvq_cache_required_bytes",
                                [_P(KvqConfig), _P(ctypes.c_size_t), _P(ctypes.c_size_t)])
kvq_cache_create = _sig("kvq_cache_create", [_P(KvqConfig), _vp, ctypes.c_size_t, _P(_vp)])
kvq_cache_destroy = _sig("kvq_cache_destroy", [_vp])
kvq_reset = _sig("kvq_reset", [_vp, _vp])
kvq_append = _sig("kvq_append", [_vp, _vp, _vp, ctypes.c_int32, _P(ctypes.c_int32),
                                 ctypes.c_int32, _vp])
kvq_decode = _sig("kvq_decode", [_vp, _vp, ctypes.c_int32, _vp, ctypes.c_int32, _vp,
                                 ctypes.c_size_t, _vp])
kvq_workspace_init = _sig("kvq_workspace_init", [_vp, ctypes.c_size_t, _vp])
kvq_workspace_status = _sig("kvq_workspace_status", [_vp, _vp])
kvq_cache_config = _sig("kvq_cache_config", [_vp, _P(KvqConfig)])
kvq_cache_layout = _sig("kvq_cache_layout", [_vp, _P(KvqLayout)])
kvq_get_lengths = _sig("kvq_get_lengths", [_vp, _P(ctypes.c_int32), ctypes.c_int32])
kvq_sync_lengths = _sig("kvq_sync_lengths", [_vp, _vp])
kvq_decode_noalloc = _sig("kvq_decode_noalloc", [_vp, _vp, ctypes.c_int32, _vp, ctypes.c_int32, _vp])
kvq_noalloc_scratch_bytes = _sig("kvq_noalloc_scratch_bytes", [], ctypes.c_size_t)
kvq_fp16_workspace_bytes = _sig("kvq_fp16_workspace_bytes",
                                [ctypes.c_int32] * 4 + [ctypes.POINTER(ctypes.c_size_t)])
kvq_decode_fp16 = _sig("kvq_decode_fp16",
                       [_vp, _vp, _vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                        ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_int32, _vp, _vp,
                        ctypes.c_size_t, _vp])

EXPORTED = ["kvq_status_string", "kvq_last_error", "kvq_layout_for", "kvq_cache_required_bytes",
            "kvq_cache_create", "kvq_cache_destroy", "kvq_reset", "kvq_append", "kvq_decode",
            "kvq_workspace_init", "kvq_workspace_status", "kvq_cache_config",
            "kvq_cache_layout", "kvq_get_lengths", "kvq_sync_lengths", "kvq_decode_noalloc",
            "kvq_noalloc_scratch_bytes", "kvq_fp16_workspace_bytes", "kvq_decode_fp16"]


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = kvq_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")


def check(status: int, where: str) -> None:
    if status != KVQ_OK:
        raise KvqError(status, where)


def make_config(k_bits, v_bits, group, head_dim, n_q_heads, n_kv_heads, max_seqs,
                max_tokens, window=0, sink=0, rotate=0, akvq_delta=0) -> KvqConfig:
    return KvqConfig(k_bits, v_bits, group, head_dim, n_q_heads, n_kv_heads, max_seqs,
                     max_tokens, LAYOUT_VERSION, window, sink, int(rotate), int(akvq_delta))


def required_bytes(cfg: KvqConfig) -> tuple[int, int]:
    c, w = ctypes.c_size_t(), ctypes.c_size_t()
    check(kvq_cache_required_bytes(ctypes.byref(cfg), ctypes.byref(c), ctypes.byref(w)),
          "kvq_cache_required_bytes")
    return c.value, w.value


def layout_for(cfg: KvqConfig) -> dict:
    lay = KvqLayout()
    check(kvq_layout_for(ctypes.byref(cfg), ctypes.byref(lay)), "kvq_layout_for")
    return {n: int(getattr(lay, n)) for n, _ in KvqLayout._fields_}


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


@dataclass
class CacheSpec:
    k_bits: int
    v_bits: int
    group: int
    head_dim: int
    n_q_heads: int
    n_kv_heads: int
    max_seqs: int
    max_tokens: int
    window: int = 0     # R: recent tokens kept in fp16 beyond the partial group
    sink: int = 0       # S: first tokens of each sequence kept in fp16
    rotate: int = 0     # 1: tokens, q and the output rotated by H / sqrt(d)
    akvq_delta: int = 0  # Delta > 0: position-adaptive key bits (4 early/recent, 2 middle)


class KVQCache:
    """A quantized KV cache in a torch-owned device buffer.

    ``append(k, v, n_new)`` adds tokens (prefill, per-step append, flush);
    ``decode(q)`` returns fp16 attention outputs [n_seq, n_q_heads, d].
    """

    def __init__(self, spec: CacheSpec, device="cuda"):
        self.spec = spec
        self.cfg = make_config(spec.k_bits, spec.v_bits, spec.group, spec.head_dim,
                               spec.n_q_heads, spec.n_kv_heads, spec.max_seqs, spec.max_tokens,
                               spec.window, spec.sink, spec.rotate, spec.akvq_delta)
        cache_bytes, ws_bytes = required_bytes(self.cfg)
        self.buffer = torch.empty(cache_bytes, dtype=torch.uint8, device=device)
        self.workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=device)
        torch.cuda.synchronize(self.buffer.device)
        h = _vp()
        check(kvq_cache_create(ctypes.byref(self.cfg), self.buffer.data_ptr(), cache_bytes,
                               ctypes.byref(h)), "kvq_cache_create")
        self._h = h
        self.layout = self._layout()

    def _layout(self) -> dict:
        lay = KvqLayout()
        check(kvq_cache_layout(self._h, ctypes.byref(lay)), "kvq_cache_layout")
        return {n: int(getattr(lay, n)) for n, _ in KvqLayout._fields_}

    def close(self):
        if getattr(self, "_h", None):
            kvq_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def lengths(self, n=None) -> list:
        n = self.spec.max_seqs if n is None else n
        arr = (ctypes.c_int32 * n)()
        check(kvq_get_lengths(self._h, arr, n), "kvq_get_lengths")
        return list(arr)

    def sync_lengths(self, stream=None):
        check(kvq_sync_lengths(self._h, _stream(stream)), "kvq_sync_lengths")

    def reset(self, stream=None):
        check(kvq_reset(self._h, _stream(stream)), "kvq_reset")

    def append(self, k: torch.Tensor, v: torch.Tensor, n_new, stream=None):
        """k, v: [sum(n_new), n_kv_heads, d] device tensors (fp16/bf16/fp32)."""
        if k.dtype != v.dtype or k.dtype not in DTYPE_CODES:
            raise ValueError("k and v must share one of fp16/bf16/fp32")
        n_new = [int(x) for x in n_new]
        rows = sum(n_new)
        want = (rows, self.spec.n_kv_heads, self.spec.head_dim)
        if tuple(k.shape) != want or tuple(v.shape) != want:
            raise ValueError(f"k and v must be {want}, got {tuple(k.shape)} and {tuple(v.shape)}")
        arr = (ctypes.c_int32 * len(n_new))(*n_new)
        kp = _dev_ptr(k, "k") if k.numel() else None
        vp = _dev_ptr(v, "v") if v.numel() else None
        check(kvq_append(self._h, kp, vp, DTYPE_CODES[k.dtype], arr, len(n_new), _stream(stream)),
              "kvq_append")

    def decode(self, q: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """q: [n_seq, n_q_heads, d] device tensor; returns fp16 [n_seq, n_q_heads, d]."""
        if q.dtype not in DTYPE_CODES:
            raise ValueError("q must be fp16, bf16 or fp32")
        if q.dim() != 3 or tuple(q.shape[1:]) != (self.spec.n_q_heads, self.spec.head_dim):
            raise ValueError(f"q must be [n_seq, {self.spec.n_q_heads}, {self.spec.head_dim}], "
                             f"got {tuple(q.shape)}")
        n_seq = q.shape[0]
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float16, device=q.device)
        elif out.dtype != torch.float16 or out.shape != q.shape:
            raise ValueError("out must be an fp16 tensor shaped like q")
        check(kvq_decode(self._h, _dev_ptr(q, "q"), DTYPE_CODES[q.dtype], _dev_ptr(out, "out"),
                         n_seq, self.workspace.data_ptr(), self.workspace.numel(),
                         _stream(stream)), "kvq_decode")
        return out

    def decode_noalloc(self, q: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
        """kvq_decode_noalloc: decode into a caller-given ``out`` using the
        library's fixed device scratch (no allocation, no workspace)."""
        if q.dtype not in DTYPE_CODES:
            raise ValueError("q must be fp16, bf16 or fp32")
        if q.dim() != 3 or tuple(q.shape[1:]) != (self.spec.n_q_heads, self.spec.head_dim):
            raise ValueError(f"q must be [n_seq, {self.spec.n_q_heads}, {self.spec.head_dim}]")
        if out.dtype != torch.float16 or out.shape != q.shape:
            raise ValueError("out must be an fp16 tensor shaped like q")
        check(kvq_decode_noalloc(self._h, _dev_ptr(q, "q"), DTYPE_CODES[q.dtype],
                                 _dev_ptr(out, "out"), q.shape[0], _stream(stream)),
              "kvq_decode_noalloc")
        return out

    def workspace_status(self, stream=None) -> int:
        return kvq_workspace_status(self.workspace.data_ptr(), _stream(stream))

    # ---- views of the raw buffer (tests, checkpointing) ----
    def block_bytes(self, seq: int, kv_head: int, n_groups: int) -> torch.Tensor:
        L = self.layout
        base = L["blocks_offset"] + ((seq * self.spec.n_kv_heads + kv_head) * L["max_groups"]) * L["block_bytes"]
        return self.buffer[base: base + n_groups * L["block_bytes"]].view(n_groups, L["block_bytes"])

    def tail_halves(self, seq: int, kv_head: int) -> tuple[torch.Tensor, torch.Tensor]:
        L = self.layout
        W, d = L["tail_slots"], self.spec.head_dim
        base = L["tails_offset"] + (seq * self.spec.n_kv_heads + kv_head) * L["tail_bytes"]
        raw = self.buffer[base: base + L["tail_bytes"]].view(torch.float16)
        return raw[: W * d], raw[W * d: 2 * W * d]

    def sink_halves(self, seq: int, kv_head: int) -> tuple[torch.Tensor, torch.Tensor]:
        L = self.layout
        SW, d = L["sink_slots"], self.spec.head_dim
        base = L["sinks_offset"] + (seq * self.spec.n_kv_heads + kv_head) * L["sink_bytes"]
        raw = self.buffer[base: base + L["sink_bytes"]].view(torch.float16)
        return raw[: SW * d], raw[SW * d: 2 * SW * d]

    def device_lengths(self) -> torch.Tensor:
        L = self.layout
        return self.buffer[L["lens_offset"]: L["lens_offset"] + 4 * self.spec.max_seqs].view(torch.int32)


def decode_fp16(k: torch.Tensor, v: torch.Tensor, lens: torch.Tensor, q: torch.Tensor,
                out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """kvq_decode_fp16, the unquantized comparison kernel: k, v fp16 CUDA
    tensors [n_seq, n_kv_heads, max_tokens, head_dim], lens int32 CUDA
    [n_seq], q [n_seq, n_q_heads, head_dim] fp16/bf16/fp32."""
    if k.dtype != torch.float16 or v.dtype != torch.float16 or k.shape != v.shape or k.dim() != 4:
        raise ValueError("k and v must be fp16 [n_seq, n_kv_heads, max_tokens, head_dim]")
    n_seq, hkv, max_tokens, d = k.shape
    if q.dtype not in DTYPE_CODES or q.dim() != 3 or q.shape[0] != n_seq or q.shape[2] != d:
        raise ValueError("q must be [n_seq, n_q_heads, head_dim] fp16/bf16/fp32")
    if lens.dtype != torch.int32 or tuple(lens.shape) != (n_seq,):
        raise ValueError("lens must be int32 [n_seq]")
    hq = q.shape[1]
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float16, device=q.device)
    nbytes = ctypes.c_size_t()
    check(kvq_fp16_workspace_bytes(n_seq, hq, hkv, d, ctypes.byref(nbytes)), "kvq_fp16_workspace_bytes")
    if workspace is None or workspace.numel() < nbytes.value:
        workspace = torch.zeros(nbytes.value, dtype=torch.uint8, device=q.device)
    check(kvq_decode_fp16(_dev_ptr(k, "k"), _dev_ptr(v, "v"), _dev_ptr(lens, "lens"), max_tokens,
                          n_seq, hq, hkv, d, _dev_ptr(q, "q"), DTYPE_CODES[q.dtype],
                          _dev_ptr(out, "out"), workspace.data_ptr(), workspace.numel(),
                          _stream(stream)), "kvq_decode_fp16")
    return out
