"""Benchmark of the quantized-KV decode step on B200.

One step = one decode step of one attention layer over a batch: append the
new token of every sequence to the cache (quantizing and flushing a key
group whenever a tail fills) and run split-K decode attention over the
whole cache (groups + fp16 tail), on inputs already resident in HBM.

Default workload: the Llama-3-8B-shaped layer (8 sequences, 32 query / 8 kv
heads, head_dim 128, K4/V2, G = 32), contexts centred on 4096 + 17 tokens.
The step rotates over C copies of the cache (each its own buffer, > 4x L2 in
total) so every decode reads its cache from HBM; each copy's contexts start
below 4113 so that over the timed steps their mean is 4113.

Timing: W untimed warm-up steps, then exactly K steps replayed from CUDA
graphs (one graph = one round over the copies, two instances alternating,
plus one graph for the remaining K mod C steps), every graph uploaded to
the device before the timed region, no host synchronisation inside it,
bracketed by barrier + synchronize, CUDA events on the launch stream, max
over ranks.  CUDA events around every 8th decode of the last replay of
each graph give the decode kernel's own time (read after the region).  Under torchrun every rank runs its own replica
(weak scaling, no collective on the data path).

`--impl reference` times the CPU oracle (test infrastructure) on the same
workload and metric, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attn KV tokens/s on K4/V2 cache; achieved HBM GB/s vs B200 peak"
UNIT = "KV tokens/s"
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# ranks: every rank takes the same collective steps in the same order
# ---------------------------------------------------------------------------
def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time (all-reduce MAX over the default group; the
    tensor lives on `device`: CUDA under NCCL, CPU under gloo)."""
    import torch
    import torch.distributed as tdist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    tdist.barrier()
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processed the same units (weak
    scaling), divided by the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------
class Workload:
    def __init__(self, args, rank: int):
        from asymmetric_kv_cache_b200 import inputs
        self.name = args.workload
        if self.name != "llama3_8b":
            raise SystemExit(f"unknown workload {self.name}")
        self.batch, self.hq, self.hkv, self.d = 8, 32, 8, 128
        self.kb, self.vb, self.G = 4, 2, 32
        self.center = 4096 + 17
        self.K, self.W = args.steps, args.warmup
        per = L2_BYTES * 4 / (self.batch * self.hkv * self.center * 128) + 1
        self.C = args.copies or int(max(16, math.ceil(per), math.ceil(self.K / 64)))
        self.C = min(self.C, 1024)
        self.seed = inputs.SEED_BASE + 1 + 1000 * rank
        # appends per copy: step s uses copy s % C
        total = self.W + self.K
        self.n_warm = [sum(1 for s in range(self.W) if s % self.C == c) for c in range(self.C)]
        self.n_time = [sum(1 for s in range(self.W, total) if s % self.C == c) for c in range(self.C)]
        self.prefill = [self.center - self.n_warm[c] - self.n_time[c] // 2 for c in range(self.C)]
        # headroom for the end-to-end pass that follows the timed steps
        self.e2e_steps = min(args.e2e_steps, 4 * self.C)
        self.max_tokens = max(p + w + t for p, w, t in zip(self.prefill, self.n_warm, self.n_time))
        self.max_tokens += -(-self.e2e_steps // self.C) + 1

    def make_inputs(self):
        from asymmetric_kv_cache_b200 import inputs
        rng = np.random.default_rng(self.seed)
        n = max(self.prefill)
        ks = np.stack([inputs.keys_channel_outliers(rng, n, self.hkv, self.d) for _ in range(self.batch)])
        vs = np.stack([inputs.values_token_norms(rng, n, self.hkv, self.d) for _ in range(self.batch)])
        pool = 64
        nk, nv = inputs.append_stream(self.seed + 7, self.batch, pool, self.hkv, self.d)
        q = rng.standard_normal((pool, self.batch, self.hq, self.d)).astype(np.float16)
        return ks.astype(np.float16), vs.astype(np.float16), nk, nv, q

    def algorithmic_bytes(self, lens) -> int:
        """codes + fp16 (scale, min) pairs + fp16 tail + queries of one decode."""
        blk = self.G * self.d * (self.kb + self.vb) // 8 + 4 * self.d + 4 * self.d
        tot = 0
        for n in lens:
            ng, T = n // self.G, n % self.G
            tot += self.hkv * (ng * blk + T * 2 * self.d * 2)
        return tot + self.batch * self.hq * self.d * 2


def run_ours(args, rank, world, device):
    import torch
    from asymmetric_kv_cache_b200 import kvq

    wl = Workload(args, rank)
    ks, vs, nk, nv, q = wl.make_inputs()
    spec = kvq.CacheSpec(wl.kb, wl.vb, wl.G, wl.d, wl.hq, wl.hkv, wl.batch, wl.max_tokens)
    caches = []
    k_dev = torch.from_numpy(ks).to(device)   # [B, n, hkv, d]
    v_dev = torch.from_numpy(vs).to(device)
    for c in range(wl.C):
        cache = kvq.KVQCache(spec, device=device)
        P = wl.prefill[c]
        kk = k_dev[:, :P].reshape(-1, wl.hkv, wl.d).contiguous()
        vv = v_dev[:, :P].reshape(-1, wl.hkv, wl.d).contiguous()
        cache.append(kk, vv, [P] * wl.batch)
        caches.append(cache)
        if c:
            cache.workspace = caches[0].workspace   # calls never overlap: share one workspace
    del k_dev, v_dev
    pool = q.shape[0]
    nk_dev = [torch.from_numpy(x).to(device) for x in nk]
    nv_dev = [torch.from_numpy(x).to(device) for x in nv]
    q_dev = [torch.from_numpy(x).to(device) for x in q]
    out = torch.empty((wl.batch, wl.hq, wl.d), dtype=torch.float16, device=device)
    stream = torch.cuda.Stream(device=device)
    torch.cuda.synchronize(device)

    def step(s, strm):
        c = s % wl.C
        caches[c].append(nk_dev[s % pool], nv_dev[s % pool], [1] * wl.batch, stream=strm)
        caches[c].decode(q_dev[s % pool], out=out, stream=strm)

    # ---- warm-up (eager: also sets launch attributes before capture)
    with torch.cuda.stream(stream):
        for s in range(wl.W):
            step(s, stream)
    stream.synchronize()

    # ---- capture: a round covers steps W + r*C ... of every copy once
    C = wl.C
    steps_in_round = min(C, wl.K)

    # CUDA events bracket the decode of every EV-th step only: an event
    # recorded between the append and the decode keeps the decode from
    # launching as a programmatic dependent of the append, so the other
    # steps run as a user's loop would
    EV = 8

    def evented(i, n):   # the 8th, 16th, ... step of a graph (its last if it has fewer)
        return i % EV == EV - 1 or (n < EV and i == n - 1)

    def capture(n_steps, first_step):
        evs = [(torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True))
               for i in range(n_steps) if evented(i, n_steps)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_steps):
                s = first_step + i
                c = s % C
                caches[c].append(nk_dev[s % pool], nv_dev[s % pool], [1] * wl.batch, stream=stream)
                if evented(i, n_steps):
                    evs[i // EV][0].record(stream)
                caches[c].decode(q_dev[s % pool], out=out, stream=stream)
                if evented(i, n_steps):
                    evs[i // EV][1].record(stream)
        return g, evs

    # the copy of step s is s % C, so every round starts at a multiple of C
    # relative to the first timed step W; record the round in that order
    rounds = wl.K // C
    rem = wl.K - rounds * C
    gA = capture(steps_in_round, wl.W) if rounds else None
    gB = capture(steps_in_round, wl.W) if rounds > 1 else None
    gR = capture(rem, wl.W + rounds * C) if rem else None
    for cache in caches:          # capture advanced the host mirrors only
        cache.sync_lengths(stream)
    # upload every instance now, so that no first-replay cost (the graph's
    # upload to the device) falls inside the timed region
    for x in (gA, gB, gR):
        if x is not None:
            _graph_upload(x[0], stream)
    stream.synchronize()

    # host view of every copy's length at each timed step (for the metric)
    lens_at = []
    cur = [wl.prefill[c] + wl.n_warm[c] for c in range(C)]
    for s in range(wl.W, wl.W + wl.K):
        c = s % C
        cur[c] += 1
        lens_at.append(cur[c])
    kv_tokens = sum(L * wl.batch for L in lens_at)
    alg_bytes = sum(wl.algorithmic_bytes([L] * wl.batch) for L in lens_at)
    ev_bytes = None

    dist = world > 1
    if dist:
        import torch.distributed as tdist
        tdist.barrier()
    torch.cuda.synchronize(device)
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(device).uuid))
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    decode_ms = []
    elapsed_ok = True

    def collect(evs):
        nonlocal elapsed_ok
        for a, b in evs:
            try:
                decode_ms.append(a.elapsed_time(b))
            except Exception:
                elapsed_ok = False

    insts = [x for x in (gA, gB) if x is not None]
    with torch.cuda.stream(stream):
        # the GPU sleeps while the host submits the first graph, so that t0
        # is not followed by an idle gap (the sleep is outside the region)
        torch.cuda._sleep(200_000)
        t0.record(stream)
        # every graph was uploaded before t0; no host synchronisation in here
        for r in range(rounds):
            insts[r % len(insts)][0].replay()
        if gR is not None:
            gR[0].replay()
        t1.record(stream)
    t1.synchronize()
    # the decode events of the last replay of every instance (a replay
    # overwrites its events, so these are read only after t1)
    ev_idx = []
    for ii, (gx, evs) in enumerate(insts):
        last = max((r for r in range(rounds) if r % len(insts) == ii), default=None)
        if last is None:
            continue
        collect(evs)
        ev_idx += [last * C + i for i in range(steps_in_round) if evented(i, steps_in_round)]
    if gR is not None:
        collect(gR[1])
        ev_idx += [rounds * C + i for i in range(rem) if evented(i, rem)]
    if ev_idx:
        ev_bytes = statistics.fmean(wl.algorithmic_bytes([lens_at[j]] * wl.batch)
                                    for j in ev_idx)
    clocks = sampler.stop()
    total_ms = t0.elapsed_time(t1)
    if dist:
        total_ms = max_over_ranks(total_ms, device)

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, wl, caches, nk, nv, q, stream, device)
    fp16 = run_fp16_baseline(wl, ks, vs, q, stream, device)
    long_ctx = run_long_context(stream, device) if args.long_context else None
    window = (run_long_context(stream, device, window=args.window, fp16=False)
              if args.long_context and args.window else None)
    sinkw = (run_long_context(stream, device, window=args.window, sink=args.sink, fp16=False)
             if args.long_context and args.sink else None)
    akvq = (run_long_context(stream, device, akvq_delta=args.akvq_delta, fp16=False)
            if args.long_context and args.akvq_delta else None)
    rot = (run_long_context(stream, device, rotate=1, fp16=False)
           if args.long_context and args.rotate else None)
    qa = run_quant_append(stream, device) if args.other_legs else None
    c70 = run_concurrent_70b(stream, device) if args.other_legs else None

    for cache in caches:
        if cache.workspace_status(stream) != 0:
            raise RuntimeError("decode kernel reported a failed wait")

    value = weak_scaling_value(kv_tokens, world, total_ms)
    dec_avg_ms = statistics.fmean(decode_ms) if decode_ms and elapsed_ok else None
    peak, peak_kind = _peaks()
    roof = None
    if dec_avg_ms and ev_bytes:
        achieved = ev_bytes / (dec_avg_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": _traffic(),
                "kernel": "kvq decode_kernel<128,4,2,32,packed,wide> + combine_kernel<128>",
                "peak_kind": peak_kind,
                "bytes_per_launch": int(ev_bytes),
                "avg_launch_us": round(dec_avg_ms * 1e3, 3),
                "timed_launches": len(decode_ms),
                "note": "decode (+ combine when launched) of every 8th step of the last replay "
                        "of each graph, bracketed by CUDA events, read after the timed region"}
    return {
        "value": value, "ms_per_step": total_ms / wl.K, "e2e": e2e, "roofline": roof,
        "clocks": clocks, "gpu_launches": 3 * wl.K, "wl": wl, "fp16": fp16,
        "decode_ms": dec_avg_ms, "kv_tokens_per_step": kv_tokens / wl.K, "long_ctx": long_ctx,
        "window": window, "sink": sinkw, "akvq": akvq, "rot": rot, "quant_append": qa,
        "conc70b": c70,
    }


def run_fp16_baseline(wl, ks, vs, q, stream, device, iters=200):
    """The unquantized comparison kernel (kvq_decode_fp16) on the same layer
    shape: contexts of `wl.center` tokens, fp16 K/V [B, Hkv, n, d], two or
    more copies rotated so that every decode reads HBM."""
    import torch
    from asymmetric_kv_cache_b200 import kvq
    n = min(wl.center, ks.shape[1])
    one = wl.batch * wl.hkv * n * wl.d * 2 * 2
    copies = max(2, math.ceil(2 * L2_BYTES / one))
    kk = torch.from_numpy(np.ascontiguousarray(ks[:, :n].transpose(0, 2, 1, 3))).to(device)
    vv = torch.from_numpy(np.ascontiguousarray(vs[:, :n].transpose(0, 2, 1, 3))).to(device)
    kc = [kk] + [kk.clone() for _ in range(copies - 1)]
    vc = [vv] + [vv.clone() for _ in range(copies - 1)]
    lens = torch.full((wl.batch,), n, dtype=torch.int32, device=device)
    qd = torch.from_numpy(q[0]).to(device)
    out = torch.empty_like(qd)
    ws = None
    with torch.cuda.stream(stream):
        for i in range(4):
            out = kvq.decode_fp16(kc[i % copies], vc[i % copies], lens, qd, out=out, stream=stream)
        nb = __import__("ctypes").c_size_t()
        kvq.kvq_fp16_workspace_bytes(wl.batch, wl.hq, wl.hkv, wl.d, __import__("ctypes").byref(nb))
        ws = torch.zeros(nb.value, dtype=torch.uint8, device=device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(iters):
            kvq.decode_fp16(kc[i % copies], vc[i % copies], lens, qd, out=out, workspace=ws,
                            stream=stream)
        e1.record(stream)
    e1.synchronize()
    us = e0.elapsed_time(e1) / iters * 1e3
    byts = wl.batch * wl.hkv * n * wl.d * 4 + wl.batch * wl.hq * wl.d * 2
    return {"kernel": "kvq_decode_fp16 (f16_decode_kernel<128,packed> + combine)",
            "context": n, "bytes_per_launch": byts, "avg_launch_us": round(us, 3),
            "achieved_gbs": round(byts / us / 1e3, 1), "launches": iters, "copies": copies}


def decode_bytes_one_seq(n, G, d, kb, vb, hkv, hq, window=0, sink=0, akvq_delta=0):
    """Algorithmic bytes of one decode over one sequence of n tokens: every
    quantized group's block (codes + fp16 scale/min pairs; with adaptive key
    widths the 2-bit groups' smaller block), 4d bytes per fp16 token (tail
    and sink), and the fp16 queries.  Returns (bytes, quantized tokens)."""
    blk = G * d * (kb + vb) // 8 + 8 * d
    after = n - min(n, sink)                                  # tokens after the sink
    nq = G * ((after - window) // G) if after > window else 0   # quantized tokens
    if akvq_delta:
        # groups wholly before Delta or ending after n - Delta keep 4-bit keys
        blk2 = G * d * (2 + vb) // 8 + 8 * d
        wide = sum(1 for g in range(nq // G)
                   if (g + 1) * G <= akvq_delta or (g + 1) * G > n - akvq_delta)
        qbytes = wide * blk + (nq // G - wide) * blk2
    else:
        qbytes = (nq // G) * blk
    return hkv * (qbytes + (n - nq) * 4 * d) + hq * d * 2, nq


def run_long_context(stream, device, iters=100, window=0, fp16=True, sink=0, akvq_delta=0,
                     rotate=0):
    """Decode alone on the 128k-token long-context workload (batch 1, 32 q /
    8 kv heads, d 128, K2/V2, G 32): the configuration the HBM-roofline
    target is stated on.  Copies of the cache (> 3x L2 in total) are
    rotated so that every decode reads HBM; CUDA events on the launch
    stream around `iters` decodes.  The unquantized comparison kernel runs
    the same shape (fp16 K/V, two copies) when `fp16`.  `window` > 0 keeps
    that many recent tokens in fp16 beyond the partial group, `sink` > 0 the
    first tokens of the sequence (their bytes counted at 4d per
    token-head).  `akvq_delta` > 0: position-adaptive key widths on the same
    context (4-bit keys for the first and the last Delta tokens' groups,
    2-bit keys in between, 2-bit values), each group's bytes counted at its
    own width.  `rotate` = 1: the rotating cache (q rotated in, the output
    rotated back)."""
    import torch
    from asymmetric_kv_cache_b200 import inputs, kvq
    w = inputs.WORKLOADS["long_ctx"]()
    n = w.lens[0]
    kb = 4 if akvq_delta else w.k_bits
    spec = kvq.CacheSpec(kb, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                         w.batch, n, window=window, sink=sink, akvq_delta=akvq_delta,
                         rotate=rotate)
    G, d = w.group, w.head_dim
    byts, nq = decode_bytes_one_seq(n, G, d, kb, w.v_bits, w.n_kv_heads, w.n_q_heads,
                                    window=window, sink=sink, akvq_delta=akvq_delta)
    copies = max(2, math.ceil(3 * L2_BYTES / byts))
    k = torch.from_numpy(np.concatenate(w.keys)).to(device)
    v = torch.from_numpy(np.concatenate(w.values)).to(device)
    q = torch.from_numpy(np.ascontiguousarray(w.q, np.float16)).to(device)
    caches = []
    with torch.cuda.stream(stream):
        for _ in range(copies):
            c = kvq.KVQCache(spec)
            c.append(k, v, w.lens, stream=stream)
            caches.append(c)
        out = torch.empty_like(q)
        for i in range(2 * copies):
            caches[i % copies].decode(q, out=out, stream=stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(iters):
            caches[i % copies].decode(q, out=out, stream=stream)
        e1.record(stream)
    e1.synchronize()
    us = e0.elapsed_time(e1) / iters * 1e3
    for c in caches:
        if c.workspace_status(stream) != 0:
            raise RuntimeError("decode kernel reported a failed wait")
    peak, peak_kind = _peaks()
    res = {"workload": "long_ctx", "context": n, "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv",
           "bits": (f"K4 (first and last {akvq_delta} tokens) / K2 (middle) / V{w.v_bits}"
                    if akvq_delta else f"K{w.k_bits}/V{w.v_bits}"),
           "group": G, "window": window, "sink": sink, "akvq_delta": akvq_delta,
           "rotate": rotate,
           "fp16_tokens": n - nq, "copies": copies,
           "bytes_per_launch": int(byts), "avg_launch_us": round(us, 3),
           "achieved_gbs": round(byts / us / 1e3, 1), "peak": peak, "peak_kind": peak_kind,
           "frac": round(byts / us / 1e3 / peak, 4), "launches": iters,
           "kv_tokens_per_s": round(n * iters / (e0.elapsed_time(e1) / 1e3), 1),
           "note": "decode + combine per launch, CUDA events around the launches"}
    if not (window or sink or akvq_delta or rotate):
        res["traffic"] = _traffic("decode_long_ctx_traffic.json")
    del caches
    if not fp16:
        del k, v
        torch.cuda.empty_cache()
        return res
    # the unquantized kernel on the same shape
    kk = k.view(n, w.n_kv_heads, d).transpose(0, 1).unsqueeze(0).contiguous()
    vv = v.view(n, w.n_kv_heads, d).transpose(0, 1).unsqueeze(0).contiguous()
    del k, v
    kc, vc = [kk, kk.clone()], [vv, vv.clone()]
    lens = torch.full((1,), n, dtype=torch.int32, device=device)
    import ctypes
    nb = ctypes.c_size_t()
    kvq.kvq_fp16_workspace_bytes(1, w.n_q_heads, w.n_kv_heads, d, ctypes.byref(nb))
    ws = torch.zeros(nb.value, dtype=torch.uint8, device=device)
    with torch.cuda.stream(stream):
        for i in range(4):
            kvq.decode_fp16(kc[i % 2], vc[i % 2], lens, q, out=out, workspace=ws, stream=stream)
        e0.record(stream)
        for i in range(iters):
            kvq.decode_fp16(kc[i % 2], vc[i % 2], lens, q, out=out, workspace=ws, stream=stream)
        e1.record(stream)
    e1.synchronize()
    f_us = e0.elapsed_time(e1) / iters * 1e3
    f_bytes = w.n_kv_heads * n * d * 4 + w.n_q_heads * d * 2
    res["fp16_baseline"] = {"avg_launch_us": round(f_us, 3), "bytes_per_launch": int(f_bytes),
                            "achieved_gbs": round(f_bytes / f_us / 1e3, 1),
                            "quantized_decode_speedup": round(f_us / us, 3)}
    del kc, vc, kk, vv
    torch.cuda.empty_cache()
    return res


def _graph_upload(g, stream):
    """Upload an instantiated torch CUDA graph to the device on `stream`
    (cudaGraphUpload) without running it."""
    from cuda.bindings import runtime as rt
    err, = rt.cudaGraphUpload(rt.cudaGraphExec_t(init_value=g.raw_cuda_graph_exec()),
                              rt.cudaStream_t(init_value=stream.cuda_stream))
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphUpload failed: {err}")


def run_quant_append(stream, device, reps=8):
    """The quantize/append workload (4 x 32768 tokens x 8 kv heads x d 128,
    fp16 K/V, K4/V2, G 32): (i) prefill quantization of the whole batch in
    one kvq_append call, CUDA events around `reps` calls on a cache reset
    between calls (537 MB read, 134 MB written per call: larger than L2);
    (ii) 64 sequences starting empty, 256 steps appending one token to each
    (a key group flushed every 32 steps), timed eagerly (host launch
    included) and replayed from a CUDA graph."""
    import torch
    from asymmetric_kv_cache_b200 import inputs, kvq
    w = inputs.WORKLOADS["quant_append"]()
    n, B, hkv, d = w.lens[0], w.batch, w.n_kv_heads, w.head_dim
    spec = kvq.CacheSpec(w.k_bits, w.v_bits, w.group, d, hkv, hkv, B, n)
    k = torch.from_numpy(np.concatenate(w.keys)).to(device)
    v = torch.from_numpy(np.concatenate(w.values)).to(device)
    del w
    cache = kvq.KVQCache(spec, device=device)
    rd = 2 * k.numel() * 2
    wr = B * hkv * (n // 32) * (32 * d * (4 + 2) // 8 + 8 * d)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ms = []
    with torch.cuda.stream(stream):
        for r in range(reps + 2):
            cache.reset(stream)
            # keep the GPU busy while the host plans and launches the call,
            # so that the events time the kernel and not the host
            torch.cuda._sleep(2_000_000)
            e0.record(stream)
            cache.append(k, v, [n] * B, stream=stream)
            e1.record(stream)
            e1.synchronize()
            if r >= 2:
                ms.append(e0.elapsed_time(e1))
    del k, v, cache
    us = statistics.median(ms) * 1e3
    peak, peak_kind = _peaks()
    prefill = {"tokens": B * n, "kv_heads": hkv, "head_dim": d, "bits": "K4/V2", "group": 32,
               "read_bytes": rd, "write_bytes": wr, "median_us": round(us, 2), "calls": reps,
               "achieved_gbs": round((rd + wr) / us / 1e3, 1), "peak": peak,
               "peak_kind": peak_kind, "frac": round((rd + wr) / us / 1e3 / peak, 4)}
    # (ii) one-token appends to 64 sequences, 256 steps from empty
    S, steps = 64, 256
    nk, nv = inputs.append_stream(inputs.SEED_BASE + 3 + 7, S, steps, hkv, d)
    nk_dev = [torch.from_numpy(x).to(device) for x in nk]
    nv_dev = [torch.from_numpy(x).to(device) for x in nv]
    spec2 = kvq.CacheSpec(4, 2, 32, d, hkv, hkv, S, steps + 32)
    c2 = kvq.KVQCache(spec2, device=device)
    with torch.cuda.stream(stream):
        c2.reset(stream)
        for s in range(steps):                     # warm-up (launch attributes set)
            c2.append(nk_dev[s], nv_dev[s], [1] * S, stream=stream)
        c2.reset(stream)
        stream.synchronize()
        e0.record(stream)
        for s in range(steps):
            c2.append(nk_dev[s], nv_dev[s], [1] * S, stream=stream)
        e1.record(stream)
        e1.synchronize()
        eager_us = e0.elapsed_time(e1) * 1e3 / steps
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            c2.reset(stream)
            for s in range(steps):
                c2.append(nk_dev[s], nv_dev[s], [1] * S, stream=stream)
        _graph_upload(g, stream)
        g.replay()
        stream.synchronize()
        e0.record(stream)
        for _ in range(4):
            g.replay()
        e1.record(stream)
        e1.synchronize()
        graph_us = e0.elapsed_time(e1) * 1e3 / (4 * steps)
    c2.sync_lengths(stream)
    if c2.lengths(S) != [steps] * S:
        raise RuntimeError("append stream: unexpected lengths after the replays")
    del g, c2
    torch.cuda.empty_cache()
    return {"workload": "quant_append", "prefill": prefill,
            "append_stream": {"sequences": S, "steps": steps, "flush_every": 32,
                              "eager_us_per_step": round(eager_us, 2),
                              "graph_us_per_step": round(graph_us, 2),
                              "note": "one kvq_append per step (one token per sequence), "
                                      "CUDA events; graph: 256 steps + reset per replay"}}


def run_concurrent_70b(stream, device, iters=100):
    """Decode alone on the 70B-shaped high-concurrency batch (64 sequences,
    64 q / 8 kv heads, d 128, contexts ~ U{1024..8192}, K4/V2, G 64, bf16
    queries), two cache copies alternated (each larger than L2)."""
    import torch
    from asymmetric_kv_cache_b200 import inputs, kvq
    w = inputs.WORKLOADS["llama70b_conc"]()
    G, d = w.group, w.head_dim
    blk = G * d * (w.k_bits + w.v_bits) // 8 + 8 * d
    byts = sum(w.n_kv_heads * ((L // G) * blk + (L % G) * 4 * d) for L in w.lens)
    byts += w.batch * w.n_q_heads * d * 2
    spec = kvq.CacheSpec(w.k_bits, w.v_bits, G, d, w.n_q_heads, w.n_kv_heads, w.batch,
                         max(w.lens))
    k = torch.from_numpy(np.concatenate(w.keys)).to(device)
    v = torch.from_numpy(np.concatenate(w.values)).to(device)
    q = torch.from_numpy(w.q_bits.view(np.int16)).to(device).view(torch.bfloat16)
    copies = max(2, math.ceil(2 * L2_BYTES / byts))
    caches = []
    with torch.cuda.stream(stream):
        for _ in range(copies):
            c = kvq.KVQCache(spec, device=device)
            c.append(k, v, w.lens, stream=stream)
            caches.append(c)
        del k, v
        out = torch.empty(q.shape, dtype=torch.float16, device=device)
        for i in range(2 * copies):
            caches[i % copies].decode(q, out=out, stream=stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(iters):
            caches[i % copies].decode(q, out=out, stream=stream)
        e1.record(stream)
    e1.synchronize()
    us = e0.elapsed_time(e1) / iters * 1e3
    for c in caches:
        if c.workspace_status(stream) != 0:
            raise RuntimeError("decode kernel reported a failed wait")
    del caches
    torch.cuda.empty_cache()
    peak, peak_kind = _peaks()
    return {"workload": "llama70b_conc", "batch": w.batch, "context_sum": int(sum(w.lens)),
            "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv", "bits": f"K{w.k_bits}/V{w.v_bits}",
            "group": G, "q_dtype": "bf16", "copies": copies, "bytes_per_launch": int(byts),
            "avg_launch_us": round(us, 3), "achieved_gbs": round(byts / us / 1e3, 1),
            "peak": peak, "peak_kind": peak_kind, "frac": round(byts / us / 1e3 / peak, 4),
            "launches": iters,
            "kv_tokens_per_s": round(sum(w.lens) * iters / (e0.elapsed_time(e1) / 1e3), 1),
            "note": "decode (+ combine when launched) per call, CUDA events around the calls"}


def run_e2e(args, wl, caches, nk, nv, q, stream, device):
    """Same metric through the C ABI with host buffers: per step, pinned host
    -> device copies of the new token and the query, append, decode, and the
    output back to pinned host memory, all inside the timed region.  As a
    serving loop would, the steps are captured once into a CUDA graph and
    the copies are double-buffered on two more streams: step s+1's inputs
    travel while step s computes, and step s's output travels back while
    step s+1 computes (events order every buffer's reuse)."""
    import torch
    steps = wl.e2e_steps
    pool = q.shape[0]
    hk = [torch.from_numpy(x).pin_memory() for x in nk]
    hv = [torch.from_numpy(x).pin_memory() for x in nv]
    hq = [torch.from_numpy(x).pin_memory() for x in q]
    dk = [torch.empty_like(hk[0], device=device) for _ in range(2)]
    dv = [torch.empty_like(hv[0], device=device) for _ in range(2)]
    dq = [torch.empty_like(hq[0], device=device) for _ in range(2)]
    dout = [torch.empty((wl.batch, wl.hq, wl.d), dtype=torch.float16, device=device)
            for _ in range(2)]
    hout = [torch.empty((wl.batch, wl.hq, wl.d), dtype=torch.float16).pin_memory()
            for _ in range(2)]
    hs = torch.cuda.Stream(device=device)   # host -> device copies
    ds = torch.cuda.Stream(device=device)   # device -> host copies
    ev_in = [torch.cuda.Event() for _ in range(steps)]     # inputs of step s on the device
    ev_done = [torch.cuda.Event() for _ in range(steps)]   # step s computed
    ev_out = [torch.cuda.Event() for _ in range(steps)]    # output of step s on the host
    fork, jh, jd = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()

    def h2d(s):
        j = s % 2
        with torch.cuda.stream(hs):
            if s >= 2:
                hs.wait_event(ev_done[s - 2])   # step s-2 has read buffer j
            dk[j].copy_(hk[s % pool], non_blocking=True)
            dv[j].copy_(hv[s % pool], non_blocking=True)
            dq[j].copy_(hq[s % pool], non_blocking=True)
            ev_in[s].record(hs)

    for cache in caches:
        cache.sync_lengths(stream)
    lens0 = [cache.lengths(wl.batch)[0] for cache in caches]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fork.record(stream)
        hs.wait_event(fork)
        ds.wait_event(fork)
        h2d(0)
        for s in range(steps):
            j, c = s % 2, s % wl.C
            if s + 1 < steps:
                h2d(s + 1)                          # travels while step s computes
            stream.wait_event(ev_in[s])
            if s >= 2:
                stream.wait_event(ev_out[s - 2])    # dout[j] of step s-2 has left
            caches[c].append(dk[j], dv[j], [1] * wl.batch, stream=stream)
            caches[c].decode(dq[j], out=dout[j], stream=stream)
            ev_done[s].record(stream)
            with torch.cuda.stream(ds):
                ds.wait_event(ev_done[s])
                hout[j].copy_(dout[j], non_blocking=True)
                ev_out[s].record(ds)
        jh.record(hs)
        jd.record(ds)
        stream.wait_event(jh)
        stream.wait_event(jd)
    for cache in caches:          # capture advanced the host mirrors only
        cache.sync_lengths(stream)
    kv = 0
    for s in range(steps):
        c = s % wl.C
        lens0[c] += 1
        kv += lens0[c] * wl.batch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    for cache in caches:
        cache.sync_lengths(stream)
    del g
    h2d = hk[0].numel() * 2 + hv[0].numel() * 2 + hq[0].numel() * 2
    return {"value": kv / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": hout[0].numel() * 2, "steps": steps,
            "mode": "CUDA graph; host<->device copies double-buffered on copy streams"}


def _traffic(record="decode_traffic.json"):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current decode kernel source; else None."""
    path = os.path.join(ROOT, "profiles", record)
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_sha256_16") != decode_source_hash():
        return None
    return rec.get("dram_bytes_per_launch_full_workload")


# the sources of the timed decode kernel (the record of its DRAM traffic is
# valid only for these bytes)
DECODE_SOURCES = ("kvq_decode.cu", "kvq_decode_kernels.cuh", "kvq_decode_d128_g32_v2.cu",
                  "kvq_split.h", "kvq_device.cuh", "kvq_internal.h")


def decode_source_hash(root=None) -> str:
    """Hash of the decode sources with their comments and blank lines taken
    out (a comment edit does not change the kernel the record was taken on)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(root or ROOT, "asymmetric_kv_cache_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        text = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(text.encode())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# CPU oracle arm
# ---------------------------------------------------------------------------
def _oracle_unit_inputs():
    """One (sequence, kv head) unit of the llama3_8b layer at its mean context:
    4113 tokens of one kv head and the 4 query heads that read it."""
    from asymmetric_kv_cache_b200 import inputs
    rng = np.random.default_rng(inputs.SEED_BASE + 1)
    n = 4096 + 17
    k = inputs.keys_channel_outliers(rng, n, 1, 128).astype(np.float16)
    v = inputs.values_token_norms(rng, n, 1, 128).astype(np.float16)
    q = rng.standard_normal((4, 128)).astype(np.float16).astype(np.float32)
    return k, v, q


def oracle_unit(k, v, q, tokens):
    """The oracle as it stands on the first `tokens` tokens of one unit:
    quantize, dequantize and fp64 attention (returns KV tokens processed)."""
    from oracle import kvq_oracle as o
    cfg = o.Config(4, 2, 32, 128, 4, 1)
    o.decode(cfg, k[:tokens], v[:tokens], q)
    return tokens


def cpu_oracle(budget_s: float):
    """cpu_baseline: the oracle on whole units of the workload, one thread,
    until budget_s seconds have passed.  A unit is 1/8 of a sequence (one kv
    head, all its query heads), so one KV token of the unit is 1/8 of a
    layer KV token; the rate is reported in layer KV tokens/s."""
    from threadpoolctl import threadpool_limits
    k, v, q = _oracle_unit_inputs()
    n = k.shape[0]
    done = 0
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        while True:
            oracle_unit(k, v, q, n)
            done += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
    return {"value": done * n / 8 / el, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} (sequence, kv-head) units of the llama3_8b layer at context {n} "
                      f"(quantize + dequantize + fp64 attention of 4 query heads), "
                      f"1 thread, {el:.1f} s"}


def _oracle_worker(budget_s: float, t_start: float):
    """One process of the all-cores CPU baseline: waits until wall time
    t_start (so that every process runs at the same time), then whole oracle
    units, one thread, until budget_s seconds have passed; returns (units,
    start, end, tokens per unit)."""
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    from threadpoolctl import threadpool_limits
    k, v, q = _oracle_unit_inputs()
    n = k.shape[0]
    done = 0
    with threadpool_limits(limits=1):
        while time.time() < t_start:
            time.sleep(0.01)
        t0 = time.time()
        while True:
            oracle_unit(k, v, q, n)
            done += 1
            if time.time() - t0 >= budget_s:
                break
    return done, t0, time.time(), n


def cpu_oracle_all_cores(budget_s: float):
    """The same oracle units on every host core this process may use (its
    CPU affinity, up to 64): one single-threaded process per core (a spawn
    pool, safe after CUDA is initialised), all started at one common wall
    time; the rate is all units over the window from the first start to the
    last end."""
    import multiprocessing as mp
    cores = max(1, min(len(os.sched_getaffinity(0)), 64))   # bounded memory and start-up
    ctx = mp.get_context("spawn")
    t_start = time.time() + 20.0 + 0.25 * cores             # after every worker has started
    with ctx.Pool(processes=cores) as pool:
        # bounded: a pool whose workers cannot start would otherwise wait forever
        res = pool.starmap_async(_oracle_worker, [(budget_s, t_start)] * cores).get(
            timeout=budget_s + 300)
    units = sum(r[0] for r in res)
    n = res[0][3]
    window = max(r[2] for r in res) - min(r[1] for r in res)
    return {"value": units * n / 8 / window, "unit": UNIT, "cores": cores,
            "sample": f"{units} (sequence, kv-head) units at context {n} over {cores} "
                      f"single-threaded processes started together, {window:.1f} s window"}


def reference_arm(args):
    """--impl reference: W warm-up and K timed steps of the oracle; each step
    is a bounded sample of the workload (one unit, its context cut to fit the
    whole run into about two minutes)."""
    from threadpoolctl import threadpool_limits
    k, v, q = _oracle_unit_inputs()
    n = k.shape[0]
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        oracle_unit(k, v, q, n)
        t_unit = time.perf_counter() - t0
        budget = 120.0
        tokens = n
        if (args.steps + args.warmup) * t_unit > budget:
            frac = budget / ((args.steps + args.warmup) * t_unit)
            tokens = max(32, int(n * frac) // 32 * 32)
        for _ in range(args.warmup):
            oracle_unit(k, v, q, tokens)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_unit(k, v, q, tokens)
        el = time.perf_counter() - t0
    value = args.steps * tokens / 8 / el
    sample = (f"each step: one (sequence, kv-head) unit of the llama3_8b layer, first {tokens} "
              f"of {n} tokens (quantize + dequantize + fp64 attention of 4 query heads), 1 thread")
    return value, el * 1e3 / args.steps, sample


def config_dict(wl, extra=None):
    d = {"workload": "llama3_8b_layer_decode", "batch": wl.batch, "n_q_heads": wl.hq,
         "n_kv_heads": wl.hkv, "head_dim": wl.d, "k_bits": wl.kb, "v_bits": wl.vb,
         "group": wl.G, "context_mean": wl.center,
         "step": "append 1 token per sequence (flush when a tail fills) + decode",
         "copies": wl.C,
         "l2": f"inputs larger than L2: {wl.C} cache copies rotated "
               f"({wl.C * wl.algorithmic_bytes([wl.center] * wl.batch) / 1e9:.2f} GB)",
         "parallelism": "replicas per GPU (weak scaling)"}
    if extra:
        d.update(extra)
    return d


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama3_8b",
                    choices=["llama3_8b", "long_ctx", "quant_append", "llama70b_conc"],
                    help="llama3_8b (the step, default), or one leg alone: long_ctx (decode "
                         "on the 128k context), quant_append (prefill + append stream), "
                         "llama70b_conc (decode on the 64-sequence ragged batch)")
    ap.add_argument("--copies", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=512)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--cpu-all-cores", type=int, default=1,
                    help="also time the oracle on every host core (0: one thread only)")
    ap.add_argument("--long-context", type=int, default=1,
                    help="also time decode alone on the 128k-token workload (0: skip)")
    ap.add_argument("--window", type=int, default=128,
                    help="recent fp16 window of the extra 128k-token decode leg (0: skip it)")
    ap.add_argument("--sink", type=int, default=32,
                    help="fp16 sink window of one more 128k-token leg, with --window (0: skip it)")
    ap.add_argument("--akvq-delta", type=int, default=1024,
                    help="Delta of one more 128k-token leg with position-adaptive key widths "
                         "(0: skip it)")
    ap.add_argument("--rotate", type=int, default=1,
                    help="one more 128k-token leg on the rotating cache (0: skip it)")
    ap.add_argument("--other-legs", type=int, default=1,
                    help="also time the quantize/append workload and the 70B-shaped batch "
                         "(0: skip)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        wl = Workload(args, 0)
        value, ms, sample = reference_arm(args)
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": config_dict(wl, {"l2": "n/a (CPU oracle)"}),
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device(device))
    if args.workload in ("quant_append", "llama70b_conc"):
        if rank == 0:
            stream = torch.cuda.Stream(device=device)
            if args.workload == "quant_append":
                out = {"metric": METRIC, "quant_append": run_quant_append(stream, device)}
            else:
                out = {"metric": METRIC,
                       "concurrent_70b_decode": run_concurrent_70b(stream, device,
                                                                   iters=max(1, args.steps))}
            print(json.dumps(out))
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()
        return 0
    if args.workload == "long_ctx":
        # decode alone on the 128k-token workload (the long-context leg of
        # the default run on its own, `--steps` timed launches)
        if rank == 0:
            stream = torch.cuda.Stream(device=device)
            lc = run_long_context(stream, device, iters=max(1, args.steps))
            out = {"metric": METRIC, "workload": "long_ctx", "long_context_decode": lc}
            if args.window:
                out["recent_window_decode"] = run_long_context(
                    stream, device, iters=max(1, args.steps), window=args.window, fp16=False)
            if args.sink:
                out["sink_window_decode"] = run_long_context(
                    stream, device, iters=max(1, args.steps), window=args.window, fp16=False,
                    sink=args.sink)
            if args.akvq_delta:
                out["akvq_decode"] = run_long_context(
                    stream, device, iters=max(1, args.steps), fp16=False,
                    akvq_delta=args.akvq_delta)
            if args.rotate:
                out["rotated_decode"] = run_long_context(
                    stream, device, iters=max(1, args.steps), fp16=False, rotate=1)
            print(json.dumps(out))
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()
        return 0
    res = run_ours(args, rank, world, device)
    wl = res["wl"]
    cb = cpu_oracle(args.cpu_budget) if (rank == 0 and world == 1) else None
    cb_all = (cpu_oracle_all_cores(args.cpu_budget)
              if (cb is not None and args.cpu_all_cores) else None)
    if rank == 0:
        line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "fp16", "data": "synthetic", "config": config_dict(wl),
                "e2e": res["e2e"], "roofline": res["roofline"], "cpu_baseline": cb,
                "clocks": res["clocks"], "gpu_launches": res["gpu_launches"],
                "kv_tokens_per_step": res["kv_tokens_per_step"]}
        fp16 = res["fp16"]
        if fp16 and res["roofline"]:
            fp16["quantized_decode_speedup"] = round(
                fp16["avg_launch_us"] / res["roofline"]["avg_launch_us"], 3)
        line["fp16_baseline"] = fp16
        if res["long_ctx"]:
            line["long_context_decode"] = res["long_ctx"]
        if res["window"]:
            line["recent_window_decode"] = res["window"]
        if res["sink"]:
            line["sink_window_decode"] = res["sink"]
        if res["akvq"]:
            line["akvq_decode"] = res["akvq"]
        if res["rot"]:
            line["rotated_decode"] = res["rot"]
        if res.get("quant_append"):
            line["quant_append"] = res["quant_append"]
        if res.get("conc70b"):
            line["concurrent_70b_decode"] = res["conc70b"]
        if cb_all is not None:
            line["cpu_baseline_all_cores"] = cb_all
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as tdist
        tdist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
