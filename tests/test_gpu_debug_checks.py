"""The range-checked build (libkvq_debug.so, -DKVQ_DEBUG) on the full-size
workloads.  In that build every cache, workspace, query and output index of
the decode kernels is checked before its access; a failed check records
KVQ_ERR_DEVICE and the check's number in the workspace error word and skips
the access.  Here the benchmark workloads at full size, a ragged batch that
takes the combine kernel, the window and sink options, several split counts
and the no-alloc entry point run through that build (in a child process with
KVQ_LIBRARY=debug); every call must leave the error word at zero and the
outputs must still match the oracle."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, ROOT)
import numpy as np, torch
from asymmetric_kv_cache_b200 import inputs, kvq
from tests import kvq_testlib as tl
assert kvq.LIB_PATH.endswith("libkvq_debug.so"), kvq.LIB_PATH
res = {}

def run(name, w, window=0, sink=0, caps=(None,), noalloc=False, oracle=True):
    spec = kvq.CacheSpec(w.k_bits, w.v_bits, w.group, w.head_dim, w.n_q_heads, w.n_kv_heads,
                         w.batch, max(w.lens), window=window, sink=sink)
    cache = kvq.KVQCache(spec)
    tl.append_chunks(cache, w.keys, w.values, w.kv_dtype)
    if w.q_dtype == "bf16":
        qd = torch.from_numpy(w.q_bits.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        qd = tl.to_device(w.q, w.q_dtype)
    want = None
    if oracle:
        hk = [x.astype(np.float16) for x in w.keys]
        hv = [x.astype(np.float16) for x in w.values]
        want = tl.oracle_decode(spec, hk, hv, w.q)
    errs = []
    for cap in caps:
        if cap is None:
            os.environ.pop("KVQ_DECODE_MAX_CTAS", None)
        else:
            os.environ["KVQ_DECODE_MAX_CTAS"] = str(cap)
        out = cache.decode(qd)
        torch.cuda.synchronize()
        st = cache.workspace_status()
        assert st == 0, (name, cap, kvq.kvq_last_error())
        if want is not None:
            errs.append(tl.decode_error(out, want))
    os.environ.pop("KVQ_DECODE_MAX_CTAS", None)
    if noalloc:
        out = torch.empty_like(qd, dtype=torch.float16)
        for _ in range(2):
            cache.decode_noalloc(qd, out)
        torch.cuda.synchronize()
        if want is not None:
            errs.append(tl.decode_error(out, want))
    res[name] = max(errs) if errs else 0.0

run("tiny", inputs.tiny(), caps=(None, 1, 3))
run("llama3_8b", inputs.llama3_8b(), caps=(None, 1, 7, 64, 1024), noalloc=True)
run("long_ctx", inputs.long_ctx(), caps=(None, 33))
run("llama70b_conc", inputs.llama70b_conc(), caps=(None, 100), noalloc=True)
rng = np.random.default_rng(77)
lens = [int(x) for x in rng.integers(1, 3000, size=200)]
run("ragged_200", inputs._lognormal_workload("ragged", 77, lens, 32, 8, 128, 4, 2, 32, "fp16"))
run("long_ctx_window_sink", inputs.long_ctx(n=20000), window=128, sink=32, caps=(None, 5))
run("gqa16", inputs._lognormal_workload("gqa16", 78, [700, 1500, 33], 32, 2, 64, 2, 4, 64, "bf16"))
print("RESULT " + json.dumps(res))
"""


def test_full_size_workloads_pass_every_range_check():
    env = dict(os.environ, KVQ_LIBRARY="debug")
    proc = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env,
                          capture_output=True, text=True, timeout=1500, cwd=ROOT)
    assert proc.returncode == 0, proc.stdout[-3000:] + proc.stderr[-3000:]
    line = [ln for ln in proc.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    for name, err in res.items():
        assert err <= 2e-3, (name, err)
