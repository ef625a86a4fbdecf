"""The library's slot arithmetic for the recent and sink windows, without a GPU.

``quantized_groups`` / ``unit_slots`` and their sink-window forms
``quantized_groups_s`` / ``unit_slots_s`` (csrc/kvq_internal.h) decide, on the
host and in the kernels, how many groups of a sequence are quantized, how
many tokens stay in the fp16 tail and how many decode slots a unit has;
the append planning counts the groups an append completes from them.  A
small C++ program compiled here with g++ evaluates them over a grid of
lengths, group sizes and windows, and the results must equal the oracle's
``split_tokens`` and ``segments`` (pinned against the flush rule run token
by token).
"""
import os
import shutil
import subprocess

import pytest

from oracle import kvq_oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SRC = r"""
#include <cstdio>
#include "kvq_internal.h"
int main() {
  const int Gs[2] = {32, 64};
  const int Rs[6] = {0, 16, 32, 48, 128, 1024};
  const int Ss[4] = {0, 5, 32, 100};
  for (int gi = 0; gi < 2; ++gi)
    for (int ri = 0; ri < 6; ++ri)
      for (int si = 0; si < 4; ++si)
        for (int n = 0; n <= 1400; n += (si ? 3 : 1)) {
          const int G = Gs[gi], R = Rs[ri], S = Ss[si];
          std::printf("%d %d %d %d %d %d %d %d\n", G, R, S, n, kvq::quantized_groups(n, G, R),
                      kvq::unit_slots(n, G, R), kvq::quantized_groups_s(n, G, R, S),
                      kvq::unit_slots_s(n, G, R, S));
        }
  return 0;
}
"""


def _cuda_include():
    for cand in ("/usr/local/cuda/include", os.path.join(os.environ.get("CUDA_HOME", ""), "include")):
        if cand and os.path.exists(os.path.join(cand, "cuda_runtime.h")):
            return cand
    return None


@pytest.fixture(scope="module")
def table(tmp_path_factory):
    gxx = shutil.which("g++")
    inc = _cuda_include()
    if not gxx or not inc:
        pytest.skip("g++ or the CUDA headers are not available")
    d = tmp_path_factory.mktemp("hostlogic")
    src = d / "check.cpp"
    src.write_text(SRC)
    exe = d / "check"
    subprocess.run([gxx, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "asymmetric_kv_cache_b200", "csrc"), "-I", inc,
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return [tuple(int(x) for x in line.split()) for line in out.splitlines()]


def test_quantized_groups_and_slots_match_the_oracle_split(table):
    assert len(table) == 2 * 6 * (1401 + 3 * 467)
    for G, R, S, n, ng, slots, ngs, slots_s in table:
        N, T = o.split_tokens(n, G, R)
        assert ng * G == N, (G, R, n)
        assert slots == N // G + (1 if T else 0), (G, R, n)
        Sb, Nq, Ts = o.segments(o.Config(4, 2, G, 64, 1, 1, window=R, sink=S), n)
        assert ngs * G == Nq, (G, R, S, n)
        # one decode slot per group, one for the sink and the tail together
        assert slots_s == Nq // G + (1 if Sb + Ts else 0), (G, R, S, n)


def test_groups_completed_by_an_append(table):
    """The append planning: groups completed by appending nn tokens to a
    sequence of len0 = difference of quantized_groups; at most one for
    nn < G (so a captured one-token append keeps its launch shape)."""
    q = {(G, R, n): ng for G, R, S, n, ng, *_ in table if S == 0}
    for (G, R, n), ng in q.items():
        for nn in (1, G - 1, G, 3 * G + 5):
            if (G, R, n + nn) not in q:
                continue
            F = q[(G, R, n + nn)] - ng
            N0, _ = o.split_tokens(n, G, R)
            N1, _ = o.split_tokens(n + nn, G, R)
            assert F * G == N1 - N0
            if nn < G:
                assert F in (0, 1)
