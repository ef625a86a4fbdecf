"""The position-adaptive widths' host and device arithmetic against the oracle.

The append kernel picks each new group's key width with akvq_key_bits and
requantizes the groups akvq_aging names; the host planner reserves the
requantization tasks from the same function (one task when fewer than G
tokens are appended).  Both live in csrc/kvq_internal.h.  A C++ program
compiled here with g++ prints them for many (n0, n1, G, Delta); they must
equal what the oracle's rule gives ("Asymmetric Key-Value Quantization: 2-Bit
Values and 4-Bit Keys under Long-Context Drift", §3.2, with the reading of
this library): the width of every group at n1, and the set of groups that
were quantized before the append (g < n0 / G), held 4-bit keys at n0 and
hold 2-bit keys at n1 - exactly the groups the oracle's replay requantizes.
The reserved task count must cover the count for every append of fewer than
G tokens.
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
using namespace kvq;
int main() {
  const int Gs[2] = {32, 64};
  for (int gi = 0; gi < 2; ++gi) {
    const int G = Gs[gi];
    for (int dm = 1; dm <= 6; ++dm) {
      const int delta = dm * G;
      for (int n0 = 0; n0 <= 14 * G; n0 += (n0 < 3 * G ? 1 : 3)) {
        const int steps[7] = {1, 2, G - 1, G, G + 5, 3 * G, 5 * G + 7};
        for (int si = 0; si < 7; ++si) {
          const int n1 = n0 + steps[si];
          int first = -1;
          const int cnt = akvq_aging(n0, n1, n0 / G, G, delta, &first);
          std::printf("A %d %d %d %d %d %d\n", G, delta, n0, n1, cnt > 0 ? first : -1, cnt);
        }
        for (int g = 0; g < n0 / G; ++g)
          std::printf("B %d %d %d %d %d\n", G, delta, n0, g, akvq_key_bits(g, n0, G, delta));
      }
    }
  }
  return 0;
}
"""


def _cuda_include():
    for cand in ("/usr/local/cuda/include", os.environ.get("CUDA_HOME", "") + "/include"):
        if cand and os.path.exists(os.path.join(cand, "cuda_runtime.h")):
            return cand
    return None


def test_widths_and_aging_match_the_oracle(tmp_path):
    gxx = shutil.which("g++")
    inc = _cuda_include()
    if not gxx or not inc:
        pytest.skip("g++ or the CUDA headers are not available")
    src = tmp_path / "akvq.cpp"
    src.write_text(SRC)
    exe = tmp_path / "akvq"
    subprocess.run([gxx, "-std=c++17", "-O2", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "asymmetric_kv_cache_b200", "csrc"), "-I", inc,
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0
    n_a = n_b = 0
    for line in res.stdout.splitlines():
        f = line.split()
        if f[0] == "B":
            G, delta, n, g, bits = map(int, f[1:])
            cfg = o.Config(4, 2, G, 128, 32, 8, akvq_delta=delta)
            assert bits == o.akvq_key_bits(cfg, g, n), line
            n_b += 1
            continue
        G, delta, n0, n1, first, cnt = map(int, f[1:])
        cfg = o.Config(4, 2, G, 128, 32, 8, akvq_delta=delta)
        want = [g for g in range(n0 // G)
                if o.akvq_key_bits(cfg, g, n0) == 4 and o.akvq_key_bits(cfg, g, n1) == 2]
        got = list(range(first, first + cnt)) if cnt > 0 else []
        assert got == want, (line, want)
        if n1 - n0 < G:
            assert cnt <= 1, line          # the one task the host reserves suffices
        n_a += 1
    assert n_a > 10000 and n_b > 10000
