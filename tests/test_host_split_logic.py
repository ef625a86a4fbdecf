"""The decode's split and merge index arithmetic, checked on the host.

The decode cuts the slots of all units (sequence, kv head, head slice) into
`grid` equal ranges, one per CTA; a CTA writes a partial result for each
piece of a unit that it does not hold whole, into partial slot 2k (its
first piece) or 2k + 1 (its last), and the split record of the unit (first
partial slot, number of CTAs spanned).  A split unit is merged either by
the combine kernel (from the record) or by the last CTA to finish (an
acquire-release ticket: every CTA in the unit's span counts once, and the
merge reads the pieces at merge_piece_slot).  All of this index arithmetic
lives in csrc/kvq_split.h, shared by the kernels and the host planner; a
C++ program compiled here with g++ runs it CTA by CTA, without a GPU, over
ragged and equal batches, windows, sinks, head slices and grids (the
planner's choices, the no-alloc entry point's reduced grids and arbitrary
grids up to 1024, more CTAs than slots included), and checks that:

* every partial slot written or read is below 2 * grid (the workspace, and
  the no-alloc scratch, hold two per CTA) and is written at most once;
* a CTA holds at most two split pieces, the first and the last of its range;
* every split unit's record equals the merge plan, the plan's pieces are
  exactly the slots its pieces (and the empty CTAs in its span) wrote, and
  the number of CTAs that count on its ticket equals the plan's piece count;
* the pieces of every unit cover its slots exactly once;
* the planner's grid never exceeds the slot count, and an in-kernel merge of
  more than 32 pieces fits its shared-memory scratch.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SRC = r"""
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>
#include "kvq_split.h"
using namespace kvq;

static long fails = 0, checks = 0;
#define REQ(c, ...) do { ++checks; if (!(c)) { if (fails++ < 20) { std::printf("FAIL line %d: ", __LINE__); std::printf(__VA_ARGS__); std::printf("\n"); } } } while (0)

// shared-memory bytes of the wide decode ring for a block size (the same
// rule as the kernels' configuration: 16 warps up to 4 KB blocks, 12 up to
// 7.5 KB, 8 above; two stages per warp)
static int ring_bytes(int blk) {
  const int nw = blk <= 4096 ? 16 : blk <= 7680 ? 12 : 8;
  return nw * 2 * blk;
}

static void run(const Geom& g, const std::vector<int32_t>& lens, int grid, bool inl, int blk) {
  const int n = (int)lens.size();
  const bool win = g.window > 0 || g.sink > 0;
  std::vector<int32_t> prefix(n + 1, 0);
  const int per = g.hkv * g.slices;
  for (int b = 0; b < n; ++b)
    prefix[b + 1] = prefix[b] + per * unit_slots_s(lens[b], g.G, g.window, g.sink);
  const int T = prefix[n];
  if (T == 0) return;
  const int units = n * per;
  std::vector<long> written(2 * grid, -2);     // -2 nothing; -1 empty piece; else unit
  std::vector<int> rec_first(units, -1), rec_cnt(units, -1), split_pieces(units, 0);
  std::vector<int> tickets(units, 0), covered(units, 0);
  for (int k = 0; k < grid; ++k) {
    int start, end;
    cta_range(k, T, grid, &start, &end);
    REQ(start <= end && end <= T, "range k %d", k);
    if (start == end) {
      REQ(written[2 * k] == -2, "double write %d", 2 * k);
      written[2 * k] = -1;
      if (start < T) {
        const Piece p = win ? make_piece<0, true>(g, prefix.data(), lens.data(), n, start, start + 1)
                            : make_piece<0, false>(g, prefix.data(), lens.data(), n, start, start + 1);
        if (p.slot0 > 0) tickets[p.unit]++;
      }
      continue;
    }
    int nsplit = 0;
    for (int pos = start; pos < end;) {
      const Piece p = win ? make_piece<0, true>(g, prefix.data(), lens.data(), n, pos, end)
                          : make_piece<0, false>(g, prefix.data(), lens.data(), n, pos, end);
      REQ(p.b >= 0 && p.b < n && p.unit >= 0 && p.unit < units, "piece b %d unit %d", p.b, p.unit);
      REQ(p.wb > 0 && p.slot0 >= 0 && p.slot0 < p.slot1 && p.slot1 <= p.wb, "slots");
      REQ(prefix[p.b] + (p.unit - p.b * per) * p.wb + p.slot0 == pos, "position");
      REQ(p.nh >= 1 && p.nh <= kHeadsPerSlice && p.hbase + p.nh <= (p.kvh + 1) * g.gqa, "heads");
      covered[p.unit] += p.slot1 - p.slot0;
      const bool whole = p.slot0 == 0 && p.slot1 == p.wb;
      const int ms = piece_partial_slot(k, pos, start);
      if (!whole) {
        ++nsplit;
        REQ(pos == start || pos + (p.slot1 - p.slot0) == end, "split piece inside a range");
        REQ(ms < 2 * grid && written[ms] == -2, "partial slot %d", ms);
        written[ms] = p.unit;
        split_pieces[p.unit]++;
        tickets[p.unit]++;
      }
      if (p.slot0 == 0) {
        rec_first[p.unit] = ms;
        rec_cnt[p.unit] = cta_of_slot((long long)pos + p.wb - 1, T, grid) - k + 1;
      }
      pos += p.slot1 - p.slot0;
    }
    REQ(nsplit <= 2, "%d split pieces in CTA %d", nsplit, k);
  }
  for (int u = 0; u < units; ++u) {
    const int b = u / per, uis = u % per;
    const int wb = unit_slots_s(lens[b], g.G, g.window, g.sink);
    if (wb == 0) continue;
    REQ(covered[u] == wb, "unit %d covered %d of %d", u, covered[u], wb);
    const long long p0 = prefix[b] + (long long)uis * wb;
    const MergePlan mp = merge_plan(p0, wb, T, grid);
    REQ(rec_cnt[u] == mp.npc, "record count %d plan %d", rec_cnt[u], mp.npc);
    if (split_pieces[u] == 0) {
      REQ(mp.npc == 1, "whole unit with %d pieces", mp.npc);
      continue;
    }
    REQ(rec_first[u] == mp.s0, "record first %d plan %d", rec_first[u], mp.s0);
    REQ(tickets[u] == mp.npc, "unit %d: %d ticket counts, plan %d", u, tickets[u], mp.npc);
    int got = 0;
    for (int pc = 0; pc < mp.npc; ++pc) {
      const int s = merge_piece_slot(mp.kf, mp.s0, pc);
      REQ(s >= 0 && s < 2 * grid, "merge slot %d grid %d", s, grid);
      if (s < 0 || s >= 2 * grid) continue;
      REQ(written[s] == u || written[s] == -1, "merge slot %d holds %ld, unit %d", s, written[s], u);
      if (written[s] == u) ++got;
    }
    REQ(got == split_pieces[u], "unit %d: plan reads %d of %d pieces", u, got, split_pieces[u]);
    if (inl && mp.npc > 32) REQ(3 * kHeadsPerSlice * mp.npc * 4 <= ring_bytes(blk), "merge scratch");
  }
}

int main() {
  std::mt19937 rng(1234);
  const int Gs[2] = {32, 64};
  const int wins[3] = {0, 16, 128};
  const int sinks[3] = {0, 5, 32};
  const int hkvs[3] = {1, 2, 8};
  const int gqas[3] = {1, 4, 16};
  long shapes = 0, planned = 0;
  for (int gi = 0; gi < 2; ++gi)
  for (int wi = 0; wi < 3; ++wi)
  for (int si = 0; si < 3; ++si)
  for (int hi = 0; hi < 3; ++hi)
  for (int qi = 0; qi < 3; ++qi) {
    Geom g{};
    g.G = Gs[gi]; g.window = wins[wi]; g.sink = sinks[si];
    g.hkv = hkvs[hi]; g.gqa = gqas[qi]; g.hq = g.hkv * g.gqa;
    g.slices = (g.gqa + kHeadsPerSlice - 1) / kHeadsPerSlice;
    const int blk = g.G * 128 * 6 / 8 + 8 * 128;
    for (int trial = 0; trial < 14; ++trial) {
      int n;
      std::vector<int32_t> lens;
      if (trial < 4) {                         // equal lengths
        n = 1 + (int)(rng() % 40);
        const int L = 1 + (int)(rng() % 5000);
        lens.assign(n, L);
      } else {                                 // ragged, some tiny
        n = 1 + (int)(rng() % 70);
        for (int b = 0; b < n; ++b)
          lens.push_back(rng() % 4 == 0 ? 1 + (int)(rng() % 40) : 1 + (int)(rng() % 9000));
      }
      int64_t slots = 0;
      for (int b = 0; b < n; ++b) slots += (int64_t)g.hkv * g.slices * unit_slots_s(lens[b], g.G, g.window, g.sink);
      for (int cap : {148, 296, 592, 1024, 7, 64}) {     // wide / narrow caps and env caps
        const int64_t grid = choose_grid(g, lens.data(), n, slots, cap);
        REQ(grid >= 1 && grid <= slots && grid <= cap, "planner grid %lld", (long long)grid);
        const int64_t units = (int64_t)n * g.hkv * g.slices;
        const bool wide = units <= 148;
        run(g, lens, (int)grid, use_inline_merge(wide, grid, units), blk);
        for (int mg : {1, 5, 33, 500}) {       // reduced grids (the no-alloc entry point)
          const int64_t gr = grid < mg ? grid : mg;
          run(g, lens, (int)gr, use_inline_merge(wide, gr, units), blk);
        }
        ++planned;
      }
      for (int extra = 0; extra < 3; ++extra) {  // arbitrary grids, more CTAs than slots too
        const int grid = 1 + (int)(rng() % 1024);
        run(g, lens, grid, true, blk);
      }
      ++shapes;
    }
  }
  std::printf("shapes %ld planned %ld checks %ld fails %ld\n", shapes, planned, checks, fails);
  return fails ? 1 : 0;
}
"""


def _cuda_include():
    for cand in ("/usr/local/cuda/include", os.path.join(os.environ.get("CUDA_HOME", ""), "include")):
        if cand and os.path.exists(os.path.join(cand, "cuda_runtime.h")):
            return cand
    return None


def test_split_and_merge_indices(tmp_path):
    gxx = shutil.which("g++")
    inc = _cuda_include()
    if not gxx or not inc:
        pytest.skip("g++ or the CUDA headers are not available")
    src = tmp_path / "split.cpp"
    src.write_text(SRC)
    exe = tmp_path / "split"
    subprocess.run([gxx, "-std=c++17", "-O2", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "asymmetric_kv_cache_b200", "csrc"), "-I", inc,
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    print(res.stdout)
    assert res.returncode == 0, res.stdout
    assert "fails 0" in res.stdout
