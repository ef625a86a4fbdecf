// The split of the decode work over CTAs and the merge of split units: the
// index arithmetic shared by the decode kernels, the host launch planning
// and the host-side model that checks it (tests/test_host_split_logic.py).
//
// Work is a row of slots per unit (its key groups, then one slot for the
// fp16 tail and sink); the units' rows, sequence by sequence, form one
// sequence of T slots that is cut into `grid` equal ranges, one per CTA
// (stream-K).  A CTA holds at most two pieces of split units, its first and
// its last; they write partial slots 2k and 2k + 1 of the workspace.
#pragma once

#include <cstdint>

#include "kvq_internal.h"

#ifdef __CUDACC__
#define KVQ_HD __host__ __device__ __forceinline__
#else
#define KVQ_HD inline
#endif

namespace kvq {

KVQ_HD int kvq_imin(int a, int b) { return a < b ? a : b; }

// CTA k's slot range [start, end).
KVQ_HD void cta_range(int k, int T, int grid, int* start, int* end) {
  *start = (int)((int64_t)k * T / grid);
  *end = (int)((int64_t)(k + 1) * T / grid);
}

// The CTA whose range holds slot s: the largest k with k T / grid <= s.
KVQ_HD int cta_of_slot(int64_t s, int T, int grid) {
  return (int)(((s + 1) * grid - 1) / T);
}

// Partial slot of a piece that starts at slot pos of CTA k's range.
KVQ_HD int piece_partial_slot(int k, int pos, int start) {
  return pos == start ? 2 * k : 2 * k + 1;
}

// Largest b in [0, n) with prefix[b] <= pos (prefix[0] = 0, increasing).
KVQ_HD int find_seq(const int32_t* prefix, int n, int pos) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid + 1] <= pos) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// The part of unit `unit` (sequence b, kv head kvh, head slice `slice`)
// that a CTA processes: slots [slot0, slot1) of the unit's wb slots.
struct Piece {
  int b, L, ng, Tb, wb, slot0, slot1, kvh, slice, unit, hbase, nh;
};

// Built from the slot position alone, so that it can be rebuilt after the
// group loop instead of holding registers through it.
// (G: the group size when the caller knows it at compile time - a shift
// instead of a division on the path to the piece's first copies - else 0;
// WIN: the cache has a recent and/or sink window)
template <int G = 0, bool WIN = false>
KVQ_HD Piece make_piece(const Geom& g, const int32_t* prefix, const int32_t* slen, int n_seq,
                        int pos, int end) {
  Piece p;
  p.b = find_seq(prefix, n_seq, pos);
  p.L = slen[p.b];
  if (WIN) {
    // the first min(L, sink) tokens stay in fp16; groups after them leave
    // the newest `window` tokens in fp16; the sink and the tail share the
    // unit's last (fp16) slot, Tb counts the tail alone
    const int Sb = kvq_imin(p.L, g.sink);
    const int Lq = p.L - Sb - g.window;
    p.ng = Lq <= 0 ? 0 : G ? Lq / G : Lq / g.G;
    p.Tb = p.L - Sb - p.ng * (G ? G : g.G);
    p.wb = p.ng + (p.L > p.ng * (G ? G : g.G) ? 1 : 0);
  } else {
    p.ng = G ? p.L / G : p.L / g.G;
    p.Tb = p.L - p.ng * (G ? G : g.G);
    p.wb = p.ng + (p.Tb ? 1 : 0);
  }
  const int local = pos - prefix[p.b];
  const int uis = local / p.wb;
  p.slot0 = local - uis * p.wb;
  p.slot1 = kvq_imin(p.wb, p.slot0 + (end - pos));
  p.kvh = g.slices == 1 ? uis : uis / g.slices;
  p.slice = uis - p.kvh * g.slices;
  p.unit = p.b * (g.hkv * g.slices) + uis;
  p.hbase = p.kvh * g.gqa + p.slice * kHeadsPerSlice;
  p.nh = kvq_imin(kHeadsPerSlice, g.gqa - p.slice * kHeadsPerSlice);
  return p;
}

// How the pieces of a split unit are found for the merge: the unit's first
// slot p0 lies in CTA kf (partial slot 2 kf if the unit starts that CTA's
// range, else 2 kf + 1); pieces 1 .. npc-1 are the first pieces of CTAs
// kf + 1 .. kf + npc - 1 (partial slots 2 (kf + pc)).  The split record a
// unit's first piece writes is {first partial slot, npc}.
struct MergePlan {
  int kf, npc, s0;
};

KVQ_HD MergePlan merge_plan(int64_t p0, int wb, int T, int grid) {
  MergePlan m;
  m.kf = cta_of_slot(p0, T, grid);
  const int kl = cta_of_slot(p0 + wb - 1, T, grid);
  m.npc = kl - m.kf + 1;
  m.s0 = ((int64_t)m.kf * T / grid == p0) ? 2 * m.kf : 2 * m.kf + 1;
  return m;
}

KVQ_HD int merge_piece_slot(int kf, int s0, int pc) { return pc == 0 ? s0 : 2 * (kf + pc); }

// ---- host launch planning ------------------------------------------------
#ifndef __CUDA_ARCH__
// Decode grid: one CTA per resident slot up to the cap.  When every
// sequence has the same number of slots and the units fit the cap, a
// multiple of the unit count (if it keeps >= 80% of the cap) makes every
// CTA range end on a unit boundary: one piece per CTA, no CTA pays a
// second prologue and merge.
inline int64_t choose_grid(const Geom& g, const int32_t* lens, int n_seq, int64_t slots,
                           int cap) {
  int64_t grid = slots < cap ? slots : cap;
  const int64_t units = (int64_t)n_seq * g.hkv * g.slices;
  const int w0 = unit_slots_s(lens[0], g.G, g.window, g.sink);
  bool equal = true;
  for (int b = 1; b < n_seq && equal; ++b)
    equal = unit_slots_s(lens[b], g.G, g.window, g.sink) == w0;
  if (equal && units <= cap) {
    int64_t alt = units * (cap / units);
    if (alt > slots) alt = slots;
    if (alt * 5 >= (int64_t)cap * 4) grid = alt;
  }
  return grid;
}

// Split units are merged by their last CTA (no combine kernel) for wide
// CTAs (one unit piece each) with up to 32 expected pieces per unit;
// otherwise the combine kernel runs (a narrow CTA moves on to its next
// piece, which an in-kernel merge would delay).
inline bool use_inline_merge(bool wide, int64_t grid, int64_t units) {
  return wide && (grid / units + 1) <= 32;
}
#endif

}  // namespace kvq

#undef KVQ_HD
