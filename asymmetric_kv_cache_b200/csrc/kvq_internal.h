// Internal declarations shared by the host side of libkvq (kvq_abi.cpp) and
// its CUDA kernels.  Geometry only: the offsets of LAYOUT v2 (documented in
// include/kvq.h) and the launch entry points of each kernel family.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "kvq.h"

namespace kvq {

// Upper bound on decode CTAs; sizes the split-partial region of the
// workspace (two partial slots per CTA: its first and its last piece).
constexpr int kMaxDecodeCtas = 1024;
// At most this many query heads share one pass over a kv head (the M = 16
// rows of the tensor-core tile hold up to 8 heads plus their low halves).
constexpr int kHeadsPerSlice = 8;
// Sequences per append launch (per-sequence arguments travel as kernel
// parameters); longer batches are split into several launches.
constexpr int kAppendMaxSeqs = 512;
// Sequences per decode call, and per decode launch (the CTA-local slot
// prefix and lengths live in shared memory); a call with more sequences runs
// one decode + combine pair per chunk of kSeqsPerLaunch.
constexpr int kMaxSeqsDecode = 8192;
constexpr int kSeqsPerLaunch = 2048;

struct Geom {
  int32_t kb, vb, G, d, hq, hkv, gqa, J, slices;
  int32_t max_seqs, max_tokens, max_groups;
  int32_t block_bytes;
  int32_t sec_kcodes, sec_kscale, sec_kmin, sec_vcodes, sec_vscale, sec_vmin;
  int64_t lens_off, counters_off, blocks_off, tails_off, tail_bytes, total_bytes;
  int32_t window, tail_slots;   // R, and W = R + G slots of the fp16 tail ring
  int32_t sink, sink_slots;     // S, and SW = S rounded up to 16 sink slots
  int64_t sinks_off, sink_bytes;
  int32_t rotate;               // tokens, q and the output rotated by H / sqrt(d)
  // position-adaptive key bits: Delta (0 = off) and the 2-bit group block
  // inside a slot of block_bytes (codes at 0)
  int32_t akvq_delta;
  int32_t a2_bytes, a2_kscale, a2_kmin, a2_vcodes, a2_vscale, a2_vmin;
};

// Workspace of kvq_decode: [error word | per-unit split records | per-unit
// tickets | partials].  A split record is {first partial slot, number of
// pieces} of one unit; a ticket counts the unit's finished pieces when the
// last CTA to finish merges them (it resets the ticket to 0).
struct WsLayout {
  int64_t err_off, units_off, tickets_off, partials_off, total;
  int32_t units;       // split records
  int32_t slot_floats; // floats per partial slot: heads x (o[d], m, l, 2 pad)
};

inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// Groups of a sequence of L tokens that are quantized: those followed by at
// least `window` newer tokens ("[Framework] The Asymmetric Key-Value Cache
// Compression", §III and §V: the most recent tokens stay in fp16).  The
// other L - G * groups tokens are the fp16 tail.
__host__ __device__ inline int quantized_groups(int L, int G, int window) {
  const int Lq = L - window;
  return Lq > 0 ? Lq / G : 0;
}
// Decode slots of one unit: its groups plus one for a non-empty tail.
__host__ __device__ inline int unit_slots(int L, int G, int window) {
  const int ng = quantized_groups(L, G, window);
  return ng + (L > ng * G ? 1 : 0);
}
// With a sink window of S tokens: the first min(L, S) tokens stay in fp16,
// the rule above applies to the rest; the sink shares the tail's slot.
__host__ __device__ inline int quantized_groups_s(int L, int G, int window, int sink) {
  return quantized_groups(L > sink ? L - sink : 0, G, window);
}
__host__ __device__ inline int unit_slots_s(int L, int G, int window, int sink) {
  const int ng = quantized_groups_s(L, G, window, sink);
  return ng + (L > ng * G ? 1 : 0);
}

// Position-adaptive key bits ("Asymmetric Key-Value Quantization: 2-Bit
// Values and 4-Bit Keys under Long-Context Drift", §3.2, read as 4-bit keys
// for the early and the recent key groups and 2-bit keys in between): the
// key width of quantized group g (positions gG .. gG + G - 1) when the
// sequence holds n tokens.
__host__ __device__ inline int akvq_key_bits(int g, int n, int G, int delta) {
  return ((g + 1) * G <= delta || (g + 1) * G > n - delta) ? 4 : 2;
}
// The first group that is recent at length n (every group from it on has
// its last position >= n - delta).
__host__ __device__ inline int akvq_recent_start(int n, int G, int delta) {
  return n >= delta ? (n - delta) / G : 0;
}
// Groups that an append from n0 to n1 tokens moves from the recent region
// into the middle and that were quantized before it (N0 = groups quantized
// at n0): they are requantized to 2 bits.  [first, first + count).
__host__ __device__ inline int akvq_aging(int n0, int n1, int N0g, int G, int delta,
                                          int* first) {
  const int lo0 = delta / G, lo1 = akvq_recent_start(n0, G, delta);
  const int lo = lo0 > lo1 ? lo0 : lo1;
  const int hi1 = akvq_recent_start(n1, G, delta);
  const int hi = hi1 < N0g ? hi1 : N0g;
  *first = lo;
  return hi > lo ? hi - lo : 0;
}

// Fill g from a validated configuration (no checks here).
inline void make_geom(const kvq_config& c, Geom* g) {
  g->kb = c.k_bits;
  g->vb = c.v_bits;
  g->G = c.group;
  g->d = c.head_dim;
  g->hq = c.n_q_heads;
  g->hkv = c.n_kv_heads;
  g->gqa = c.n_q_heads / c.n_kv_heads;
  g->J = c.head_dim / c.group;
  g->slices = (g->gqa + kHeadsPerSlice - 1) / kHeadsPerSlice;
  g->max_seqs = c.max_seqs;
  g->max_tokens = c.max_tokens;
  g->max_groups = c.max_tokens / c.group;
  g->window = c.window;
  g->tail_slots = c.window + c.group;
  g->sink = c.sink;
  g->sink_slots = (c.sink + 15) / 16 * 16;
  g->rotate = c.rotate;
  g->akvq_delta = c.akvq_delta;
  const int G = g->G, d = g->d, J = g->J;
  {
    int o2 = G * d * 2 / 8;   // 2-bit key codes
    g->a2_kscale = o2; o2 += 2 * d;
    g->a2_kmin = o2;   o2 += 2 * d;
    g->a2_vcodes = o2; o2 += G * d * c.v_bits / 8;
    g->a2_vscale = o2; o2 += 2 * G * J;
    g->a2_vmin = o2;   o2 += 2 * G * J;
    g->a2_bytes = o2;
  }
  int off = 0;
  g->sec_kcodes = off; off += G * d * g->kb / 8;
  g->sec_kscale = off; off += 2 * d;
  g->sec_kmin = off;   off += 2 * d;
  g->sec_vcodes = off; off += G * d * g->vb / 8;
  g->sec_vscale = off; off += 2 * G * J;
  g->sec_vmin = off;   off += 2 * G * J;
  g->block_bytes = off;
  int64_t pos = 0;
  g->lens_off = pos;
  pos = align_up(pos + 4LL * c.max_seqs, 256);
  g->counters_off = pos;   // append completion tickets, one per sequence
  pos = align_up(pos + 4LL * c.max_seqs, 256);
  g->blocks_off = pos;
  pos = align_up(pos + (int64_t)c.max_seqs * c.n_kv_heads * g->max_groups * g->block_bytes, 256);
  g->tails_off = pos;
  g->tail_bytes = 4LL * g->tail_slots * d;  // K tail + V tail, fp16
  pos = align_up(pos + (int64_t)c.max_seqs * c.n_kv_heads * g->tail_bytes, 256);
  g->sinks_off = pos;
  g->sink_bytes = 4LL * g->sink_slots * d;  // K sink + V sink, fp16
  pos = align_up(pos + (int64_t)c.max_seqs * c.n_kv_heads * g->sink_bytes, 256);
  g->total_bytes = pos;
}

inline void make_ws_layout(const Geom& g, WsLayout* w) {
  w->units = g.max_seqs * g.hkv * g.slices;
  w->slot_floats = kHeadsPerSlice * (g.d + 4);
  w->err_off = 0;
  w->units_off = 256;
  w->tickets_off = align_up(w->units_off + 8LL * w->units, 256);   // zero between calls
  w->partials_off = align_up(w->tickets_off + 4LL * w->units, 256);
  w->total = align_up(w->partials_off + 2LL * kMaxDecodeCtas * w->slot_floats * 4, 256);
}

// ---- append / quantize ----------------------------------------------------
// Per-sequence arguments of one append launch.  The current lengths are
// not among them: the kernel reads them from the device copy, so a captured
// append stays correct when replayed (as long as its task counts do not
// depend on the lengths, i.e. every n_new < G).
struct AppendSeqs {
  int32_t n;                           // sequences in this launch
  int32_t seq0;                        // index of the first one in the cache
  int32_t task_prefix[kAppendMaxSeqs + 1];
  int32_t row_off[kAppendMaxSeqs];     // first input row of each sequence
  int32_t n_new[kAppendMaxSeqs];
};

cudaError_t launch_append(const Geom& g, unsigned char* cache, const void* k, const void* v,
                          int dtype, const AppendSeqs& seqs, int n_tasks, cudaStream_t stream);

// ---- decode ---------------------------------------------------------------
struct DecodeArgs {
  const unsigned char* cache;
  const void* q;
  int32_t q_dtype;
  void* out;             // fp16 [n_seq][hq][d]
  unsigned char* ws;
  int32_t n_seq;         // sequences of this launch
  int32_t seq0;          // cache index of its first sequence (q, out start there)
  int32_t inline_merge;  // split units merged by their last CTA (no combine kernel)
};

// Resident-CTA cap of the decode kernel for this geometry on the current device.
// wide: one 12-16 warp CTA per SM; else 4-warp CTAs, several per SM.
cudaError_t decode_max_ctas(const Geom& g, bool wide, int* max_ctas);
cudaError_t launch_decode(const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid,
                          bool wide, cudaStream_t stream);
// The same two entry points per (head dim, key bits, value bits, group),
// defined in the kvq_decode_d*_g*_v*.cu translation units.
#define KVQ_DECODE_DECLARE(D_, KB_, VB_, G_)                                              \
  cudaError_t decode_max_ctas_##D_##_##KB_##_##VB_##_##G_(const Geom& g, bool wide,       \
                                                          int* out);                      \
  cudaError_t launch_decode_##D_##_##KB_##_##VB_##_##G_(                                  \
      const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid, bool wide,         \
      cudaStream_t stream);
#define KVQ_DECODE_FOR_EACH(X) \
  X(128, 4, 2, 32) X(128, 2, 2, 32) X(128, 4, 2, 64) X(128, 2, 2, 64) \
  X(128, 4, 4, 32) X(128, 2, 4, 32) X(128, 4, 4, 64) X(128, 2, 4, 64) \
  X(64, 4, 2, 32) X(64, 2, 2, 32) X(64, 4, 2, 64) X(64, 2, 2, 64)     \
  X(64, 4, 4, 32) X(64, 2, 4, 32) X(64, 4, 4, 64) X(64, 2, 4, 64)
KVQ_DECODE_FOR_EACH(KVQ_DECODE_DECLARE)

// fp16 decode baseline over K, V [n_seq][Hkv][max_tokens][d] (a.seq0 and the
// device lengths `lens` index the cache; q and out start at a.seq0).
cudaError_t launch_decode_fp16(const Geom& g, const WsLayout& w, const DecodeArgs& a,
                               const void* k, const void* v, const int32_t* lens,
                               int max_tokens, int grid, cudaStream_t stream);

// Size of the fixed device scratch used by kvq_decode_noalloc, and the device
// address of that array on the current device (looked up on first use).
constexpr int64_t kNoAllocScratchBytes = 8LL << 20;
cudaError_t noalloc_scratch(void** ptr);

}  // namespace kvq
