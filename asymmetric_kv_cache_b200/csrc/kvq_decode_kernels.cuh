// Kernel templates of the split-K decode over the quantized cache (libkvq,
// sm_100a), shared by the translation units that instantiate them: one per
// (head dim, group, value bits) family, so that the library builds in
// parallel.  The design is described at the top of kvq_decode.cu (dispatch,
// fp16 baseline, no-alloc scratch); every definition here lives in an
// unnamed namespace, so each translation unit keeps its own copies.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_split.h"

namespace kvq {
namespace {


constexpr float kLog2e = 1.4426950408889634f;

// Staging area of the fp16 tail (T tokens, 0 < T < G) of one (sequence, kv
// head), 16 tokens at a time by cp.async: key rows and value token-pair
// rows, padded so that the fragment reads are free of bank conflicts; rows
// past T are zero-filled.  It is the tail warp's (idle) ring when that is
// large enough, else a CTA area of its own (a piece has at most one tail).
template <int D>
struct TailStage {
  static constexpr int KROW = 2 * D + 16;       // bytes per padded key row
  static constexpr int VROW = 4 * D + 16;       // bytes per padded value pair-row
  static constexpr int VOFF = 16 * KROW;
  static constexpr int BYTES = VOFF + 8 * VROW;
};

template <int D, int KB, int VB, int G, bool WIDE = true>
struct DecCfg {
  static constexpr int KT = D / 16;   // 16-channel k-tiles of q.k
  static constexpr int NT = G / 8;    // 8-token n-tiles of q.k
  static constexpr int KV = G / 16;   // 16-token k-tiles of p.v
  static constexpr int MT = D / 16;   // 16-channel m-tiles of p.v
  static constexpr int J = D / G;     // value channel groups per token
  static constexpr int FK = 16 / KB;  // code pairs per 32-bit word
  static constexpr int FV = 16 / VB;
  static constexpr int LWK = D * KB / 128;  // key-code words per lane per n-tile
  static constexpr int LWV = D * VB / 64;   // value-code words per lane per k-tile
  static constexpr int SEC_KCODES = 0;
  static constexpr int SEC_KSCALE = G * D * KB / 8;
  static constexpr int SEC_KMIN = SEC_KSCALE + 2 * D;
  static constexpr int SEC_VCODES = SEC_KMIN + 2 * D;
  static constexpr int SEC_VSCALE = SEC_VCODES + G * D * VB / 8;
  static constexpr int SEC_VMIN = SEC_VSCALE + 2 * G * J;
  static constexpr int BLK = SEC_VMIN + 2 * G * J;
  // Wide: one CTA per SM - 16 warps (128 registers each) for blocks up to
  // 4 KB, 12 (up to 168 registers) up to 7.5 KB, 8 above, so that the
  // 2-stage rings fit shared memory - for calls whose units are at most one
  // per SM, so that a CTA meets at most two unit pieces.  Narrow: 4 warps,
  // 4 CTAs per SM (3 above 4 KB blocks), for calls with more units, whose
  // CTAs cross many unit boundaries: the prologue and merge of one CTA's
  // piece then overlap the other CTAs' groups.
#ifndef KVQ_WIDE_WARPS_4K
#define KVQ_WIDE_WARPS_4K 16
#endif
  static constexpr int NW = !WIDE ? 4 : (BLK <= 4096) ? KVQ_WIDE_WARPS_4K : (BLK <= 7680) ? 12 : 8;
  static constexpr int THREADS = NW * 32;
  static constexpr int MIN_BLOCKS = WIDE ? 1 : (BLK <= 4096) ? 4 : 3;
  // Ring stages per warp.  Two keep more bytes in flight than the HBM
  // latency needs; deeper rings only lengthen the queue that every other
  // request (the query, the next unit's first blocks) waits behind.
  static constexpr int NST = 2;
  static constexpr int RING = NW * NST * BLK;
  // query fragments of the current unit, shared by the CTA's warps:
  // [kt][lane][4 words] = {hi v0, lo v0, hi v1, lo v1}.  The raw query rows
  // of the unit (<= 8 heads x D, fp32 at most) land here first by a bulk
  // copy and are converted in place.
  static constexpr int QA_OFF = RING;
  static constexpr int QA_BYTES = KT * 32 * 16;
  static_assert(kHeadsPerSlice * D * 4 <= QA_BYTES, "raw query rows fit the fragment area");
  // merge area (in the idle ring between pieces): the warps' (o, m, l) per
  // head, then the per-head weights of the NW warps, the max and the sum
  // rows of D + 8 floats (o[D], m, l, pad): a warp's stores of its state
  // then fall on 32 distinct banks
  static constexpr int MRS = D + 8;
  static constexpr int MERGE_FLOATS = NW * kHeadsPerSlice * MRS;
  static constexpr int WTS_OFF = MERGE_FLOATS;
  static_assert((MERGE_FLOATS + (NW + 2) * kHeadsPerSlice) * 4 <= RING,
                "merge area must fit in the ring");
  // The tail, in chunks of 16 tokens (< G/16 chunks without a recent
  // window, up to (R + G - 1)/16 with one, after the sink's chunks when
  // there is a sink window): chunk c belongs to warp
  // c mod TAIL_CHUNKS, which stages its first chunk when the piece starts
  // (its copy latency hidden behind the query's) and processes its chunks
  // one after another before claiming groups.  For 32-token groups the
  // chunks get an area of their own, for larger ones they go through the
  // warp's ring, which then starts its group copies late.
  static constexpr int TAIL_CHUNKS = G / 16;
  static constexpr bool TAIL_EARLY = (G == 32);
  static_assert(TAIL_EARLY || TailStage<D>::BYTES <= NST * BLK, "tail chunk fits a warp's ring");
  static_assert(TAIL_CHUNKS <= NW, "a warp per tail chunk");
  static constexpr int TAIL_OFF = QA_OFF + QA_BYTES;
  // the unit's query rows rotated by H / sqrt(d), fp32 (rotating caches)
  static constexpr int QR_OFF = TAIL_OFF + (TAIL_EARLY ? TAIL_CHUNKS * TailStage<D>::BYTES : 0);
  static constexpr int QR_BYTES = kHeadsPerSlice * D * 4;
  static constexpr int BAR_OFF = QR_OFF + QR_BYTES;
  // the merge's fp32 output rows before the back-rotation (at the end of the ring)
  static constexpr int OSCR_FLOATS = kHeadsPerSlice * D;
  static constexpr int MAX_MERGE_PIECES = (RING / 4 - OSCR_FLOATS) / (3 * kHeadsPerSlice);
  static constexpr int SMEM_FIXED = BAR_OFF + (NW * NST + 1) * 8 + 56;
};

// PK (packed): the GQA group has at most 4 heads, and the q.k tiles run
// transposed - rows 16 tokens, columns 4 heads' high parts then their low
// parts - so that no tile row or column is idle.
template <int D, int KB, int VB, int G, bool PK = false>
struct WarpState {
  float o[D / 16][4];   // O^T: (channel 16mt + g, heads 2i, 2i+1), then channel + 8
  float z[4];           // rows: value-min terms (j < J) and sum p (row J); cols heads
  float m[PK ? 2 : 1];  // running max, log2 domain: head lane/4, or (PK) heads
                        // 2(i&1), 2(i&1)+1
};

// Online-softmax update for new logits in the S tile layout: s[nt] =
// {(head g, token 8nt + 2i), (head g, token 8nt + 2i + 1)} (g = lane/4,
// i = lane&3).  Produces the fp16 probabilities pt[nt] in the same places,
// which is the B fragment of the value product (tokens 2i, 2i+1 of head g).
// The accumulators O^T and Z hold heads 2i and 2i+1 in their columns; their
// rescale factors come from the lanes that own those heads.
template <int D, int NT, int KB, int VB, int G>
__device__ __forceinline__ void softmax_update(WarpState<D, KB, VB, G>& st, float (&s)[NT][2],
                                               uint32_t (&pt)[NT], int i4) {
  float mx = fmaxf(s[0][0], s[0][1]);
#pragma unroll
  for (int nt = 1; nt < NT; ++nt) mx = fmaxf(mx, fmaxf(s[nt][0], s[nt][1]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));   // the 4 lanes of head g
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float n = fmaxf(st.m[0], mx);
  if (__any_sync(0xffffffffu, n > st.m[0])) {
    // every head gets its first logits in the same call: uniform branch
    if (st.m[0] != -INFINITY) {   // accumulators hold data: rescale them
      const float al = fast_exp2(st.m[0] - n);
      const float a0 = __shfl_sync(0xffffffffu, al, 8 * i4);
      const float a1 = __shfl_sync(0xffffffffu, al, 8 * i4 + 4);
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        st.o[mt][0] *= a0;
        st.o[mt][1] *= a1;
        st.o[mt][2] *= a0;
        st.o[mt][3] *= a1;
      }
      st.z[0] *= a0;
      st.z[1] *= a1;
      st.z[2] *= a0;
      st.z[3] *= a1;
    }
    st.m[0] = n;
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    pt[nt] = pack_h2(fast_exp2(s[nt][0] - st.m[0]), fast_exp2(s[nt][1] - st.m[0]));
}

// The value side of a group (O^T += V^T (p s_v), Z += [z_v; 1]^T p), shared
// by both layouts: pt[kv] = B fragments of 16 tokens.
// KBL: key width of the block's layout (the value sections follow its keys).
template <int D, int KB, int VB, int G, bool PK, int KBL = KB>
__device__ __forceinline__ void value_side(WarpState<D, KB, VB, G, PK>& st,
                                           const unsigned char* __restrict__ sp,
                                           const uint32_t (&pt)[G / 16][2], int lane) {
  using C = DecCfg<D, KBL, VB, G>;
  const int g8 = lane >> 2, i4 = lane & 3;
  const uint32_t* vcw = reinterpret_cast<const uint32_t*>(sp + C::SEC_VCODES);
  const uint32_t* vsw = reinterpret_cast<const uint32_t*>(sp + C::SEC_VSCALE);
  const uint32_t* vzw = reinterpret_cast<const uint32_t*>(sp + C::SEC_VMIN);
  // rows of the Z tile: row g8 < J takes its group's value mins, row J is (1, 1)
  const int zrow = g8 < C::J ? g8 : 0;
  const uint32_t zsel = g8 < C::J ? 0xFFFFFFFFu : 0u;
  const uint32_t zone = g8 == C::J ? 0x3C003C00u : 0u;
  static_for<C::KV>([&](auto kv_) {
    constexpr int kv = decltype(kv_)::value;
    const uint32_t bp0 = pt[kv][0], bp1 = pt[kv][1];
    const uint2 zz = *reinterpret_cast<const uint2*>(vzw + ((4 * kv + i4) * C::J + zrow) * 2);
    mma16816(st.z, (zz.x & zsel) | zone, 0u, (zz.y & zsel) | zone, 0u, bp0, bp1);

    uint32_t sw[2 * C::J];
    lds_words<2 * C::J>(vsw + (4 * kv + i4) * C::J * 2, sw);
    uint32_t bs[C::J][2];
#pragma unroll
    for (int j = 0; j < C::J; ++j) {
      bs[j][0] = hmul2_b(bp0, sw[2 * j]);
      bs[j][1] = hmul2_b(bp1, sw[2 * j + 1]);
    }
    uint32_t vw[C::LWV];
    lds_words<C::LWV>(vcw + (kv * 32 + lane) * C::LWV, vw);
    static_for<C::MT>([&](auto mt_) {
      constexpr int mt = decltype(mt_)::value;
      constexpr int TPW = C::FV / 4;     // channel tiles per word
      constexpr int wd = mt / TPW, u = mt % TPW;
      constexpr int j = (16 * mt) / G;
      const uint32_t a0 = unpack_pair<VB, 2 * u>(vw[wd]);
      const uint32_t a1 = unpack_pair<VB, 2 * u + 1>(vw[wd]);
      const uint32_t a2 = unpack_pair<VB, 2 * u + C::FV / 2>(vw[wd]);
      const uint32_t a3 = unpack_pair<VB, 2 * u + 1 + C::FV / 2>(vw[wd]);
      mma16816(st.o[mt], a0, a1, a2, a3, bs[j][0], bs[j][1]);
    });
  });
}

// One quantized group from the shared-memory stage `sp`.
//
// Key codes enter the tensor core as x = 1024 + m*code (code_offset) against
// A = q * (s_k/m) as fp16 high (rows 0-7) and residual (rows 8-15) parts
// (one fp16 rounding of the product would cost ~2^-12 of each logit term,
// which matters for channels with large scales); the offset is removed with
// one tile per k-step against a constant -1024 operand, which sums exactly
// the fp16 A values the tensor core saw, and accumulates with the key-min
// bias.  Value codes are unpacked to exact fp16 integers (unpack_pair).
// KBL: key width of the block (the state's KB unless the cache mixes widths).
template <int D, int KB, int VB, int G, int KBL = KB>
__device__ __forceinline__ void process_group(WarpState<D, KB, VB, G>& st,
                                              const unsigned char* __restrict__ sp,
                                              const uint4* __restrict__ qsm, int lane) {
  using C = DecCfg<D, KBL, VB, G>;
  constexpr int NT = G / 8;
  // key-code words held at once per token tile: all of them when that is at
  // most 8 registers, two at a time otherwise
  constexpr int WCH = (NT * C::LWK <= 8) ? C::LWK : (C::LWK >= 2 ? 2 : 1);
  constexpr int KT_PER_CH = WCH * C::FK / 2;   // k-steps covered by a chunk
  static_assert(C::KT % KT_PER_CH == 0, "k-steps split evenly into code chunks");
  const int i4 = lane & 3;

  const uint32_t* kcw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KCODES);
  const uint32_t* ksw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KSCALE) + i4 * (D / 8);
  const uint32_t* kzw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KMIN) + i4 * (D / 8);
  constexpr uint32_t kH2Neg1024 = 0xE400E400u;   // (-1024, -1024)

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  float bacc[4] = {0.f, 0.f, 0.f, 0.f};   // key-min bias (rows: high, low part)
  float cacc[4] = {0.f, 0.f, 0.f, 0.f};   // minus the code offset
  static_for<C::KT / KT_PER_CH>([&](auto ch_) {
    constexpr int ch = decltype(ch_)::value;
    uint32_t kw[NT][WCH];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      lds_words<WCH>(kcw + (nt * 32 + lane) * C::LWK + ch * WCH, kw[nt]);
    static_for<KT_PER_CH>([&](auto kk_) {
      constexpr int kt = ch * KT_PER_CH + decltype(kk_)::value;
      constexpr int p0 = 2 * kt, p1 = 2 * kt + 1;   // code pairs: channels +0-7, +8-15
      const uint2 s2 = *reinterpret_cast<const uint2*>(ksw + 2 * kt);
      const uint2 z2 = *reinterpret_cast<const uint2*>(kzw + 2 * kt);
      const uint4 q4 = qsm[kt * 32 + lane];
      // s_k / m of the code pair's field (a power-of-two scaling: exact
      // while s_k / m stays a normal fp16 number)
      constexpr int e0 = code_log2_mul<KBL, p0 % C::FK>(), e1 = code_log2_mul<KBL, p1 % C::FK>();
      const uint32_t sm0 = e0 ? hmul2_b(s2.x, h2_pow2_neg(e0)) : s2.x;
      const uint32_t sm1 = e1 ? hmul2_b(s2.y, h2_pow2_neg(e1)) : s2.y;
      // high part: one rounding of hi*s + lo*s; residual: (hi*s - high) in
      // one fused step (exact), plus lo*s
      const uint32_t a0 = hfma2_b(q4.x, sm0, hmul2_b(q4.y, sm0));
      const uint32_t a2 = hfma2_b(q4.z, sm1, hmul2_b(q4.w, sm1));
      const uint32_t a1 = hfma2_b(q4.y, sm0, hfma2_negc_b(q4.x, sm0, a0));
      const uint32_t a3 = hfma2_b(q4.w, sm1, hfma2_negc_b(q4.z, sm1, a2));
      mma16816(bacc, q4.x, q4.y, q4.z, q4.w, z2.x, z2.y);
      mma16816(cacc, a0, a1, a2, a3, kH2Neg1024, kH2Neg1024);
      static_for<NT>([&](auto nt_) {
        constexpr int nt = decltype(nt_)::value;
        constexpr int w0 = p0 / C::FK - ch * WCH, w1 = p1 / C::FK - ch * WCH;
        mma16816(acc[nt], a0, a1, a2, a3, code_offset<KBL, p0 % C::FK>(kw[nt][w0]),
                 code_offset<KBL, p1 % C::FK>(kw[nt][w1]));
      });
    });
  });
  // head g's bias: both row halves (every column holds the same value)
  const float bias = (bacc[0] + cacc[0]) + (bacc[2] + cacc[2]);
  float s[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    s[nt][0] = (acc[nt][0] + acc[nt][2]) + bias;
    s[nt][1] = (acc[nt][1] + acc[nt][3]) + bias;
  }

  uint32_t pt[G / 16][2];   // B fragments of the value product, 16 tokens each
  softmax_update<D, NT, KB, VB, G>(st, s, *reinterpret_cast<uint32_t(*)[NT]>(&pt[0][0]),
                                   lane & 3);
  value_side<D, KB, VB, G, false, KBL>(st, sp, pt, lane);
}

// Decode slots of a unit with L tokens: its quantized groups plus one for a
// non-empty tail (the window-free form when WIN is false).
template <int G, bool WIN>
__device__ __forceinline__ int dec_unit_slots(int L, const Geom& g) {
  if constexpr (WIN) return unit_slots_s(L, G, g.window, g.sink);
  else return L / G + (L % G ? 1 : 0);
}

// Ring slot of the first token of tail chunk c (tokens 16c .. 16c + 15 of a
// tail whose first token sits at sequence position `first`) in a tail ring
// of W slots (token p in slot p mod W).  first and W are multiples of 16, so
// a chunk never wraps.
__device__ __forceinline__ int tail_chunk_slot(int first, int c, int W) {
  return (first + 16 * c) % W;
}

// Where fp16 chunk c (16 tokens) of a unit lives, for caches with a sink
// and/or a recent window: chunks 0 .. ns-1 are the sink (tokens 16c ..,
// ns = ceil(min(L, sink) / 16)), the rest the tail ring's chunks (tail chunk
// c - ns starts at ring slot (ng G + 16 (c - ns)) mod W, positions counted
// after the sink).  Returns the key and value base pointers and the chunk's
// token count.
template <int D, int G>
__device__ __forceinline__ int fp16_chunk_src(const Geom& g, const unsigned char* cache,
                                              int64_t ui, int L, int ng, int Tb, int c,
                                              const __half*& k, const __half*& v) {
  const int Sb = min(L, g.sink);
  const int ns = (Sb + 15) / 16;
  if (c < ns) {
    const __half* sk = reinterpret_cast<const __half*>(cache + g.sinks_off + ui * g.sink_bytes);
    k = sk + (int64_t)16 * c * D;
    v = sk + (int64_t)g.sink_slots * D + (int64_t)16 * c * D;
    return min(16, Sb - 16 * c);
  }
  const int ct = c - ns;
  const __half* tk = reinterpret_cast<const __half*>(cache + g.tails_off + ui * g.tail_bytes);
  const int64_t so = (int64_t)tail_chunk_slot(ng * G, ct, g.tail_slots) * D;
  k = tk + so;
  v = tk + (int64_t)g.tail_slots * D + so;
  return min(16, Tb - 16 * ct);
}
// Chunks of the fp16 slot: the sink's, then the tail's.
__device__ __forceinline__ int fp16_chunks(const Geom& g, int L, int Tb) {
  return (min(L, g.sink) + 15) / 16 + (Tb + 15) / 16;
}

// Debug builds: the key rows and value token-pair rows that staging chunk
// kv (T tokens) reads from k and v must lie inside the cache's fp16 tail and
// sink regions (check 4).  Always true in release builds.
template <int D>
__device__ __forceinline__ bool debug_fp16_rows(const Geom& g, const unsigned char* cache,
                                                const __half* k, const __half* v, int T, int kv,
                                                int32_t* err) {
  if (!kDebug) return true;
  const int rows = min(16, T - 16 * kv);
  if (rows <= 0) return true;
  const unsigned char* lo = cache + g.tails_off;
  const unsigned char* hi = cache + g.total_bytes;
  const unsigned char* k0 = reinterpret_cast<const unsigned char*>(k + (int64_t)16 * kv * D);
  const unsigned char* k1 = reinterpret_cast<const unsigned char*>(k + (int64_t)(16 * kv + rows) * D);
  const unsigned char* v0 = reinterpret_cast<const unsigned char*>(v + (int64_t)16 * kv * D);
  const unsigned char* v1 = reinterpret_cast<const unsigned char*>(
      v + (int64_t)(16 * kv + ((rows + 1) & ~1)) * D);
  return debug_ok(k0 >= lo && k1 <= hi && v0 >= lo && v1 <= hi, err, 4);
}

// Issue the cp.async copies of tail chunk kv (16 tokens: key rows and
// value token-pair rows) into `buf`; nothing waits here.
template <int D>
__device__ __forceinline__ void stage_tail_chunk(unsigned char* __restrict__ buf,
                                                 const __half* __restrict__ tk,
                                                 const __half* __restrict__ tv, int T, int kv,
                                                 int lane) {
  using TS = TailStage<D>;
  for (int seg = lane; seg < 16 * (D / 8); seg += 32) {
    const int r = seg / (D / 8), cs = seg % (D / 8), t = 16 * kv + r;
    cp_async16(buf + r * TS::KROW + cs * 16, tk + (t < T ? (int64_t)t * D + cs * 8 : 0),
               t < T ? 16u : 0u);
  }
  for (int seg = lane; seg < 8 * (D / 4); seg += 32) {
    const int pr = seg / (D / 4), cs = seg % (D / 4), pp = 8 * kv + pr;
    cp_async16(buf + TS::VOFF + pr * TS::VROW + cs * 16,
               tv + (2 * pp < T ? (int64_t)pp * 2 * D + cs * 8 : 0), 2 * pp < T ? 16u : 0u);
  }
}

// Attention over staged tail chunk kv (tokens 16kv .. 16kv + 15, those
// past T masked out).
template <int D, int KB, int VB, int G>
__device__ __forceinline__ void tail_chunk(WarpState<D, KB, VB, G>& st,
                                           const unsigned char* __restrict__ buf, int T, int kv,
                                           const uint4* __restrict__ qsm, int lane) {
  using C = DecCfg<D, KB, VB, G>;
  using TS = TailStage<D>;
  const int g8 = lane >> 2, i4 = lane & 3;
  {
    // S = q K^T, rows: q high / low parts, columns: 8 tokens per tile
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const unsigned char* k0 = buf + g8 * TS::KROW + 4 * i4;
#pragma unroll
    for (int kt = 0; kt < C::KT; ++kt) {
      const uint4 q4 = qsm[kt * 32 + lane];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const unsigned char* kr = k0 + 8 * nt * TS::KROW + 32 * kt;
        mma16816(acc[nt], q4.x, q4.y, q4.z, q4.w, *reinterpret_cast<const uint32_t*>(kr),
                 *reinterpret_cast<const uint32_t*>(kr + 16));
      }
    }
    float s[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int t = 16 * kv + 8 * nt + 2 * i4;
      s[nt][0] = (t < T) ? acc[nt][0] + acc[nt][2] : -INFINITY;
      s[nt][1] = (t + 1 < T) ? acc[nt][1] + acc[nt][3] : -INFINITY;
    }
    uint32_t pt[2];
    softmax_update<D, 2, KB, VB, G>(st, s, pt, i4);
    const uint32_t ones = (g8 == C::J) ? 0x3C003C00u : 0u;
    mma16816(st.z, ones, 0u, ones, 0u, pt[0], pt[1]);
    // V^T fragments; the second token of the last pair may be stale: mask it
    const int ta = 16 * kv + 2 * i4, tb = ta + 8;
    const uint32_t ma = (ta + 1 < T) ? 0xFFFFFFFFu : 0x0000FFFFu;
    const uint32_t mb = (tb + 1 < T) ? 0xFFFFFFFFu : 0x0000FFFFu;
    const unsigned char* va = buf + TS::VOFF + i4 * TS::VROW + 4 * g8;
    const unsigned char* vb = va + 4 * TS::VROW;
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) {
      const uint32_t a0 = *reinterpret_cast<const uint32_t*>(va + 64 * mt) & ma;
      const uint32_t a1 = *reinterpret_cast<const uint32_t*>(va + 64 * mt + 32) & ma;
      const uint32_t a2 = *reinterpret_cast<const uint32_t*>(vb + 64 * mt) & mb;
      const uint32_t a3 = *reinterpret_cast<const uint32_t*>(vb + 64 * mt + 32) & mb;
      mma16816(st.o[mt], a0, a1, a2, a3, pt[0], pt[1]);
    }
  }
}

// ---------------------------------------------------------------------------
// Packed variant (GQA group of at most 4 heads).
//
// S^T = codes q'^T on m16n8k16 tiles: rows = 16 tokens (two 8-token code
// tiles), columns n = heads 0-3 with q' rounded to fp16 (n < 4) and the
// rounding residual of the same heads (n >= 4).  Lane (g, i) then holds the
// B operand of column g, so each lane computes either a high or a low part:
// its query words (convert_query) are y = (low lane ? q_hi : 0) and
// x = (low lane ? q_lo : q_hi), and
//   h = y s,  B = x s + (y s - h)
// gives fp16(q_hi s) on high lanes (y = 0) and the exact residual of that
// product on low lanes with the same instructions.  The two halves of a
// logit meet with one shuffle (lane i and i ^ 2 hold columns n and n + 4).
// The fp16 tail's B operand is x itself (q_hi on high lanes, q_lo on low).

// The query conversion split over NCW warps (k-tiles cw, cw + NCW, ...):
// every converting warp reads its raw values first, the warps meet at a
// named barrier, then they write their fragments into the same bytes.
// q is scaled by log2(e)/sqrt(d) and split into fp16 high and low parts; the
// fragments of k-step kt sit at qs[kt * 32 + lane] as a quad over the
// channels 16kt + 2i + {0,1} (v = 0) and + 8 (v = 1), i = lane & 3:
//   PK = false: {hi v0, lo v0, hi v1, lo v1} of head lane/4 - the A quad of
//     the q.k tiles (rows g: high part, rows g + 8: low part);
//   PK: {y v0, x v0, y v1, x v1} of head (lane/4) mod 4 (see above).
// A padding head gets zeros.
template <int D, bool PK, int NCW>
__device__ __forceinline__ void convert_query(int dtype, int nh, bool ok, int cw, int lane,
                                              uint4* qs, const unsigned char* raw) {
  constexpr int KT = D / 16;
  static_assert(KT % NCW == 0, "k-tiles split evenly over the converting warps");
  constexpr int J = KT / NCW;
  const int g8 = lane >> 2, i4 = lane & 3;
  const int hh = PK ? (g8 & 3) : g8;
  const bool low = PK && g8 >= 4;
  const bool valid = ok && hh < nh;
  const float sc = kLog2e * rsqrtf((float)D);
  float2 x[J][2];
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int kt = cw + j * NCW;
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int idx = hh * D + 16 * kt + 8 * v + 2 * i4;
      float2 f = make_float2(0.f, 0.f);
      if (valid) {
        if (dtype == KVQ_FP16) {
          f = __half22float2(*reinterpret_cast<const __half2*>(raw + 2 * idx));
        } else if (dtype == KVQ_BF16) {
          f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(raw + 2 * idx));
        } else {
          f = *reinterpret_cast<const float2*>(raw + 4 * idx);
        }
      }
      x[j][v] = f;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int kt = cw + j * NCW;
    uint32_t wv[4];
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const float x0 = x[j][v].x * sc, x1 = x[j][v].y * sc;
      const __half2 h = __floats2half2_rn(x0, x1);
      const float2 hf = __half22float2(h);
      const uint32_t hi = h2_as_u32(h);
      const uint32_t lo = pack_h2(x0 - hf.x, x1 - hf.y);
      wv[2 * v] = (PK && !low) ? 0u : hi;
      wv[2 * v + 1] = (PK && !low) ? hi : lo;
    }
    qs[kt * 32 + lane] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
}

// Rotating caches: the unit's raw query rows (head hh at hh * D elements of
// `raw`, dtype) rotated by H / sqrt(d) into fp32 rows `qr`, before the
// conversion into fragments (the cache holds rotated keys, so q . k is the
// same in the rotated domain).  Converting warp cw takes heads cw, cw + NCW,
// ...; a lane holds D / 32 consecutive channels.
template <int D, int NCW>
__device__ __forceinline__ void rotate_query_rows(int dtype, int nh, bool ok, int cw, int lane,
                                                  const unsigned char* raw, float* qr) {
  constexpr int V = D / 32;
  for (int hh = cw; hh < nh; hh += NCW) {
    float y[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int idx = hh * D + V * lane + j;
      y[j] = !ok ? 0.f
             : dtype == KVQ_FP16 ? __half2float(reinterpret_cast<const __half*>(raw)[idx])
             : dtype == KVQ_BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(raw)[idx])
                                 : reinterpret_cast<const float*>(raw)[idx];
    }
    fwht_lanes<D, V>(y, lane);
#pragma unroll
    for (int j = 0; j < V; ++j) qr[hh * D + V * lane + j] = y[j] * rot_scale<D>();
  }
}

// A warp's four channels (4l .. 4l + 3) of a head's output row, rotated
// back by H / sqrt(d) when `rot` (D / 4 lanes per row, aligned groups).
template <int D>
__device__ __forceinline__ float4 rotate_out4(float4 o, int l, bool rot) {
  if (!rot) return o;
  float y[4] = {o.x, o.y, o.z, o.w};
  fwht_lanes<D, 4>(y, l);
  const float sc = rot_scale<D>();
  return make_float4(y[0] * sc, y[1] * sc, y[2] * sc, y[3] * sc);
}

// Per-head weights of the NW warps' pieces, (h, warp) per thread: the
// head's max M and sum L over the warps, and each warp's factor
// 2^(m_w - M) (divided by L when the piece is the whole unit).
template <int D, int NW, int RS = D + 2>
__device__ __forceinline__ void merge_weights(const float* __restrict__ merge,
                                              float* __restrict__ wts, bool whole, int tid) {
  constexpr int NWP = NW <= 4 ? 4 : NW <= 8 ? 8 : 16;   // lanes per head
  static_assert(NW <= 16, "at most 16 warps");
  if (tid < kHeadsPerSlice * NWP) {   // whole warps: 8 * NWP is a multiple of 32
    const int h = tid / NWP, ww = tid % NWP;
    const bool v = ww < NW;
    const float* mo = merge + (ww * kHeadsPerSlice + h) * RS;
    const float mw = v ? mo[D] : -INFINITY;
    const float lw = v ? mo[D + 1] : 0.f;
    float M = mw;
#pragma unroll
    for (int o = 1; o < NWP; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
    float Ls = f * lw;
#pragma unroll
    for (int o = 1; o < NWP; o <<= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (v) wts[h * NW + ww] = whole ? f / Ls : f;
    if (ww == 0) {
      wts[NW * kHeadsPerSlice + h] = M;
      wts[(NW + 1) * kHeadsPerSlice + h] = Ls;
    }
  }
}

// Online softmax in the S^T layout: s[mt] = {(token g, head 2i'), (g, 2i'+1),
// (g+8, 2i'), (g+8, 2i'+1)}, i' = i & 1 (lanes i and i ^ 2 agree).  P goes
// through movmatrix into the B fragments of the value product; its columns
// 4-7 repeat heads 0-3 and are never read back.
template <int D, int NM, int KB, int VB, int G>
__device__ __forceinline__ void softmax_pk(WarpState<D, KB, VB, G, true>& st, float (&s)[NM][4],
                                           uint32_t (&pt)[NM][2]) {
  float mx0 = fmaxf(s[0][0], s[0][2]), mx1 = fmaxf(s[0][1], s[0][3]);
#pragma unroll
  for (int mt = 1; mt < NM; ++mt) {
    mx0 = fmaxf(mx0, fmaxf(s[mt][0], s[mt][2]));
    mx1 = fmaxf(mx1, fmaxf(s[mt][1], s[mt][3]));
  }
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1) {   // across the 8 token rows (lane bits 2-4)
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const float n0 = fmaxf(st.m[0], mx0), n1 = fmaxf(st.m[1], mx1);
  if (__any_sync(0xffffffffu, n0 > st.m[0] || n1 > st.m[1])) {
    if (st.m[0] != -INFINITY) {   // accumulators hold data: rescale them
      const float a0 = fast_exp2(st.m[0] - n0), a1 = fast_exp2(st.m[1] - n1);
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        st.o[mt][0] *= a0;
        st.o[mt][1] *= a1;
        st.o[mt][2] *= a0;
        st.o[mt][3] *= a1;
      }
      st.z[0] *= a0;
      st.z[1] *= a1;
      st.z[2] *= a0;
      st.z[3] *= a1;
    }
    st.m[0] = n0;
    st.m[1] = n1;
  }
#pragma unroll
  for (int mt = 0; mt < NM; ++mt) {
    pt[mt][0] = movmatrix_trans(
        pack_h2(fast_exp2(s[mt][0] - st.m[0]), fast_exp2(s[mt][1] - st.m[1])));
    pt[mt][1] = movmatrix_trans(
        pack_h2(fast_exp2(s[mt][2] - st.m[0]), fast_exp2(s[mt][3] - st.m[1])));
  }
}

// Logits of one group in the S^T layout (first packed form): s[mt] =
// {(token g, head 2i'), (g, 2i'+1), (g+8, 2i'), (g+8, 2i'+1)}, i' = i & 1.
template <int D, int KB, int VB, int G>
__device__ __forceinline__ void kside_pk(const unsigned char* __restrict__ sp,
                                         const uint4* __restrict__ qsm, int lane,
                                         float (&s)[G / 16][4]) {
  using C = DecCfg<D, KB, VB, G>;
  constexpr int NM = G / 16;
  constexpr int NT = G / 8;
  constexpr int WCH = (NT * C::LWK <= 8) ? C::LWK : (C::LWK >= 2 ? 2 : 1);
  constexpr int KT_PER_CH = WCH * C::FK / 2;
  static_assert(C::KT % KT_PER_CH == 0, "k-steps split evenly into code chunks");
  const int i4 = lane & 3;
  const uint32_t* kcw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KCODES);
  const uint32_t* ksw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KSCALE) + i4 * (D / 8);
  const uint32_t* kzw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KMIN) + i4 * (D / 8);
  constexpr uint32_t kH2Neg1024 = 0xE400E400u;

  float acc[NM][4];
#pragma unroll
  for (int mt = 0; mt < NM; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float oacc[4] = {0.f, 0.f, 0.f, 0.f};   // minus the code offset, per column
  // the key-min bias sum_c q_c z_c on an untransposed tile: A = the query
  // quad (rows g: y of head g mod 4, rows g + 8: x), B = the mins (the same
  // in every column): rows g + 4 (q_hi) and g + 12 (q_lo), g < 4, hold the
  // bias of head g - no operand to build
  float zacc[4] = {0.f, 0.f, 0.f, 0.f};
  static_for<C::KT / KT_PER_CH>([&](auto ch_) {
    constexpr int ch = decltype(ch_)::value;
    uint32_t kw[NT][WCH];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      lds_words<WCH>(kcw + (nt * 32 + lane) * C::LWK + ch * WCH, kw[nt]);
    static_for<KT_PER_CH>([&](auto kk_) {
      constexpr int kt = ch * KT_PER_CH + decltype(kk_)::value;
      constexpr int p0 = 2 * kt, p1 = 2 * kt + 1;
      const uint2 s2 = *reinterpret_cast<const uint2*>(ksw + 2 * kt);
      const uint2 z2 = *reinterpret_cast<const uint2*>(kzw + 2 * kt);
      const uint4 q4 = qsm[kt * 32 + lane];   // {y v0, x v0, y v1, x v1}
      constexpr int e0 = code_log2_mul<KB, p0 % C::FK>(), e1 = code_log2_mul<KB, p1 % C::FK>();
      const uint32_t sm0 = e0 ? hmul2_b(s2.x, h2_pow2_neg(e0)) : s2.x;
      const uint32_t sm1 = e1 ? hmul2_b(s2.y, h2_pow2_neg(e1)) : s2.y;
      const uint32_t h0 = hmul2_b(q4.x, sm0), h1 = hmul2_b(q4.z, sm1);
      const uint32_t b0 = hfma2_b(q4.y, sm0, hfma2_negc_b(q4.x, sm0, h0));
      const uint32_t b1 = hfma2_b(q4.w, sm1, hfma2_negc_b(q4.z, sm1, h1));
      mma16816(zacc, q4.x, q4.y, q4.z, q4.w, z2.x, z2.y);
      mma16816(oacc, kH2Neg1024, kH2Neg1024, kH2Neg1024, kH2Neg1024, b0, b1);
      static_for<NM>([&](auto mt_) {
        constexpr int mt = decltype(mt_)::value;
        constexpr int w0 = p0 / C::FK - ch * WCH, w1 = p1 / C::FK - ch * WCH;
        mma16816(acc[mt], code_offset<KB, p0 % C::FK>(kw[2 * mt][w0]),
                 code_offset<KB, p0 % C::FK>(kw[2 * mt + 1][w0]),
                 code_offset<KB, p1 % C::FK>(kw[2 * mt][w1]),
                 code_offset<KB, p1 % C::FK>(kw[2 * mt + 1][w1]), b0, b1);
      });
    });
  });
  // column 2 i4 + e (after the high + low sum) is head h = (2 i4 + e) mod 4,
  // whose whole bias (high rows + low rows) sits in lane 4 (h + 4)
  const float zb = zacc[0] + zacc[2];
  const float bias0 = __shfl_sync(0xffffffffu, zb, 16 + 4 * ((2 * i4) & 3));
  const float bias1 = __shfl_sync(0xffffffffu, zb, 16 + 4 * ((2 * i4 + 1) & 3));
#pragma unroll
  for (int mt = 0; mt < NM; ++mt) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float x = acc[mt][r] + oacc[r & 1];
      s[mt][r] = (x + __shfl_xor_sync(0xffffffffu, x, 2)) + ((r & 1) ? bias1 : bias0);
    }
  }
}

template <int D, int KB, int VB, int G, int KBL = KB>
__device__ __forceinline__ void process_group_pk(WarpState<D, KB, VB, G, true>& st,
                                                 const unsigned char* __restrict__ sp,
                                                 const uint4* __restrict__ qsm, int lane) {
  constexpr int NM = G / 16;
  float s[NM][4];
  kside_pk<D, KBL, VB, G>(sp, qsm, lane, s);
  uint32_t pt[NM][2];
  softmax_pk<D, NM, KB, VB, G>(st, s, pt);
  value_side<D, KB, VB, G, true, KBL>(st, sp, pt, lane);
}

template <int D, int KB, int VB, int G>
__device__ __forceinline__ void tail_chunk_pk(WarpState<D, KB, VB, G, true>& st,
                                              const unsigned char* __restrict__ buf, int T, int kv,
                                              const uint4* __restrict__ qsm, int lane) {
  using C = DecCfg<D, KB, VB, G>;
  using TS = TailStage<D>;
  const int g8 = lane >> 2, i4 = lane & 3;
  // S^T = K q^T: rows 16 tokens, columns q_hi (n < 4) / q_lo (n >= 4): the
  // lanes' x words
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const unsigned char* k0 = buf + g8 * TS::KROW + 4 * i4;
  const unsigned char* k1 = k0 + 8 * TS::KROW;
#pragma unroll
  for (int kt = 0; kt < C::KT; ++kt) {
    const uint4 q4 = qsm[kt * 32 + lane];
    const uint32_t b0 = q4.y, b1 = q4.w;
    mma16816(acc, *reinterpret_cast<const uint32_t*>(k0 + 32 * kt),
             *reinterpret_cast<const uint32_t*>(k1 + 32 * kt),
             *reinterpret_cast<const uint32_t*>(k0 + 32 * kt + 16),
             *reinterpret_cast<const uint32_t*>(k1 + 32 * kt + 16), b0, b1);
  }
  const int t0 = 16 * kv + g8, t1 = t0 + 8;
  float s[1][4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float x = acc[r] + __shfl_xor_sync(0xffffffffu, acc[r], 2);
    s[0][r] = ((r < 2 ? t0 : t1) < T) ? x : -INFINITY;
  }
  uint32_t pt[1][2];
  softmax_pk<D, 1, KB, VB, G>(st, s, pt);
  const uint32_t ones = (g8 == C::J) ? 0x3C003C00u : 0u;
  mma16816(st.z, ones, 0u, ones, 0u, pt[0][0], pt[0][1]);
  const int ta = 16 * kv + 2 * i4, tb = ta + 8;
  const uint32_t ma = (ta + 1 < T) ? 0xFFFFFFFFu : 0x0000FFFFu;
  const uint32_t mb = (tb + 1 < T) ? 0xFFFFFFFFu : 0x0000FFFFu;
  const unsigned char* va = buf + TS::VOFF + i4 * TS::VROW + 4 * g8;
  const unsigned char* vb = va + 4 * TS::VROW;
#pragma unroll
  for (int mt = 0; mt < C::MT; ++mt) {
    const uint32_t a0 = *reinterpret_cast<const uint32_t*>(va + 64 * mt) & ma;
    const uint32_t a1 = *reinterpret_cast<const uint32_t*>(va + 64 * mt + 32) & ma;
    const uint32_t a2 = *reinterpret_cast<const uint32_t*>(vb + 64 * mt) & mb;
    const uint32_t a3 = *reinterpret_cast<const uint32_t*>(vb + 64 * mt + 32) & mb;
    mma16816(st.o[mt], a0, a1, a2, a3, pt[0][0], pt[0][1]);
  }
}

// The last CTA to finish a split unit merges the unit's pieces.  Every
// piece's CTA has written its partial (o, m, l per head); the CTA's threads
// meet at a barrier, one thread bumps the unit's ticket with an acquire-
// release atomic at GPU scope (so the partials written before it by any
// piece's CTA are visible to whoever sees the final count), and the CTA
// that brings the count to the number of pieces reads every piece back
// from L2 and writes the output.  Piece 0 is the unit's first slot's CTA
// kf (partial slot 2kf if the unit starts its range, else 2kf + 1); pieces
// 1.. are the first pieces of CTAs kf + 1 .. kl (slots 2k).
template <int D, int THREADS>
__device__ __noinline__ void finish_split_unit(const Geom& g, const WsLayout& w,
                                               const DecodeArgs& a, int unit, int64_t p0,
                                               int wb, int T, int grid, int b, int hbase, int nh,
                                               float* __restrict__ scratch, int max_pieces,
                                               int* __restrict__ flag, int tid, bool rot,
                                               float* __restrict__ oscr) {
  int32_t* tickets = reinterpret_cast<int32_t*>(a.ws + w.tickets_off);
  const float* partials = reinterpret_cast<const float*>(a.ws + w.partials_off);
  int32_t* err = reinterpret_cast<int32_t*>(a.ws + w.err_off);
  __syncthreads();
  if (tid == 0) {
    const MergePlan mp = merge_plan(p0, wb, T, grid);
    // debug builds: the ticket, every piece's partial slot, the output rows
    // and the shared scratch must fit their buffers (checks 10, 9, 8, 11);
    // a failed check skips the merge
    const bool fits =
        debug_ok(unit >= 0 && unit < w.units, err, 10) &&
        debug_ok(mp.kf >= 0 && merge_piece_slot(mp.kf, mp.s0, mp.npc - 1) < 2 * grid &&
                     w.partials_off + (int64_t)2 * grid * w.slot_floats * 4 <= w.total,
                 err, 9) &&
        debug_ok(b < a.n_seq && hbase + nh <= g.hq, err, 8) &&
        debug_ok(mp.npc <= 32 || mp.npc <= max_pieces, err, 11);
    int npc = 0;
    if (fits) {
      const int old = atomic_add_acq_rel_gpu(tickets + unit, 1);
      const bool last = old == mp.npc - 1;
      if (last) tickets[unit] = 0;   // every piece has counted: ready for the next call
      npc = last ? mp.npc : 0;
    }
    flag[0] = npc;
    flag[1] = mp.kf;
    flag[2] = mp.s0;
  }
  __syncthreads();
  const int npc = flag[0], kf = flag[1], s0 = flag[2];
  if (npc == 0) return;
  auto piece = [&](int pc, int h) {
    return partials + (int64_t)merge_piece_slot(kf, s0, pc) * w.slot_floats + h * (D + 4);
  };
  // the unit's output: fp16 rows of out, or (rotating caches) fp32 rows of
  // oscr, rotated back and written by the epilogue below
  __half* orow = reinterpret_cast<__half*>(a.out) + ((int64_t)b * g.hq + hbase) * D;
  auto put = [&](int h, int c, float v) {
    if (rot) oscr[h * D + c] = v;
    else orow[h * D + c] = __float2half_rn(v);
  };
  if (npc > 4 && npc <= 32) {
    // up to 32 pieces: an item is (head, 4 channels); 4 threads share an
    // item, each loading its pieces' 4 values and (m, l) (up to 8 pieces,
    // every load in flight at once: one round of L2 latency), merging them
    // in registers, then the 4 threads merge through shuffles
    constexpr int TPI = 4;
    const int sub = tid % TPI;
    for (int it = tid / TPI; it < nh * (D / 4); it += THREADS / TPI) {
      const int h = it / (D / 4), c = 4 * (it % (D / 4));
      float2 ml[8];
      float4 o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int pc = sub + TPI * k;
        if (pc < npc) {
          ml[k] = __ldcg(reinterpret_cast<const float2*>(piece(pc, h) + D));
          o[k] = __ldcg(reinterpret_cast<const float4*>(piece(pc, h) + c));
        } else {
          ml[k] = make_float2(-INFINITY, 0.f);
          o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float M = ml[0].x;
#pragma unroll
      for (int k = 1; k < 8; ++k) M = fmaxf(M, ml[k].x);
      M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
      M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
      float L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float f = ml[k].x == -INFINITY ? 0.f : fast_exp2(ml[k].x - M);
        L = fmaf(f, ml[k].y, L);
        O.x = fmaf(f, o[k].x, O.x);
        O.y = fmaf(f, o[k].y, O.y);
        O.z = fmaf(f, o[k].z, O.z);
        O.w = fmaf(f, o[k].w, O.w);
      }
#pragma unroll
      for (int x = 1; x < TPI; x <<= 1) {
        L += __shfl_xor_sync(0xffffffffu, L, x);
        O.x += __shfl_xor_sync(0xffffffffu, O.x, x);
        O.y += __shfl_xor_sync(0xffffffffu, O.y, x);
        O.z += __shfl_xor_sync(0xffffffffu, O.z, x);
        O.w += __shfl_xor_sync(0xffffffffu, O.w, x);
      }
      if (sub == 0) {
        const float inv = 1.0f / L;
        const float4 on = make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
        if (rot)
          *reinterpret_cast<float4*>(oscr + h * D + c) = on;
        else
          *reinterpret_cast<uint2*>(orow + h * D + c) =
              make_uint2(pack_h2(on.x, on.y), pack_h2(on.z, on.w));
      }
    }
  } else if (npc <= 4) {
    // few pieces: every thread loads its element's values and the pieces'
    // (m, l) in one round of L2 loads and forms the weights itself
    for (int idx = tid; idx < nh * D; idx += THREADS) {
      const int h = idx / D, c = idx % D;
      float2 ml[4];
      float o[4];
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        if (pc < npc) {
          ml[pc] = __ldcg(reinterpret_cast<const float2*>(piece(pc, h) + D));
          o[pc] = __ldcg(piece(pc, h) + c);
        } else {
          ml[pc] = make_float2(-INFINITY, 0.f);
          o[pc] = 0.f;
        }
      }
      float M = fmaxf(fmaxf(ml[0].x, ml[1].x), fmaxf(ml[2].x, ml[3].x));
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        const float f = ml[pc].x == -INFINITY ? 0.f : fast_exp2(ml[pc].x - M);
        L += f * ml[pc].y;
        O += f * o[pc];
      }
      put(h, c, O / L);
    }
  } else if (npc <= max_pieces) {
    // (m, l) of every (piece, head) in one round of loads, then the per-head
    // weights, then every element's pieces with all loads in flight
    float* mlw = scratch;                              // [pc][h]: m, l
    float* wt = scratch + 2 * kHeadsPerSlice * npc;    // [pc][h]: weight
    for (int i = tid; i < npc * kHeadsPerSlice; i += THREADS) {
      const int pc = i / kHeadsPerSlice, h = i % kHeadsPerSlice;
      const float2 ml = h < nh ? __ldcg(reinterpret_cast<const float2*>(piece(pc, h) + D))
                               : make_float2(-INFINITY, 0.f);
      mlw[2 * i] = ml.x;
      mlw[2 * i + 1] = ml.y;
    }
    __syncthreads();
    if (tid < kHeadsPerSlice) {
      const int h = tid;
      float M = -INFINITY;
      for (int pc = 0; pc < npc; ++pc) M = fmaxf(M, mlw[2 * (pc * kHeadsPerSlice + h)]);
      float L = 0.f;
      for (int pc = 0; pc < npc; ++pc) {
        const float m = mlw[2 * (pc * kHeadsPerSlice + h)];
        const float f = m == -INFINITY ? 0.f : fast_exp2(m - M);
        wt[pc * kHeadsPerSlice + h] = f;
        L += f * mlw[2 * (pc * kHeadsPerSlice + h) + 1];
      }
      const float inv = 1.0f / L;
      for (int pc = 0; pc < npc; ++pc) wt[pc * kHeadsPerSlice + h] *= inv;
    }
    __syncthreads();
    for (int idx = tid; idx < nh * D; idx += THREADS) {
      const int h = idx / D, c = idx % D;
      float O = 0.f;
      int pc = 0;
      for (; pc + 4 <= npc; pc += 4) {
        float x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = __ldcg(piece(pc + u, h) + c);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float f = wt[(pc + u) * kHeadsPerSlice + h];
          if (f != 0.f) O += f * x[u];
        }
      }
      for (; pc < npc; ++pc) {
        const float f = wt[pc * kHeadsPerSlice + h];
        if (f != 0.f) O += f * __ldcg(piece(pc, h) + c);
      }
      put(h, c, O);
    }
  } else {
  // more pieces than the scratch holds: an online merge per element
  for (int idx = tid; idx < nh * D; idx += THREADS) {
    const int h = idx / D, c = idx % D;
    float M = -INFINITY, L = 0.f, O = 0.f;
    for (int pc = 0; pc < npc; ++pc) {
      const float* ps = piece(pc, h);
      const float m = __ldcg(ps + D);
      if (m == -INFINITY) continue;
      const float l = __ldcg(ps + D + 1), o = __ldcg(ps + c);
      const float Mn = fmaxf(M, m);
      const float sa = (M == -INFINITY) ? 0.f : fast_exp2(M - Mn), sb = fast_exp2(m - Mn);
      L = L * sa + l * sb;
      O = O * sa + o * sb;
      M = Mn;
    }
    put(h, c, O / L);
  }
  }
  if (rot) {
    // rotating caches: each head's fp32 row rotated back by H / sqrt(d),
    // four channels per lane (whole warps, D / 4 lanes per row)
    __syncthreads();
    for (int i0 = tid - tid % 32; i0 < nh * (D / 4); i0 += THREADS) {
      const int idx = i0 + tid % 32;
      const bool act = idx < nh * (D / 4);
      const int h = act ? idx / (D / 4) : 0, l = idx % (D / 4);
      const float4 O = rotate_out4<D>(*reinterpret_cast<const float4*>(oscr + h * D + 4 * l), l, true);
      if (act)
        *reinterpret_cast<uint2*>(orow + h * D + 4 * l) =
            make_uint2(pack_h2(O.x, O.y), pack_h2(O.z, O.w));
    }
  }
}

// WIN: compiled for caches with a recent window (tails of up to R + G - 1
// tokens in a ring of R + G slots) and/or a sink window (the first S tokens
// in an fp16 area, folded in with the tail); the kernels without it keep
// the single-chunk-per-warp tail and its register budget.
// AK: position-adaptive key widths (KB = 4): a group whose width is 2 holds
// the 2-bit block at the start of its slot; only those bytes are copied.
template <int D, int KB, int VB, int G, bool PK, bool WIDE, bool WIN, bool AK = false>
__global__ void __launch_bounds__(DecCfg<D, KB, VB, G, WIDE>::THREADS,
                                  DecCfg<D, KB, VB, G, WIDE>::MIN_BLOCKS)
    decode_kernel(const Geom g, const WsLayout w, const DecodeArgs a) {
  using C = DecCfg<D, KB, VB, G, WIDE>;
  constexpr int NW = C::NW;
  static_assert(C::NST == 2, "the ring rotation below holds two stages");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int32_t wsum[NW];
  __shared__ int32_t claim;   // next unclaimed group of the current piece
  __shared__ int32_t ticket_flag[3];
  __shared__ Piece piece_s;   // the current piece, for the merge after the group loop
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint4* qsm = reinterpret_cast<uint4*>(smem + C::QA_OFF);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + C::SMEM_FIXED);
  int32_t* slen = prefix + (a.n_seq + 1);   // the sequences' lengths
  float* merge = reinterpret_cast<float*>(smem);   // reuses the ring between pieces

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, i4 = lane & 3;
  const int n_seq = a.n_seq;
  const int per_seq_units = g.hkv * g.slices;
  const int32_t* lens = reinterpret_cast<const int32_t*>(a.cache + g.lens_off) + a.seq0;
  int32_t* err = reinterpret_cast<int32_t*>(a.ws + w.err_off);
  float* partials = reinterpret_cast<float*>(a.ws + w.partials_off);

  // the combine kernel (a programmatic dependent of this grid) may be
  // scheduled now; it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // launched as a programmatic dependent of the previous kernel on the
  // stream (the append, typically): nothing it writes is read before this
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < C::NST; ++s) mbar_init(&bars[warp * C::NST + s], 1);
    if (warp == 0) mbar_init(&bars[NW * C::NST], 1);   // the query copy
    fence_mbar_init();
  }
  // ---- slot prefix over sequences: slots(b) = units(b) * (groups + has_tail)
  if (tid == 0) {
    prefix[0] = 0;
    claim = 0;
  }
  if (n_seq <= 32) {
    // one warp: a lane per sequence and a shuffle scan (no block barrier on
    // the way to the first copies)
    if (warp == 0) {
      const int L = lane < n_seq ? lens[lane] : 0;
      const int32_t run = per_seq_units * dec_unit_slots<G, WIN>(L, g);
      int32_t incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < n_seq) {
        prefix[lane + 1] = incl;
        slen[lane] = L;
      }
    }
  } else {
    const int chunk = (n_seq + C::THREADS - 1) / C::THREADS;
    const int b0 = tid * chunk, b1 = min(n_seq, b0 + chunk);
    int32_t run = 0;
    for (int bb = b0; bb < b1; ++bb) {
      const int L = lens[bb];
      run += per_seq_units * dec_unit_slots<G, WIN>(L, g);
    }
    // exclusive scan of the per-thread sums across the block
    int32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int32_t base = 0;
    for (int ww = 0; ww < warp; ++ww) base += wsum[ww];
    int32_t acc = base + incl - run;
    for (int bb = b0; bb < b1; ++bb) {
      const int L = lens[bb];
      acc += per_seq_units * dec_unit_slots<G, WIN>(L, g);
      prefix[bb + 1] = acc;
      slen[bb] = L;
    }
  }
  __syncthreads();

  // this CTA's slot range (the only 64-bit divisions of the kernel, once)
  const int T = prefix[n_seq];
  const int grid = gridDim.x;
  const int k = blockIdx.x;
  int start, end;
  cta_range(k, T, grid, &start, &end);
  if (start == end) {
    // an empty range (more CTAs than slots; the host never plans one, but a
    // captured decode replayed over shorter lengths can meet it): the split
    // record of a unit counts every CTA between its first and its last
    // slot, so publish an empty piece (m = -inf, l = 0) that the merge
    // skips, and, when split units are merged in the kernel, count it on
    // the ticket of the unit whose span it lies in (the unit holding slot
    // `start`, unless that slot is the unit's first)
    if (tid < kHeadsPerSlice &&
        debug_ok(w.partials_off + (int64_t)(2 * k + 1) * w.slot_floats * 4 <= w.total, err, 13)) {
      float* ps = partials + (int64_t)(2 * k) * w.slot_floats + tid * (D + 4);
      ps[D] = -INFINITY;
      ps[D + 1] = 0.f;
    }
    if (a.inline_merge && start < T) {
      const Piece p = make_piece<0, WIN>(g, prefix, slen, n_seq, start, start + 1);
      if (p.slot0 > 0)
        finish_split_unit<D, C::THREADS>(g, w, a, p.unit, (int64_t)start - p.slot0, p.wb, T,
                                         grid, p.b, p.hbase, p.nh, merge, C::MAX_MERGE_PIECES,
                                         ticket_flag, tid, g.rotate != 0,
                                         merge + C::RING / 4 - C::OSCR_FLOATS);
    }
  }

  // The warp's 2-stage ring: `head` is the stage consumed next, bit s of
  // `phase` the parity of stage s's next completion.
  int head = 0;
  uint32_t phase = 0;
  uint32_t qphase = 0;      // query copies so far (one per piece)
  bool ok = true;           // no wait has run out
  unsigned char* wring = smem + warp * C::NST * C::BLK;
  uint64_t* wbars = bars + warp * C::NST;
  uint64_t* qbar = bars + NW * C::NST;
  const unsigned char* blocks = a.cache + g.blocks_off;

  for (int pos = start; pos < end;) {
    WarpState<D, KB, VB, G, PK> st;
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) st.o[mt][0] = st.o[mt][1] = st.o[mt][2] = st.o[mt][3] = 0.f;
    st.z[0] = st.z[1] = st.z[2] = st.z[3] = 0.f;
#pragma unroll
    for (int r = 0; r < (PK ? 2 : 1); ++r) st.m[r] = -INFINITY;

    int ngr, nh;         // groups in this piece, heads of the unit
    int gs0, glen;       // the piece's first group in its sequence, the length
    int64_t gb;          // global block index of the piece's first group
    bool my_tail;        // this warp owns tail chunks warp, warp + TAIL_CHUNKS, ...
    {
      const Piece p = make_piece<G, WIN>(g, prefix, slen, n_seq, pos, end);
      if (tid == 0) piece_s = p;   // published by the barriers below
      gb = ((int64_t)(a.seq0 + p.b) * g.hkv + p.kvh) * g.max_groups + p.slot0;
      ngr = max(0, min(p.slot1, p.ng) - p.slot0);
      nh = p.nh;
      gs0 = p.slot0;
      glen = p.L;
      if constexpr (WIN)
        my_tail = ok && p.slot1 == p.wb && p.slot0 <= p.ng && warp < C::TAIL_CHUNKS &&
                  warp < fp16_chunks(g, p.L, p.Tb);
      else
        my_tail = ok && p.Tb > 0 && p.slot1 == p.wb && p.slot0 <= p.ng && warp * 16 < p.Tb;
      // the unit's raw query rows first, so that they are not queued behind
      // the group blocks
      if (tid == 0) {
        const int esz = a.q_dtype == KVQ_FP32 ? 4 : 2;
        const uint32_t qbytes = (uint32_t)(p.nh * D * esz);
        const unsigned char* q0 = static_cast<const unsigned char*>(a.q);
        fence_proxy_async_smem();
        checked_bulk_copy(qsm, q0 + ((int64_t)p.b * g.hq + p.hbase) * D * esz, qbytes, qbar, q0,
                          q0 + (int64_t)a.n_seq * g.hq * D * esz, err, 1);
      }
      if (my_tail) {
        const __half* tk = reinterpret_cast<const __half*>(
            a.cache + g.tails_off + ((int64_t)(a.seq0 + p.b) * g.hkv + p.kvh) * g.tail_bytes);
        unsigned char* tb = C::TAIL_EARLY ? smem + C::TAIL_OFF + warp * TailStage<D>::BYTES : wring;
        if constexpr (WIN) {
          const __half *ck, *cv;
          const int Tc = fp16_chunk_src<D, G>(g, a.cache, (int64_t)(a.seq0 + p.b) * g.hkv + p.kvh,
                                              p.L, p.ng, p.Tb, warp, ck, cv);
          if (debug_fp16_rows<D>(g, a.cache, ck, cv, Tc, 0, err))
            stage_tail_chunk<D>(tb, ck, cv, Tc, 0, lane);
        } else {
          if (debug_fp16_rows<D>(g, a.cache, tk, tk + G * D, p.Tb, warp, err))
            stage_tail_chunk<D>(tb, tk, tk + G * D, p.Tb, warp, lane);
        }
      }
    }
    // group c of the piece holds 2-bit keys (position-adaptive widths)
    auto narrow = [&](int c) -> bool {
      return AK && akvq_key_bits(gs0 + c, glen, G, g.akvq_delta) != KB;
    };
    // Claim a group (lane 0) and start its copy into stage `stg`; -1 once
    // the piece has none left.
    auto claim_into = [&](int stg) -> int {
      int gi = -1;
      if (lane == 0 && ok) {
        const int c = atomicAdd(&claim, 1);
        if (c < ngr) {
          gi = c;
          checked_bulk_copy(wring + stg * C::BLK, blocks + (gb + c) * C::BLK,
                            narrow(c) ? (uint32_t)g.a2_bytes : (uint32_t)C::BLK, &wbars[stg],
                            blocks, a.cache + g.tails_off, err, 2);
        }
      }
      return __shfl_sync(0xffffffffu, gi, 0);
    };
    // the ring's two items: cur in stage head, nxt in stage head ^ 1
    int cur = -1, nxt = -1;
    if (!(my_tail && !C::TAIL_EARLY)) {   // a ring that stages a tail starts later
      cur = claim_into(head);
      nxt = cur >= 0 ? claim_into(head ^ 1) : -1;
    }
    // while the blocks fly, the first warps turn the query rows into fragments
    {
      // converting warps: one per k-step of d/16
      constexpr int NCW = (NW < D / 16) ? NW : D / 16;
      if (warp < NCW) {
        bool got = mbar_wait_bounded(qbar, qphase & 1);
        got = __all_sync(0xffffffffu, got);
        if (!got && lane == 0) atomicExch(err, KVQ_ERR_DEVICE);
        const unsigned char* src = smem + C::QA_OFF;
        int sdt = a.q_dtype;
        if (g.rotate) {   // rotate the raw rows first (fp32), then convert those
          float* qr = reinterpret_cast<float*>(smem + C::QR_OFF);
          rotate_query_rows<D, NCW>(a.q_dtype, nh, got, warp, lane, src, qr);
          asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
          src = reinterpret_cast<const unsigned char*>(qr);
          sdt = KVQ_FP32;
        }
        convert_query<D, PK, NCW>(sdt, nh, got, warp, lane, qsm, src);
      }
    }
    ++qphase;
    __syncthreads();
    if (my_tail) {
      cp_async_wait_all();
      __syncwarp();
      unsigned char* tb = C::TAIL_EARLY ? smem + C::TAIL_OFF + warp * TailStage<D>::BYTES : wring;
      if constexpr (!WIN) {
        const Piece p = piece_s;
        if constexpr (PK) tail_chunk_pk<D, KB, VB, G>(st, tb, p.Tb, warp, qsm, lane);
        else tail_chunk<D, KB, VB, G>(st, tb, p.Tb, warp, qsm, lane);
      } else {
        // fp16 chunks warp, warp + TAIL_CHUNKS, ... (sink chunks first, then
        // the tail ring's), each staged once the previous one is done
        const Piece p = piece_s;
        const int64_t ui = (int64_t)(a.seq0 + p.b) * g.hkv + p.kvh;
        const int nck = fp16_chunks(g, p.L, p.Tb);
        for (int c = warp;;) {
          const __half *ck, *cv;
          const int Tc = fp16_chunk_src<D, G>(g, a.cache, ui, p.L, p.ng, p.Tb, c, ck, cv);
          if (c != warp) {
            __syncwarp();   // every lane's reads of the stage are done
            if (debug_fp16_rows<D>(g, a.cache, ck, cv, Tc, 0, err))
              stage_tail_chunk<D>(tb, ck, cv, Tc, 0, lane);
            cp_async_wait_all();
            __syncwarp();
          }
          if constexpr (PK) tail_chunk_pk<D, KB, VB, G>(st, tb, Tc, 0, qsm, lane);
          else tail_chunk<D, KB, VB, G>(st, tb, Tc, 0, qsm, lane);
          c += C::TAIL_CHUNKS;
          if (c >= nck) break;
        }
      }
      if (!C::TAIL_EARLY) {   // the ring is free again: start its copies
        __syncwarp();
        cur = claim_into(head);
        nxt = cur >= 0 ? claim_into(head ^ 1) : -1;
      }
    }
    while (cur >= 0) {
      // the claim for this stage's refill goes out now: its latency hides
      // behind the wait and the group's arithmetic
      int nc = -1;
      if (lane == 0 && nxt >= 0) nc = atomicAdd(&claim, 1);
      bool got = mbar_wait_bounded(&wbars[head], (phase >> head) & 1);
      got = __all_sync(0xffffffffu, got);
      if (!got) {
        ok = false;
        if (lane == 0) atomicExch(err, KVQ_ERR_DEVICE);
        break;
      }
      phase ^= 1u << head;
      if constexpr (AK) {
        if (narrow(cur)) {
          if constexpr (PK) process_group_pk<D, KB, VB, G, 2>(st, wring + head * C::BLK, qsm, lane);
          else process_group<D, KB, VB, G, 2>(st, wring + head * C::BLK, qsm, lane);
        } else {
          if constexpr (PK) process_group_pk<D, KB, VB, G>(st, wring + head * C::BLK, qsm, lane);
          else process_group<D, KB, VB, G>(st, wring + head * C::BLK, qsm, lane);
        }
      } else if constexpr (PK) {
        process_group_pk<D, KB, VB, G>(st, wring + head * C::BLK, qsm, lane);
      } else {
        process_group<D, KB, VB, G>(st, wring + head * C::BLK, qsm, lane);
      }
      __syncwarp();
      // refill the stage: the warp's reads of it are complete (their values
      // were consumed before __syncwarp), and a bulk copy that overwrites
      // bytes which were only read needs no proxy fence.  Claims come in
      // increasing order, so once one fails every later one does.
      int nn = -1;
      if (lane == 0 && nc >= 0 && nc < ngr) {
        nn = nc;
        checked_bulk_copy(wring + head * C::BLK, blocks + (gb + nc) * C::BLK,
                          narrow(nc) ? (uint32_t)g.a2_bytes : (uint32_t)C::BLK, &wbars[head],
                          blocks, a.cache + g.tails_off, err, 3);
      }
      nn = __shfl_sync(0xffffffffu, nn, 0);
      cur = nxt;
      nxt = nn;
      head ^= 1;
    }

    // ---- merge the NW warps (the rings are idle: every issued copy was
    // waited on, except after a failed wait)
    fence_proxy_async_smem();
    __syncthreads();
    // the piece again (from shared memory rather than kept through the loop)
    const Piece p = piece_s;
    const int b = p.b, slot0 = p.slot0, slot1 = p.slot1, wb = p.wb, unit = p.unit;
    const int hbase = p.hbase;
    if (tid == 0) claim = 0;   // for the next piece (published by the barriers below)
    {
      constexpr int RS = C::MRS;
      float* mo = merge + (warp * kHeadsPerSlice) * RS;
      // value-min terms for channel group j and heads 2*i4, 2*i4+1 live in
      // lane 4j + i4; the denominators in lane 4J + i4
      float zl0[C::J], zl1[C::J];
#pragma unroll
      for (int j = 0; j < C::J; ++j) {
        zl0[j] = __shfl_sync(0xffffffffu, st.z[0], 4 * j + i4);
        zl1[j] = __shfl_sync(0xffffffffu, st.z[1], 4 * j + i4);
      }
      const float l0 = __shfl_sync(0xffffffffu, st.z[0], 4 * C::J + i4);
      const float l1 = __shfl_sync(0xffffffffu, st.z[1], 4 * C::J + i4);
      if constexpr (PK) {
        // columns 4-7 repeat heads 0-3 bit for bit (the same B columns and
        // rescale factors), so lanes i4 >= 2 store the channel + 8 half of
        // lane i4 - 2's heads: every lane stores two values per m-tile.
        const int hh = 2 * (i4 & 1);
        const int co = (i4 >= 2) ? 8 : 0;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          const int c = 16 * mt + g8 + co;
          const int j = (16 * mt) / G;
          const float o0 = (i4 >= 2) ? st.o[mt][2] : st.o[mt][0];
          const float o1 = (i4 >= 2) ? st.o[mt][3] : st.o[mt][1];
          mo[hh * RS + c] = o0 + zl0[j];
          mo[(hh + 1) * RS + c] = o1 + zl1[j];
        }
        if (g8 == 0 && i4 < 2) {
          mo[(2 * i4) * RS + D] = st.m[0];
          mo[(2 * i4 + 1) * RS + D] = st.m[1];
        }
      } else {
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          const int c0 = 16 * mt + g8, c1 = c0 + 8;
          const int j = (16 * mt) / G;
          mo[(2 * i4) * RS + c0] = st.o[mt][0] + zl0[j];
          mo[(2 * i4 + 1) * RS + c0] = st.o[mt][1] + zl1[j];
          mo[(2 * i4) * RS + c1] = st.o[mt][2] + zl0[j];
          mo[(2 * i4 + 1) * RS + c1] = st.o[mt][3] + zl1[j];
        }
        if (i4 == 0) mo[g8 * RS + D] = st.m[0];
      }
      if (g8 == 0) {
        mo[(2 * i4) * RS + D + 1] = l0;
        mo[(2 * i4 + 1) * RS + D + 1] = l1;
      }
    }
    __syncthreads();

    const bool whole = (slot0 == 0 && slot1 == wb);
    // [h][NW] weights of the warps' shares, then [h] max and [h] sum
    float* wts = merge + C::WTS_OFF;
    merge_weights<D, NW, C::MRS>(merge, wts, whole, tid);
    // Partial slots: a CTA holds at most two split pieces, its first (slot
    // 2k) and its last (2k + 1); pieces in between are whole units.
    const int myslot = piece_partial_slot(k, pos, start);
    if (slot0 == 0 && tid == 0) {
      // split record of the unit for the combine kernel: its first partial
      // slot and the number of CTAs holding a piece of it
      const int kl = cta_of_slot((int64_t)pos + wb - 1, T, grid);   // the unit's last slot
      if (debug_ok(unit >= 0 && unit < w.units, err, 7))
        *reinterpret_cast<int2*>(a.ws + w.units_off + 8LL * unit) = make_int2(myslot, kl - k + 1);
    }
    const bool slot_ok =
        whole || debug_ok(myslot < 2 * grid &&
                              w.partials_off + (int64_t)(myslot + 1) * w.slot_floats * 4 <= w.total,
                          err, 6);
    const bool out_ok = debug_ok(b < a.n_seq && hbase + nh <= g.hq, err, 8);
    __syncthreads();
    // four channels per thread: 128-bit loads of the warps' rows, 128-bit
    // partial stores (rows of D + 8 floats and partial rows of D + 4 keep
    // every such address 16-byte aligned)
    static_assert(C::MRS % 4 == 0 && (D + 4) % 4 == 0, "16-byte aligned merge rows");
    const bool rot_out = whole && g.rotate != 0;   // final rows of a rotating cache
    for (int i0 = tid - lane; i0 < nh * (D / 4); i0 += C::THREADS) {
      const int idx = i0 + lane;
      const bool act = idx < nh * (D / 4);
      const int h = act ? idx / (D / 4) : 0, c = 4 * (idx % (D / 4));
      const float* f = wts + h * NW;
      const float* mo = merge + h * C::MRS + c;
      constexpr int WS = kHeadsPerSlice * C::MRS;   // stride between the warps' areas
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) {
        const float fw = f[ww];
        const float4 x = *reinterpret_cast<const float4*>(mo + ww * WS);
        O.x = fmaf(fw, x.x, O.x);
        O.y = fmaf(fw, x.y, O.y);
        O.z = fmaf(fw, x.z, O.z);
        O.w = fmaf(fw, x.w, O.w);
      }
      O = rotate_out4<D>(O, idx % (D / 4), rot_out);
      if (!act) continue;
      if (whole) {
        const uint2 hv = make_uint2(pack_h2(O.x, O.y), pack_h2(O.z, O.w));
        if (out_ok)
          *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(a.out) +
                                    ((int64_t)b * g.hq + hbase + h) * D + c) = hv;
      } else if (slot_ok) {
        float* ps = partials + myslot * w.slot_floats + h * (D + 4);
        *reinterpret_cast<float4*>(ps + c) = O;
        if (c == 0) {
          ps[D] = wts[NW * kHeadsPerSlice + h];
          ps[D + 1] = wts[(NW + 1) * kHeadsPerSlice + h];
        }
      }
    }
    if (!whole && a.inline_merge)
      finish_split_unit<D, C::THREADS>(g, w, a, unit, (int64_t)pos - slot0, wb, T, grid, b, hbase,
                                       nh, merge, C::MAX_MERGE_PIECES, ticket_flag, tid,
                                       g.rotate != 0, merge + C::RING / 4 - C::OSCR_FLOATS);
    fence_proxy_async_smem();   // generic accesses before the next bulk copies
    __syncthreads();            // merge area and ctl are reused by the next piece
    pos += slot1 - slot0;
  }
}

// Merges the pieces of every unit that the decode kernel split across CTAs;
// units held by one CTA were written by the decode kernel itself.  Runs as a
// programmatic dependent launch of the decode grid and waits for it before
// touching the partials.  An item is (unit, head of its slice); `wpi` warps
// of a 256-thread block share an item and stride over its pieces, 4 pieces
// in flight per warp, each lane holding D/32 channels (one 16- or 8-byte
// load per piece).  The launch picks wpi from the expected pieces per unit.
constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const Geom g, const WsLayout w,
                                                                  const DecodeArgs a, int wpi,
                                                                  int heads, int n_items) {
  constexpr int CPL = D / 32;   // channels per lane
  __shared__ __align__(16) float red[kCombineWarps][D + 4];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * (kCombineWarps / wpi) + warp / wpi;
  const int wi = warp % wpi;
  const int unit = item / heads, h = item % heads;
  bool active = item < n_items;
  int npc = 0, sl0 = 0;
  if (active) {
    const int2 rec = *reinterpret_cast<const int2*>(a.ws + w.units_off + 8LL * unit);
    sl0 = rec.x;
    npc = rec.y;
  }
  const int per_seq = g.hkv * g.slices;
  const int b = unit / per_seq, uis = unit % per_seq;
  const int kvh = uis / g.slices, slice = uis % g.slices;
  const int nh = min(kHeadsPerSlice, g.gqa - slice * kHeadsPerSlice);
  active = active && npc > 1 && h < nh;
  const int kf = sl0 / 2;
  // debug builds: the record's pieces and the output row must fit (checks 12, 8)
  if (active && kDebug) {
    int32_t* err = reinterpret_cast<int32_t*>(a.ws + w.err_off);
    active = debug_ok(sl0 >= 0 && w.partials_off + (int64_t)(merge_piece_slot(kf, sl0, npc - 1) + 1) *
                                                        w.slot_floats * 4 <= w.total,
                      err, 12) &&
             debug_ok(b < a.n_seq, err, 8);
  }
  const float* part = reinterpret_cast<const float*>(a.ws + w.partials_off) + h * (D + 4);
  auto piece = [&](int pc) { return part + (int64_t)merge_piece_slot(kf, sl0, pc) * w.slot_floats; };

  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
  float lsum = 0.f;
  if (active) {
    float M = -INFINITY;
    for (int pc = lane; pc < npc; pc += 32) M = fmaxf(M, __ldcg(piece(pc) + D));
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    for (int p0 = wi; p0 < npc; p0 += 4 * wpi) {
      float2 ml[4];
      float ov[4][CPL];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int pc = p0 + u * wpi;
        ml[u] = make_float2(-INFINITY, 0.f);
#pragma unroll
        for (int c = 0; c < CPL; ++c) ov[u][c] = 0.f;
        if (pc < npc) {
          const float* ps = piece(pc);
          ml[u] = __ldcg(reinterpret_cast<const float2*>(ps + D));
          if constexpr (CPL == 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(ps) + lane);
            ov[u][0] = v.x; ov[u][1] = v.y; ov[u][2] = v.z; ov[u][3] = v.w;
          } else {
            const float2 v = __ldcg(reinterpret_cast<const float2*>(ps) + lane);
            ov[u][0] = v.x; ov[u][1] = v.y;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (ml[u].x != -INFINITY) {   // an empty piece contributes nothing
          const float wk = fast_exp2(ml[u].x - M);
          lsum += wk * ml[u].y;
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[c] += wk * ov[u][c];
        }
      }
    }
  }
  if (wpi > 1) {   // uniform over the block
#pragma unroll
    for (int c = 0; c < CPL; ++c) red[warp][lane * CPL + c] = acc[c];
    if (lane == 0) red[warp][D] = lsum;
    __syncthreads();
    if (wi == 0 && active) {
      for (int ww = 1; ww < wpi; ++ww) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] += red[warp + ww][lane * CPL + c];
        lsum += red[warp + ww][D];
      }
    }
  }
  if (wi == 0 && active) {
    const float inv = 1.0f / lsum;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] *= inv;
    if (g.rotate) {   // rotating cache: the head's row rotated back (one warp)
      fwht_lanes<D, CPL>(acc, lane);
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc[c] *= rot_scale<D>();
    }
    const int hbase = kvh * g.gqa + slice * kHeadsPerSlice;
    __half* o = reinterpret_cast<__half*>(a.out) + ((int64_t)b * g.hq + hbase + h) * D + lane * CPL;
    if constexpr (CPL == 4) {
      *reinterpret_cast<uint2*>(o) = make_uint2(pack_h2(acc[0], acc[1]), pack_h2(acc[2], acc[3]));
    } else {
      *reinterpret_cast<uint32_t*>(o) = pack_h2(acc[0], acc[1]);
    }
  }
}

template <int D, int KB, int VB, int G, bool WIDE>
size_t smem_bytes(int n_seq) {   // + slot prefix and lengths of the sequences
  return DecCfg<D, KB, VB, G, WIDE>::SMEM_FIXED + 4 * (size_t)(2 * n_seq + 1);
}

// The position-adaptive variant exists for 4-bit keys.
template <int KB, bool PK>
constexpr bool has_ak() {
  return KB == 4;
}

template <int D, int KB, int VB, int G, bool PK, bool WIDE>
cudaError_t max_ctas_t(bool ak, int* out) {
  using C = DecCfg<D, KB, VB, G, WIDE>;
  const size_t sm = smem_bytes<D, KB, VB, G, WIDE>(64);
  // residency of the kernels with and without a recent window (the same
  // launch bounds and shared memory: normally equal), the smaller one; of
  // the position-adaptive one alone when the cache uses it
  using K = decltype(&decode_kernel<D, KB, VB, G, PK, WIDE, false>);
  K kerns[2] = {decode_kernel<D, KB, VB, G, PK, WIDE, false>,
                decode_kernel<D, KB, VB, G, PK, WIDE, true>};
  int nk = 2;
  if (ak) {
    if constexpr (has_ak<KB, PK>()) {
      kerns[0] = decode_kernel<D, KB, VB, G, PK, WIDE, false, true>;
      nk = 1;
    } else {
      return cudaErrorInvalidValue;
    }
  }
  int per_sm = 1 << 30;
  for (int ki = 0; ki < nk; ++ki) {
    const K kern = kerns[ki];
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes<D, KB, VB, G, WIDE>(kSeqsPerLaunch));
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, C::THREADS, sm);
    if (e != cudaSuccess) return e;
    per_sm = min(per_sm, n);
  }
  cudaError_t e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  *out = max(1, min(kMaxDecodeCtas, per_sm * sms));
  return cudaSuccess;
}

template <int D, int KB, int VB, int G, bool PK, bool WIDE>
cudaError_t launch_t(const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid,
                     cudaStream_t stream) {
  using C = DecCfg<D, KB, VB, G, WIDE>;
  if (g.block_bytes != C::BLK || g.sec_vmin != C::SEC_VMIN || g.sec_kscale != C::SEC_KSCALE)
    return cudaErrorInvalidValue;
  const bool win = g.window > 0 || g.sink > 0;
  const bool ak = g.akvq_delta > 0;
  auto kern = win ? decode_kernel<D, KB, VB, G, PK, WIDE, true>
                  : decode_kernel<D, KB, VB, G, PK, WIDE, false>;
  if (ak) {
    if constexpr (has_ak<KB, PK>()) {
      if (win) return cudaErrorInvalidValue;
      kern = decode_kernel<D, KB, VB, G, PK, WIDE, false, true>;
    } else {
      return cudaErrorInvalidValue;
    }
  }
  const int variant = ak ? 2 : (int)win;
  const size_t sm = smem_bytes<D, KB, VB, G, WIDE>(a.n_seq);
  static bool configured[3] = {false, false, false};   // attribute set once, before any capture
  if (!configured[variant]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes<D, KB, VB, G, WIDE>(kSeqsPerLaunch));
    if (e != cudaSuccess) return e;
    configured[variant] = true;
  }
  {
    // a programmatic dependent of the previous kernel (it waits for it
    // before reading anything): its launch overlaps the append's tail
    cudaLaunchConfig_t dc = {};
    dc.gridDim = dim3((unsigned)grid);
    dc.blockDim = dim3(C::THREADS);
    dc.dynamicSmemBytes = sm;
    dc.stream = stream;
    cudaLaunchAttribute da[1];
    da[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    da[0].val.programmaticStreamSerializationAllowed = 1;
    dc.attrs = da;
    dc.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&dc, kern, g, w, a);
    if (e != cudaSuccess) return e;
  }
  if (a.inline_merge) return cudaSuccess;   // split units merged in the kernel
  // the combine kernel, a programmatic dependent of the decode grid; warps
  // per item from the expected pieces of a split unit (grid / units + 1)
  const int units = a.n_seq * g.hkv * g.slices;
  const int npc_est = grid / units + 1;
  const int wpi = npc_est <= 4 ? 1 : npc_est <= 8 ? 2 : npc_est <= 16 ? 4 : 8;
  const int heads = g.gqa < kHeadsPerSlice ? g.gqa : kHeadsPerSlice;
  const int n_items = units * heads;
  const int ipb = kCombineWarps / wpi;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)((n_items + ipb - 1) / ipb));
  lc.blockDim = dim3(kCombineThreads);
  lc.dynamicSmemBytes = 0;
  lc.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, combine_kernel<D>, g, w, a, wpi, heads, n_items);
}

}  // namespace

// One instantiation per (head dim, key bits, value bits, group), per layout
// (packed when the GQA group has at most 4 heads) and per CTA width; the
// entry points are declared in kvq_internal.h (KVQ_DECODE_DECLARE).
#define KVQ_DECODE_DEFINE(D_, KB_, VB_, G_)                                               \
  cudaError_t decode_max_ctas_##D_##_##KB_##_##VB_##_##G_(const Geom& g, bool wide,       \
                                                          int* out) {                     \
    const bool ak = g.akvq_delta > 0;                                                     \
    return g.gqa <= 4 ? (wide ? max_ctas_t<D_, KB_, VB_, G_, true, true>(ak, out)         \
                              : max_ctas_t<D_, KB_, VB_, G_, true, false>(ak, out))       \
                      : (wide ? max_ctas_t<D_, KB_, VB_, G_, false, true>(ak, out)        \
                              : max_ctas_t<D_, KB_, VB_, G_, false, false>(ak, out));     \
  }                                                                                       \
  cudaError_t launch_decode_##D_##_##KB_##_##VB_##_##G_(                                  \
      const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid, bool wide,         \
      cudaStream_t stream) {                                                              \
    return g.gqa <= 4                                                                     \
               ? (wide ? launch_t<D_, KB_, VB_, G_, true, true>(g, w, a, grid, stream)    \
                       : launch_t<D_, KB_, VB_, G_, true, false>(g, w, a, grid, stream))  \
               : (wide ? launch_t<D_, KB_, VB_, G_, false, true>(g, w, a, grid, stream)   \
                       : launch_t<D_, KB_, VB_, G_, false, false>(g, w, a, grid, stream)); \
  }

}  // namespace kvq
