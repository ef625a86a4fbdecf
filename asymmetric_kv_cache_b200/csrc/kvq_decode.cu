// Split-K decode attention over the quantized cache (libkvq, sm_100a).
//
// out_h = sum_t alpha_t v_hat_t, alpha = softmax(q_h . k_hat_t / sqrt(d))
// ("Asymmetric Key-Value Quantization: 2-Bit Values and 4-Bit Keys under
// Long-Context Drift", §1, §2.1) over the dequantized groups and the fp16
// tail of each sequence.  Decode is bound by reading the cache ("WUSH-KV"
// page, NOVA-KV abstract: loading the cache takes longer than the attention
// arithmetic), so the kernel is built around moving packed codes at HBM
// speed and doing the dequantization in registers.
//
// Work decomposition.  A unit is (sequence, kv head, slice of <= 8 query
// heads).  A unit's work is a row of slots: one per key group plus one for
// the fp16 tail.  All units' slots form one sequence that is cut into
// `gridDim.x` equal ranges, one per CTA (a stream-K split: every CTA gets the
// same number of slots whatever the lengths are).  Inside a CTA the 4 warps
// take the slots of each unit round-robin, each with its own online softmax,
// and merge through shared memory at the end of the unit's piece.  A unit
// cut by CTA boundaries writes per-piece partials (m, l, o); the last CTA to
// finish it (atomic ticket, no waiting) merges them and writes the output.
//
// Per group (one 32/64-token slot) a warp:
//   * waits for the group block, brought into its own shared-memory ring by
//     a 1-D bulk (TMA) copy issued NST groups ahead;
//   * folds the per-channel key scales into the query: q'_c = q_c s_c, so
//     q . k_hat = sum_c q'_c code_c + sum_c q_c z_c; the second sum (one per
//     group and head) runs on the tensor core with q split into fp16 high and
//     low halves (rows 0-7 and 8-15 of the tile) against the key mins;
//   * unpacks key codes to exact fp16 pairs and runs S^T = codes q'^T on
//     m16n8k16 tiles (rows = 16 tokens, columns = the 8 query heads of the
//     GQA group), so each lane's softmax state covers two heads;
//   * updates the running max / rescales, exponentiates (exp2 domain) and
//     transposes the fp16 P tile in registers (movmatrix);
//   * runs O^T += V_code^T (p s_v) on tiles whose rows are channels and whose
//     columns are heads, with the per-token value scale folded into p for
//     each channel group, and sum_t p_t z_t (value mins) and sum_t p_t (the
//     softmax denominator) on one more tile.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int KB, int VB, int G>
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
  static constexpr int NST = (BLK <= 4096) ? 3 : 2;   // ring stages per warp
  // resident CTAs per SM the register budget aims at (shared memory allows
  // four CTAs with 3-stage rings of blocks up to 4 KB, three otherwise)
  static constexpr int MIN_BLOCKS = (BLK <= 4096) ? 4 : 3;
  static constexpr int RING = kWarps * NST * BLK;
  // query fragments of the current unit, shared by the CTA's warps:
  // [kt][lane][4 words] = {hi v0, lo v0, hi v1, lo v1}
  static constexpr int QA_OFF = RING;
  static constexpr int QA_BYTES = KT * 32 * 16;
  // both parts divided by the key code multiplier m of their register,
  // [kt][lane][4 words] (the B operand of q.k is (q_hi/m + q_lo/m) * s_k)
  static constexpr int QM_OFF = QA_OFF + QA_BYTES;
  static constexpr int QM_BYTES = KT * 32 * 16;
  static constexpr int MERGE_FLOATS = kWarps * kHeadsPerSlice * (D + 2);
  static_assert(MERGE_FLOATS * 4 <= RING, "merge area must fit in the ring");
  static constexpr int BAR_OFF = QM_OFF + QM_BYTES;
  static constexpr int SMEM_FIXED = BAR_OFF + kWarps * NST * 8 + 64;
};

template <int D, int KB, int VB, int G>
struct WarpState {
  float o[D / 16][4];   // O^T: (channel 16mt + g, heads 2i, 2i+1), then channel + 8
  float z[4];           // rows: value-min terms (j < J) and sum p (row J); cols heads
  float m[2];           // running max of heads 2i, 2i+1 (i = lane & 3), log2 domain
};

// Query fragments of head g = lane/4 (zeros for a padding head), channels
// 16kt + 2i + {0,1} (v = 0) and + 8 (v = 1), i = lane & 3: q is scaled by
// log2(e)/sqrt(d), split into fp16 high and low parts and stored per lane
// as qs[kt * 32 + lane] = {hi v0, lo v0, hi v1, lo v1} - the A quad of the
// key-min tile (rows g: high part, rows g + 8: low part).
template <int D, int KB>
__device__ __forceinline__ void load_query(const void* q, int dtype, int64_t row, bool valid,
                                           int lane, uint4* __restrict__ qs,
                                           uint4* __restrict__ qm) {
  const int i4 = lane & 3;
  const float sc = kLog2e * rsqrtf((float)D);
  float2 x[D / 16][2];
#pragma unroll
  for (int kt = 0; kt < D / 16; ++kt) {
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int64_t idx = row * D + 16 * kt + 8 * v + 2 * i4;
      float2 f = make_float2(0.f, 0.f);
      if (valid) {
        if (dtype == KVQ_FP16) {
          f = __half22float2(*reinterpret_cast<const __half2*>(reinterpret_cast<const __half*>(q) + idx));
        } else if (dtype == KVQ_BF16) {
          f = __bfloat1622float2(
              *reinterpret_cast<const __nv_bfloat162*>(reinterpret_cast<const __nv_bfloat16*>(q) + idx));
        } else {
          f = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(q) + idx);
        }
      }
      x[kt][v] = f;
    }
  }
  static_for<D / 16>([&](auto kt_) {
    constexpr int kt = decltype(kt_)::value;
    uint32_t w[4];
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const float x0 = x[kt][v].x * sc, x1 = x[kt][v].y * sc;
      const __half2 h = __floats2half2_rn(x0, x1);
      const float2 hf = __half22float2(h);
      w[2 * v] = h2_as_u32(h);
      w[2 * v + 1] = pack_h2(x0 - hf.x, x1 - hf.y);
    }
    qs[kt * 32 + lane] = make_uint4(w[0], w[1], w[2], w[3]);
    constexpr int FK = 16 / KB;
    constexpr int e0 = code_log2_mul<KB, (2 * kt) % FK>();
    constexpr int e1 = code_log2_mul<KB, (2 * kt + 1) % FK>();
    qm[kt * 32 + lane] = make_uint4(hmul2_b(w[0], h2_pow2_neg(e0)), hmul2_b(w[1], h2_pow2_neg(e0)),
                                    hmul2_b(w[2], h2_pow2_neg(e1)), hmul2_b(w[3], h2_pow2_neg(e1)));
  });
}

// Online-softmax update for new logits in the transposed tile layout:
// s[mt] = {(token g, head 2i), (token g, head 2i+1), (token g+8, head 2i),
// (token g+8, head 2i+1)} of a 16-token tile mt (g = lane/4, i = lane&3).
// Produces the fp16 probabilities as B fragments of the p.v tile
// (pt[mt] = {tokens 0-7, tokens 8-15} of head g, 2 tokens per lane).
template <int D, int NM, int KB, int VB, int G>
__device__ __forceinline__ void softmax_update(WarpState<D, KB, VB, G>& st, float (&s)[NM][4],
                                               uint32_t (&pt)[NM][2]) {
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int mt = 0; mt < NM; ++mt) {
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

// One quantized group from the shared-memory stage `sp`.
//
// Key codes enter the tensor core as x = 1024 + m*code (code_offset) against
// B = (q/m) * s_k, carried as an fp16 high + low pair (one fp16 rounding of
// the product would cost ~2^-12 of each logit term, which matters for
// channels with large scales); the offset is removed with tiles against a
// constant 1024 operand, which sum exactly the fp16 B values the tensor core
// saw.  Value
// codes are unpacked to exact fp16 integers (unpack_pair).
template <int D, int KB, int VB, int G>
__device__ __forceinline__ void process_group(WarpState<D, KB, VB, G>& st,
                                              const unsigned char* __restrict__ sp,
                                              const uint4* __restrict__ qsm,
                                              const uint4* __restrict__ qmsm, int lane) {
  using C = DecCfg<D, KB, VB, G>;
  constexpr int NM = G / 16;
  const int g8 = lane >> 2, i4 = lane & 3;

  // B = (q s_k) / m as an fp16 high + low pair, the key-min term and the
  // offset correction
  uint32_t qs[C::KT][2], ql[C::KT][2];
  float bias[4] = {0.f, 0.f, 0.f, 0.f};
  float kcor[4] = {0.f, 0.f, 0.f, 0.f};
  {
    uint32_t ksw[D / 8], kzw[D / 8];
    lds_words<D / 8>(reinterpret_cast<const uint32_t*>(sp + C::SEC_KSCALE) + i4 * (D / 8), ksw);
    lds_words<D / 8>(reinterpret_cast<const uint32_t*>(sp + C::SEC_KMIN) + i4 * (D / 8), kzw);
    static_for<C::KT>([&](auto kt_) {
      constexpr int kt = decltype(kt_)::value;
      const uint4 q4 = qsm[kt * 32 + lane];
      const uint4 qm = qmsm[kt * 32 + lane];
      // high part: one rounding of hi*s + lo*s; low part: the rest of it,
      // (hi*s - high) exact in one fused step, plus lo*s
      const uint32_t s0 = ksw[2 * kt], s1 = ksw[2 * kt + 1];
      qs[kt][0] = hfma2_b(qm.x, s0, hmul2_b(qm.y, s0));
      qs[kt][1] = hfma2_b(qm.z, s1, hmul2_b(qm.w, s1));
      ql[kt][0] = hfma2_b(qm.y, s0, hfma2_b(qm.x, s0, qs[kt][0] ^ 0x80008000u));
      ql[kt][1] = hfma2_b(qm.w, s1, hfma2_b(qm.z, s1, qs[kt][1] ^ 0x80008000u));
      mma16816(bias, q4.x, q4.y, q4.z, q4.w, kzw[2 * kt], kzw[2 * kt + 1]);
      mma16816(kcor, kH2One024, kH2One024, kH2One024, kH2One024, qs[kt][0], qs[kt][1]);
      mma16816(kcor, kH2One024, kH2One024, kH2One024, kH2One024, ql[kt][0], ql[kt][1]);
    });
  }
  // bias of head g8 is in every lane of quad g8; fetch heads 2*i4 and 2*i4+1
  const float bg = bias[0] + bias[2];
  const float b0 = __shfl_sync(0xffffffffu, bg, 8 * i4) - kcor[0];
  const float b1 = __shfl_sync(0xffffffffu, bg, 8 * i4 + 4) - kcor[1];

  // S^T = codes q'^T: rows = tokens (two 8-token code tiles), cols = heads
  float s[NM][4];
  const uint32_t* kcw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KCODES);
  static_for<NM>([&](auto mt_) {
    constexpr int mt = decltype(mt_)::value;
    uint32_t kw0[C::LWK], kw1[C::LWK];
    lds_words<C::LWK>(kcw + ((2 * mt) * 32 + lane) * C::LWK, kw0);
    lds_words<C::LWK>(kcw + ((2 * mt + 1) * 32 + lane) * C::LWK, kw1);
    float acc[4] = {b0, b1, b0, b1};
    static_for<C::KT>([&](auto kt_) {
      constexpr int kt = decltype(kt_)::value;
      constexpr int p0 = 2 * kt, p1 = 2 * kt + 1;
      const uint32_t a0 = code_offset<KB, p0 % C::FK>(kw0[p0 / C::FK]);   // token g
      const uint32_t a1 = code_offset<KB, p0 % C::FK>(kw1[p0 / C::FK]);   // token g + 8
      const uint32_t a2 = code_offset<KB, p1 % C::FK>(kw0[p1 / C::FK]);   // channels + 8
      const uint32_t a3 = code_offset<KB, p1 % C::FK>(kw1[p1 / C::FK]);
      mma16816(acc, a0, a1, a2, a3, qs[kt][0], qs[kt][1]);
      mma16816(acc, a0, a1, a2, a3, ql[kt][0], ql[kt][1]);
    });
    s[mt][0] = acc[0];
    s[mt][1] = acc[1];
    s[mt][2] = acc[2];
    s[mt][3] = acc[3];
  });

  uint32_t pt[NM][2];
  softmax_update<D, NM, KB, VB, G>(st, s, pt);

  // O^T += V^T (p * s_v); Z += [z_v; 1]^T p
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

// The fp16 tail (T tokens, 0 < T < G) of one (sequence, kv head), staged
// 16 tokens at a time through the warp's (idle) ring with cp.async: key rows
// and value token-pair rows, padded so that the fragment reads below are
// free of bank conflicts; rows past T are zero-filled.
template <int D>
struct TailStage {
  static constexpr int KROW = 2 * D + 16;       // bytes per padded key row
  static constexpr int VROW = 4 * D + 16;       // bytes per padded value pair-row
  static constexpr int VOFF = 16 * KROW;
  static constexpr int BYTES = VOFF + 8 * VROW;
};

template <int D, int KB, int VB, int G>
__device__ __forceinline__ void process_tail(WarpState<D, KB, VB, G>& st,
                                             const __half* __restrict__ tk,
                                             const __half* __restrict__ tv, int T,
                                             const uint4* __restrict__ qsm, int lane,
                                             unsigned char* __restrict__ buf) {
  using C = DecCfg<D, KB, VB, G>;
  using TS = TailStage<D>;
  static_assert(TS::BYTES <= C::NST * C::BLK, "tail chunk must fit in a warp's ring");
  const int g8 = lane >> 2, i4 = lane & 3;
  for (int kv = 0; kv * 16 < T; ++kv) {
    // stage 16 key rows and 8 value pair-rows (16-byte pieces)
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
    cp_async_wait_all();
    __syncwarp();

    // S^T = K q^T with q = high + low parts (two products per tile)
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const unsigned char* k0 = buf + g8 * TS::KROW + 4 * i4;
    const unsigned char* k1 = k0 + 8 * TS::KROW;
#pragma unroll
    for (int kt = 0; kt < C::KT; ++kt) {
      const uint32_t a0 = *reinterpret_cast<const uint32_t*>(k0 + 32 * kt);
      const uint32_t a1 = *reinterpret_cast<const uint32_t*>(k1 + 32 * kt);
      const uint32_t a2 = *reinterpret_cast<const uint32_t*>(k0 + 32 * kt + 16);
      const uint32_t a3 = *reinterpret_cast<const uint32_t*>(k1 + 32 * kt + 16);
      const uint4 q4 = qsm[kt * 32 + lane];
      mma16816(acc, a0, a1, a2, a3, q4.x, q4.z);
      mma16816(acc, a0, a1, a2, a3, q4.y, q4.w);
    }
    const int t0 = 16 * kv + g8, t1 = t0 + 8;
    float s[1][4];
    s[0][0] = (t0 < T) ? acc[0] : -INFINITY;
    s[0][1] = (t0 < T) ? acc[1] : -INFINITY;
    s[0][2] = (t1 < T) ? acc[2] : -INFINITY;
    s[0][3] = (t1 < T) ? acc[3] : -INFINITY;
    uint32_t pt[1][2];
    softmax_update<D, 1, KB, VB, G>(st, s, pt);
    const uint32_t ones = (g8 == C::J) ? 0x3C003C00u : 0u;
    mma16816(st.z, ones, 0u, ones, 0u, pt[0][0], pt[0][1]);
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
      mma16816(st.o[mt], a0, a1, a2, a3, pt[0][0], pt[0][1]);
    }
    __syncwarp();   // every lane is done with this chunk before the next copy
  }
}

// Largest b in [0, n) with prefix[b] <= pos (prefix[0] = 0, increasing).
__device__ __forceinline__ int find_seq(const int32_t* prefix, int n, int pos) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid + 1] <= pos) lo = mid + 1; else hi = mid;
  }
  return lo;
}

template <int D, int KB, int VB, int G>
__global__ void __launch_bounds__(kThreads, (DecCfg<D, KB, VB, G>::MIN_BLOCKS))
    decode_kernel(const Geom g, const WsLayout w, const DecodeArgs a) {
  using C = DecCfg<D, KB, VB, G>;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint4* qsm = reinterpret_cast<uint4*>(smem + C::QA_OFF);
  uint4* qmsm = reinterpret_cast<uint4*>(smem + C::QM_OFF);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + C::SMEM_FIXED);
  float* merge = reinterpret_cast<float*>(smem);   // reuses the ring between pieces

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, i4 = lane & 3;
  const int n_seq = a.n_seq;
  const int per_seq_units = g.hkv * g.slices;
  const int32_t* lens = reinterpret_cast<const int32_t*>(a.cache + g.lens_off);
  int32_t* err = reinterpret_cast<int32_t*>(a.ws + w.err_off);
  float* partials = reinterpret_cast<float*>(a.ws + w.partials_off);

  // the combine kernel (a programmatic dependent of this grid) may be
  // scheduled now; it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < C::NST; ++s) mbar_init(&bars[warp * C::NST + s], 1);
    fence_mbar_init();
  }
  // ---- slot prefix over sequences: slots(b) = units(b) * (groups + has_tail)
  if (tid == 0) prefix[0] = 0;
  {
    const int chunk = (n_seq + kThreads - 1) / kThreads;
    const int b0 = tid * chunk, b1 = min(n_seq, b0 + chunk);
    int32_t run = 0;
    for (int bb = b0; bb < b1; ++bb) {
      const int L = lens[bb];
      run += per_seq_units * (L / G + (L % G ? 1 : 0));
    }
    // exclusive scan of the per-thread sums across the block
    int32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    __shared__ int32_t wsum[kWarps];
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int32_t base = 0;
    for (int ww = 0; ww < warp; ++ww) base += wsum[ww];
    int32_t acc = base + incl - run;
    for (int bb = b0; bb < b1; ++bb) {
      const int L = lens[bb];
      acc += per_seq_units * (L / G + (L % G ? 1 : 0));
      prefix[bb + 1] = acc;
    }
  }
  __syncthreads();

  // this CTA's slot range (the only 64-bit divisions of the kernel, once)
  const int T = prefix[n_seq];
  const int grid = gridDim.x;
  const int k = blockIdx.x;
  const int start = (int)((int64_t)k * T / grid), end = (int)((int64_t)(k + 1) * T / grid);

  uint32_t uses = 0;        // ring stage uses of this warp so far
  bool ok = true;           // no wait has run out
  unsigned char* wring = ring + warp * C::NST * C::BLK;
  uint64_t* wbars = bars + warp * C::NST;
  const unsigned char* blocks = a.cache + g.blocks_off;

  for (int pos = start; pos < end;) {
    const int b = find_seq(prefix, n_seq, pos);
    const int L = lens[b];
    const int ng = L / G, Tb = L % G;
    const int wb = ng + (Tb ? 1 : 0);
    const int local = pos - prefix[b];
    const int uis = local / wb;
    const int slot0 = local - uis * wb;
    const int slot1 = min(wb, slot0 + (end - pos));
    const int kvh = uis / g.slices, slice = uis % g.slices;
    const int unit = b * per_seq_units + uis;
    const int hbase = kvh * g.gqa + slice * kHeadsPerSlice;
    const int nh = min(kHeadsPerSlice, g.gqa - slice * kHeadsPerSlice);
    const int64_t ublk = ((int64_t)b * g.hkv + kvh) * g.max_groups;

    WarpState<D, KB, VB, G> st;
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) st.o[mt][0] = st.o[mt][1] = st.o[mt][2] = st.o[mt][3] = 0.f;
    st.z[0] = st.z[1] = st.z[2] = st.z[3] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;

    // this warp's group slots: slot0 + warp + 4k below min(slot1, ng)
    const int gend = min(slot1, ng);
    const int first = slot0 + warp;
    const int count = (ok && first < gend) ? (gend - first + kWarps - 1) / kWarps : 0;
    if (lane == 0) {
      for (int s = 0; s < min(C::NST, count); ++s) {
        const uint32_t u = uses + s;
        const int stg = u % C::NST;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&wbars[stg], C::BLK);
        bulk_copy_g2s(wring + stg * C::BLK, blocks + (ublk + first + kWarps * s) * C::BLK, C::BLK,
                      &wbars[stg]);
      }
    }
    // while the copies fly, warp 0 prepares the unit's query fragments
    if (warp == 0)
      load_query<D, KB>(a.q, a.q_dtype, (int64_t)b * g.hq + hbase + g8, g8 < nh, lane, qsm, qmsm);
    __syncthreads();
    for (int it = 0; it < count; ++it) {
      const uint32_t u = uses + it;
      const int stg = u % C::NST;
      bool got = mbar_wait_bounded(&wbars[stg], (u / C::NST) & 1);
      got = __all_sync(0xffffffffu, got);
      if (!got) {
        ok = false;
        if (lane == 0) atomicExch(err, KVQ_ERR_DEVICE);
        break;
      }
      process_group<D, KB, VB, G>(st, wring + stg * C::BLK, qsm, qmsm, lane);
      __syncwarp();
      if (lane == 0 && it + C::NST < count) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&wbars[stg], C::BLK);
        bulk_copy_g2s(wring + stg * C::BLK,
                      blocks + (ublk + first + kWarps * (it + C::NST)) * C::BLK, C::BLK,
                      &wbars[stg]);
      }
    }
    uses += count;
    // the tail slot (index ng) belongs to warp (ng - slot0) % 4
    if (ok && Tb > 0 && slot1 == wb && slot0 <= ng && ((ng - slot0) % kWarps) == warp) {
      const __half* tk = reinterpret_cast<const __half*>(
          a.cache + g.tails_off + ((int64_t)b * g.hkv + kvh) * g.tail_bytes);
      process_tail<D, KB, VB, G>(st, tk, tk + G * D, Tb, qsm, lane, wring);
    }

    // ---- merge the 4 warps (the ring is idle: every issued copy was waited on)
    fence_proxy_async_smem();
    __syncthreads();
    {
      float* mo = merge + (warp * kHeadsPerSlice) * (D + 2);
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
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        const int c0 = 16 * mt + g8, c1 = c0 + 8;
        const int j = (16 * mt) / G;
        mo[(2 * i4) * (D + 2) + c0] = st.o[mt][0] + zl0[j];
        mo[(2 * i4 + 1) * (D + 2) + c0] = st.o[mt][1] + zl1[j];
        mo[(2 * i4) * (D + 2) + c1] = st.o[mt][2] + zl0[j];
        mo[(2 * i4 + 1) * (D + 2) + c1] = st.o[mt][3] + zl1[j];
      }
      if (g8 == 0) {
        mo[(2 * i4) * (D + 2) + D] = st.m[0];
        mo[(2 * i4 + 1) * (D + 2) + D] = st.m[1];
        mo[(2 * i4) * (D + 2) + D + 1] = l0;
        mo[(2 * i4 + 1) * (D + 2) + D + 1] = l1;
      }
    }
    __syncthreads();

    const bool whole = (slot0 == 0 && slot1 == wb);
    // Partial slots: a CTA holds at most two split pieces, its first (slot
    // 2k) and its last (2k + 1); pieces in between are whole units.
    const int myslot = (pos == start) ? 2 * k : 2 * k + 1;
    if (slot0 == 0 && tid == 0) {
      // split record of the unit for the combine kernel: its first partial
      // slot and the number of CTAs holding a piece of it
      const int64_t last = (int64_t)pos + wb - 1;   // the unit's last slot
      const int kl = (int)(((last + 1) * grid - 1) / T);
      *reinterpret_cast<int2*>(a.ws + w.units_off + 8LL * unit) = make_int2(myslot, kl - k + 1);
    }
    for (int idx = tid; idx < nh * D; idx += kThreads) {
      const int h = idx / D, c = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, merge[(ww * kHeadsPerSlice + h) * (D + 2) + D]);
      float Lsum = 0.f, O = 0.f;
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) {
        const float* mo = merge + (ww * kHeadsPerSlice + h) * (D + 2);
        const float f = (mo[D] == -INFINITY) ? 0.f : fast_exp2(mo[D] - M);
        Lsum += mo[D + 1] * f;
        O += mo[c] * f;
      }
      if (whole) {
        reinterpret_cast<__half*>(a.out)[((int64_t)b * g.hq + hbase + h) * D + c] =
            __float2half_rn(O / Lsum);
      } else {
        float* ps = partials + myslot * w.slot_floats + h * (D + 2);
        ps[c] = O;
        if (c == 0) {
          ps[D] = M;
          ps[D + 1] = Lsum;
        }
      }
    }
    fence_proxy_async_smem();   // generic accesses before the next bulk copies
    __syncthreads();            // merge area and ctl are reused by the next piece
    pos += slot1 - slot0;
  }
}

// Merges the pieces of every unit that the decode kernel split across CTAs.
// One block per (unit, head, 32-channel chunk); units held by one CTA were
// written by the decode kernel itself.  Runs as a programmatic dependent
// launch of the decode grid and waits for it before touching the partials.
// Warp 0 turns the pieces' (max, sum) into normalized weights; each warp
// then folds every 4th piece for the block's 32 channels (lane = channel)
// with up to 8 loads in flight, and the warps' sums meet in shared memory.
constexpr int kCombineChunk = 32;
constexpr int kCombineMaxPieces = 2 * kMaxDecodeCtas;

template <int D>
__global__ void __launch_bounds__(kThreads) combine_kernel(const Geom g, const WsLayout w,
                                                           const DecodeArgs a) {
  __shared__ float wgt[kCombineMaxPieces];
  __shared__ float red[kWarps][32];
  __shared__ float sinv;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kChunks = D / kCombineChunk;
  const int chunk = blockIdx.x % kChunks;
  const int h = (blockIdx.x / kChunks) % kHeadsPerSlice;
  const int unit = blockIdx.x / (kChunks * kHeadsPerSlice);
  const int2 rec = *reinterpret_cast<const int2*>(a.ws + w.units_off + 8LL * unit);
  const int npc = rec.y;
  if (npc <= 1) return;   // whole unit: already written
  const int per_seq = g.hkv * g.slices;
  const int b = unit / per_seq, uis = unit % per_seq;
  const int kvh = uis / g.slices, slice = uis % g.slices;
  const int nh = min(kHeadsPerSlice, g.gqa - slice * kHeadsPerSlice);
  if (h >= nh) return;
  const int hbase = kvh * g.gqa + slice * kHeadsPerSlice;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t sl0 = rec.x, kf = sl0 / 2;
  const float* partials = reinterpret_cast<const float*>(a.ws + w.partials_off) + h * (D + 2);
  auto piece = [&](int pc) { return partials + (pc == 0 ? sl0 : 2 * (kf + pc)) * w.slot_floats; };

  if (warp == 0) {
    // weights e^(m_k - M) / L, L = sum_k l_k e^(m_k - M)
    float M = -INFINITY;
    for (int pc = lane; pc < npc; pc += 32) M = fmaxf(M, __ldcg(piece(pc) + D));
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int pc = lane; pc < npc; pc += 32) {
      const float* ps = piece(pc);
      const float wk = fast_exp2(__ldcg(ps + D) - M);
      wgt[pc] = wk;
      L += wk * __ldcg(ps + D + 1);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) sinv = 1.0f / L;
  }
  __syncthreads();
  const int c = chunk * kCombineChunk + lane;
  float acc = 0.f;
  for (int p0 = warp; p0 < npc; p0 += 8 * kWarps) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int pc = p0 + u * kWarps;
      v[u] = pc < npc ? __ldcg(piece(pc) + c) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int pc = p0 + u * kWarps;
      if (pc < npc) acc += wgt[pc] * v[u];
    }
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float o = 0.f;
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) o += red[ww][lane];
    reinterpret_cast<__half*>(a.out)[((int64_t)b * g.hq + hbase + h) * D + c] =
        __float2half_rn(o * sinv);
  }
}

template <int D, int KB, int VB, int G>
size_t smem_bytes(int n_seq) {
  return DecCfg<D, KB, VB, G>::SMEM_FIXED + 4 * (size_t)(n_seq + 1);
}

template <int D, int KB, int VB, int G>
cudaError_t max_ctas_t(int* out) {
  using C = DecCfg<D, KB, VB, G>;
  auto kern = decode_kernel<D, KB, VB, G>;
  const size_t sm = smem_bytes<D, KB, VB, G>(64);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(C::SMEM_FIXED + 4 * (kMaxSeqsDecode + 1)));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, sm);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  *out = max(1, min(kMaxDecodeCtas, per_sm * sms));
  return cudaSuccess;
}

template <int D, int KB, int VB, int G>
cudaError_t launch_t(const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid,
                     cudaStream_t stream) {
  using C = DecCfg<D, KB, VB, G>;
  if (g.block_bytes != C::BLK || g.sec_vmin != C::SEC_VMIN || g.sec_kscale != C::SEC_KSCALE)
    return cudaErrorInvalidValue;
  auto kern = decode_kernel<D, KB, VB, G>;
  const size_t sm = smem_bytes<D, KB, VB, G>(a.n_seq);
  static bool configured = false;   // attribute set once, before any capture
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(C::SMEM_FIXED + 4 * (kMaxSeqsDecode + 1)));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  kern<<<grid, kThreads, sm, stream>>>(g, w, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the combine kernel, a programmatic dependent of the decode grid
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)(a.n_seq * g.hkv * g.slices * kHeadsPerSlice * (D / kCombineChunk)));
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = 0;
  lc.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, combine_kernel<D>, g, w, a);
}

}  // namespace

#define KVQ_DECODE_DISPATCH(FN, ...)                                                     \
  do {                                                                                   \
    if (g.d == 128 && g.kb == 4 && g.vb == 2 && g.G == 32) return FN<128, 4, 2, 32>(__VA_ARGS__); \
    if (g.d == 128 && g.kb == 2 && g.vb == 2 && g.G == 32) return FN<128, 2, 2, 32>(__VA_ARGS__); \
    if (g.d == 128 && g.kb == 4 && g.vb == 2 && g.G == 64) return FN<128, 4, 2, 64>(__VA_ARGS__); \
    if (g.d == 128 && g.kb == 2 && g.vb == 2 && g.G == 64) return FN<128, 2, 2, 64>(__VA_ARGS__); \
    if (g.d == 128 && g.kb == 4 && g.vb == 4 && g.G == 32) return FN<128, 4, 4, 32>(__VA_ARGS__); \
    if (g.d == 128 && g.kb == 2 && g.vb == 4 && g.G == 32) return FN<128, 2, 4, 32>(__VA_ARGS__); \
    if (g.d == 128 && g.kb == 4 && g.vb == 4 && g.G == 64) return FN<128, 4, 4, 64>(__VA_ARGS__); \
    if (g.d == 128 && g.kb == 2 && g.vb == 4 && g.G == 64) return FN<128, 2, 4, 64>(__VA_ARGS__); \
    if (g.d == 64 && g.kb == 4 && g.vb == 2 && g.G == 32) return FN<64, 4, 2, 32>(__VA_ARGS__);   \
    if (g.d == 64 && g.kb == 2 && g.vb == 2 && g.G == 32) return FN<64, 2, 2, 32>(__VA_ARGS__);   \
    if (g.d == 64 && g.kb == 4 && g.vb == 2 && g.G == 64) return FN<64, 4, 2, 64>(__VA_ARGS__);   \
    if (g.d == 64 && g.kb == 2 && g.vb == 2 && g.G == 64) return FN<64, 2, 2, 64>(__VA_ARGS__);   \
    if (g.d == 64 && g.kb == 4 && g.vb == 4 && g.G == 32) return FN<64, 4, 4, 32>(__VA_ARGS__);   \
    if (g.d == 64 && g.kb == 2 && g.vb == 4 && g.G == 32) return FN<64, 2, 4, 32>(__VA_ARGS__);   \
    if (g.d == 64 && g.kb == 4 && g.vb == 4 && g.G == 64) return FN<64, 4, 4, 64>(__VA_ARGS__);   \
    if (g.d == 64 && g.kb == 2 && g.vb == 4 && g.G == 64) return FN<64, 2, 4, 64>(__VA_ARGS__);   \
    return cudaErrorInvalidValue;                                                        \
  } while (0)

cudaError_t decode_max_ctas(const Geom& g, int* max_ctas) {
  KVQ_DECODE_DISPATCH(max_ctas_t, max_ctas);
}

cudaError_t launch_decode(const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid,
                          cudaStream_t stream) {
  KVQ_DECODE_DISPATCH(launch_t, g, w, a, grid, stream);
}

#undef KVQ_DECODE_DISPATCH

// ---------------------------------------------------------------------------
// Decode without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// code running while a CUDA graph is being captured (an allocation there
// breaks or pollutes the capture), plugins whose host framework owns every
// device allocation and offers no workspace hook, and deployments that forbid
// allocation after start-up.  For them the scratch the decode kernel needs
// (error word, per-unit tickets, split partials) lives in this fixed
// file-scope device array instead of a caller buffer.  Every GPU that loads
// the library holds it until the process exits.  All such calls share it:
// calls that overlap on the GPU race on it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};   // device address of the array, per device
}  // namespace

// Set-up, once per device, with that device current: the address the
// kernels must be given (the array's name is only a host-side stand-in).
cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace kvq
