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
//     low halves (rows 8-15 of the tile) against the key mins;
//   * unpacks key codes to exact fp16 pairs and runs S = q' K^T on m16n8k16
//     tiles (rows = query heads, columns = tokens);
//   * updates the running max / rescales, exponentiates (exp2 domain);
//   * runs O^T += V_code^T (p s_v) on tiles whose rows are channels and whose
//     columns are heads (the P fragment of S is already the B fragment), with
//     the per-token value scale folded into p for each channel group, and
//     sum_t p_t z_t (value mins) and sum_t p_t (the softmax denominator) on
//     one more tile.
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
  static constexpr int NST = (BLK <= 4096) ? 4 : 2;   // ring stages per warp
  static constexpr int RING = kWarps * NST * BLK;
  static constexpr int MERGE_FLOATS = kWarps * kHeadsPerSlice * (D + 2);
  static_assert(MERGE_FLOATS * 4 <= RING, "merge area must fit in the ring");
  static constexpr int SMEM_FIXED = RING + kWarps * NST * 8 + 64;
};

struct SharedCtl {
  int last;   // this CTA completes the current unit
};

template <int D, int KB, int VB, int G>
struct WarpState {
  float o[D / 16][4];   // O^T: rows channels, cols heads (unnormalized)
  float z[4];           // rows: value-min terms (j < J) and sum p (row J)
  float m;              // running max of head (lane / 4), log2 domain
};

// Load this lane's query fragments (or zeros for a padding head): rows g of
// the A tile, channels 16kt + 2i + {0,1} and + 8 + {0,1}; q is scaled by
// log2(e)/sqrt(d) and split into fp16 high and low parts.
template <int D>
__device__ __forceinline__ void load_query(const void* q, int dtype, int64_t row, bool valid,
                                           int i4, uint32_t (&qh)[D / 16][2],
                                           uint32_t (&ql)[D / 16][2]) {
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
#pragma unroll
  for (int kt = 0; kt < D / 16; ++kt) {
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const float x0 = x[kt][v].x * sc, x1 = x[kt][v].y * sc;
      const __half2 h = __floats2half2_rn(x0, x1);
      const float2 hf = __half22float2(h);
      qh[kt][v] = h2_as_u32(h);
      ql[kt][v] = pack_h2(x0 - hf.x, x1 - hf.y);
    }
  }
}

// Online-softmax update of a warp for new logits s[n][0..1] (head = lane/4,
// tokens in the C layout) and conversion to fp16 probabilities p[n].
template <int D, int N, int KB, int VB, int G>
__device__ __forceinline__ void softmax_update(WarpState<D, KB, VB, G>& st, float (&s)[N][2],
                                               uint32_t (&p)[N], int lane) {
  float mx = -INFINITY;
#pragma unroll
  for (int n = 0; n < N; ++n) mx = fmaxf(mx, fmaxf(s[n][0], s[n][1]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float mnew = fmaxf(st.m, mx);
  if (__any_sync(0xffffffffu, mnew > st.m)) {
    const float alpha = fast_exp2(st.m - mnew);   // 0 when st.m = -inf
    const int i4 = lane & 3;
    const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * i4);
    const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * i4 + 4);
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
    st.m = mnew;
  }
#pragma unroll
  for (int n = 0; n < N; ++n)
    p[n] = pack_h2(fast_exp2(s[n][0] - st.m), fast_exp2(s[n][1] - st.m));
}

// One quantized group from the shared-memory stage `sp`.
template <int D, int KB, int VB, int G>
__device__ __forceinline__ void process_group(WarpState<D, KB, VB, G>& st,
                                              const unsigned char* __restrict__ sp,
                                              const uint32_t (&qh)[D / 16][2],
                                              const uint32_t (&ql)[D / 16][2], int lane) {
  using C = DecCfg<D, KB, VB, G>;
  const int g8 = lane >> 2, i4 = lane & 3;

  // q' = q * s_key (fp16, one rounding) and the min term sum_c q_c z_c
  uint32_t qs[C::KT][2];
  float bias[4] = {0.f, 0.f, 0.f, 0.f};
  {
    uint32_t ksw[D / 8], kzw[D / 8];
    lds_words<D / 8>(reinterpret_cast<const uint32_t*>(sp + C::SEC_KSCALE) + i4 * (D / 8), ksw);
    lds_words<D / 8>(reinterpret_cast<const uint32_t*>(sp + C::SEC_KMIN) + i4 * (D / 8), kzw);
#pragma unroll
    for (int kt = 0; kt < C::KT; ++kt) {
      const uint32_t s0 = ksw[2 * kt], s1 = ksw[2 * kt + 1];
      qs[kt][0] = h2_as_u32(__hfma2(u32_as_h2(qh[kt][0]), u32_as_h2(s0),
                                    __hmul2(u32_as_h2(ql[kt][0]), u32_as_h2(s0))));
      qs[kt][1] = h2_as_u32(__hfma2(u32_as_h2(qh[kt][1]), u32_as_h2(s1),
                                    __hmul2(u32_as_h2(ql[kt][1]), u32_as_h2(s1))));
      mma16816(bias, qh[kt][0], ql[kt][0], qh[kt][1], ql[kt][1], kzw[2 * kt], kzw[2 * kt + 1]);
    }
  }
  const float b = bias[0] + bias[2];   // head g8: high-part rows + low-part rows

  // S = q' K^T over the G tokens
  float s[C::NT][2];
  const uint32_t* kcw = reinterpret_cast<const uint32_t*>(sp + C::SEC_KCODES);
  static_for<C::NT>([&](auto nt_) {
    constexpr int nt = decltype(nt_)::value;
    uint32_t kw[C::LWK];
    lds_words<C::LWK>(kcw + (nt * 32 + lane) * C::LWK, kw);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    static_for<C::KT>([&](auto kt_) {
      constexpr int kt = decltype(kt_)::value;
      constexpr int p0 = 2 * kt, p1 = 2 * kt + 1;
      const uint32_t b0 = unpack_pair<KB, p0 % C::FK>(kw[p0 / C::FK]);
      const uint32_t b1 = unpack_pair<KB, p1 % C::FK>(kw[p1 / C::FK]);
      mma16816(acc, qs[kt][0], 0u, qs[kt][1], 0u, b0, b1);
    });
    s[nt][0] = acc[0] + b;
    s[nt][1] = acc[1] + b;
  });

  uint32_t p[C::NT];
  softmax_update<D, C::NT, KB, VB, G>(st, s, p, lane);

  // O^T += V^T (p * s_v); Z += [z_v; 1]^T p
  const uint32_t* vcw = reinterpret_cast<const uint32_t*>(sp + C::SEC_VCODES);
  const uint32_t* vsw = reinterpret_cast<const uint32_t*>(sp + C::SEC_VSCALE);
  const uint32_t* vzw = reinterpret_cast<const uint32_t*>(sp + C::SEC_VMIN);
  static_for<C::KV>([&](auto kv_) {
    constexpr int kv = decltype(kv_)::value;
    const uint32_t bp0 = p[2 * kv], bp1 = p[2 * kv + 1];
    uint32_t za0 = 0u, za2 = 0u;
    if (g8 < C::J) {
      const uint32_t* zz = vzw + ((4 * kv + i4) * C::J + g8) * 2;
      za0 = zz[0];
      za2 = zz[1];
    } else if (g8 == C::J) {
      za0 = za2 = 0x3C003C00u;   // fp16 pair (1, 1)
    }
    mma16816(st.z, za0, 0u, za2, 0u, bp0, bp1);

    uint32_t sw[2 * C::J];
    lds_words<2 * C::J>(vsw + (4 * kv + i4) * C::J * 2, sw);
    uint32_t bs[C::J][2];
#pragma unroll
    for (int j = 0; j < C::J; ++j) {
      bs[j][0] = h2_as_u32(__hmul2(u32_as_h2(bp0), u32_as_h2(sw[2 * j])));
      bs[j][1] = h2_as_u32(__hmul2(u32_as_h2(bp1), u32_as_h2(sw[2 * j + 1])));
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
                                             const uint32_t (&qh)[D / 16][2],
                                             const uint32_t (&ql)[D / 16][2], int lane,
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

    float s[2][2];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const unsigned char* krow = buf + (8 * n + g8) * TS::KROW + 4 * i4;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kt = 0; kt < C::KT; ++kt) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(krow + 32 * kt);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(krow + 32 * kt + 16);
        mma16816(acc, qh[kt][0], ql[kt][0], qh[kt][1], ql[kt][1], b0, b1);
      }
      const int t0 = 16 * kv + 8 * n + 2 * i4;      // tokens of this lane's C columns
      s[n][0] = (t0 < T) ? acc[0] + acc[2] : -INFINITY;
      s[n][1] = (t0 + 1 < T) ? acc[1] + acc[3] : -INFINITY;
    }
    uint32_t p[2];
    softmax_update<D, 2, KB, VB, G>(st, s, p, lane);
    const uint32_t ones = (g8 == C::J) ? 0x3C003C00u : 0u;
    mma16816(st.z, ones, 0u, ones, 0u, p[0], p[1]);
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
      mma16816(st.o[mt], a0, a1, a2, a3, p[0], p[1]);
    }
    __syncwarp();   // every lane is done with this chunk before the next copy
  }
}

// Largest b in [0, n) with prefix[b] <= pos (prefix[0] = 0, increasing).
__device__ __forceinline__ int find_seq(const int32_t* prefix, int n, int64_t pos) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid + 1] <= pos) lo = mid + 1; else hi = mid;
  }
  return lo;
}

template <int D, int KB, int VB, int G>
__global__ void __launch_bounds__(kThreads, 3)
    decode_kernel(const Geom g, const WsLayout w, const DecodeArgs a) {
  using C = DecCfg<D, KB, VB, G>;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::RING);
  SharedCtl* ctl = reinterpret_cast<SharedCtl*>(bars + kWarps * C::NST);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + C::SMEM_FIXED);
  float* merge = reinterpret_cast<float*>(smem);   // reuses the ring between pieces

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, i4 = lane & 3;
  const int n_seq = a.n_seq;
  const int per_seq_units = g.hkv * g.slices;
  const int32_t* lens = reinterpret_cast<const int32_t*>(a.cache + g.lens_off);
  int32_t* err = reinterpret_cast<int32_t*>(a.ws + w.err_off);
  int32_t* tickets = reinterpret_cast<int32_t*>(a.ws + w.tickets_off);
  float* partials = reinterpret_cast<float*>(a.ws + w.partials_off);

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

  const int64_t T = prefix[n_seq];
  const int64_t grid = gridDim.x;
  const int64_t k = blockIdx.x;
  const int64_t start = k * T / grid, end = (k + 1) * T / grid;
  auto cta_of = [&](int64_t p) { return ((p + 1) * grid - 1) / T; };
  auto cta_start = [&](int64_t kk) { return kk * T / grid; };

  uint32_t uses = 0;        // ring stage uses of this warp so far
  bool ok = true;           // no wait has run out
  unsigned char* wring = ring + warp * C::NST * C::BLK;
  uint64_t* wbars = bars + warp * C::NST;
  const unsigned char* blocks = a.cache + g.blocks_off;

  for (int64_t pos = start; pos < end;) {
    const int b = find_seq(prefix, n_seq, pos);
    const int L = lens[b];
    const int ng = L / G, Tb = L % G;
    const int wb = ng + (Tb ? 1 : 0);
    const int64_t local = pos - prefix[b];
    const int uis = (int)(local / wb);
    const int slot0 = (int)(local % wb);
    const int slot1 = (int)(((int64_t)slot0 + (end - pos)) < wb ? ((int64_t)slot0 + (end - pos)) : wb);
    const int kvh = uis / g.slices, slice = uis % g.slices;
    const int unit = b * per_seq_units + uis;
    const int hbase = kvh * g.gqa + slice * kHeadsPerSlice;
    const int nh = min(kHeadsPerSlice, g.gqa - slice * kHeadsPerSlice);
    const int64_t ublk = ((int64_t)b * g.hkv + kvh) * g.max_groups;

    uint32_t qh[C::KT][2], ql[C::KT][2];
    load_query<D>(a.q, a.q_dtype, (int64_t)b * g.hq + hbase + g8, g8 < nh, i4, qh, ql);

    WarpState<D, KB, VB, G> st;
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) st.o[mt][0] = st.o[mt][1] = st.o[mt][2] = st.o[mt][3] = 0.f;
    st.z[0] = st.z[1] = st.z[2] = st.z[3] = 0.f;
    st.m = -INFINITY;

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
      process_group<D, KB, VB, G>(st, wring + stg * C::BLK, qh, ql, lane);
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
      process_tail<D, KB, VB, G>(st, tk, tk + G * D, Tb, qh, ql, lane, wring);
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
        mo[(2 * i4) * (D + 2) + D + 1] = l0;
        mo[(2 * i4 + 1) * (D + 2) + D + 1] = l1;
      }
      if (i4 == 0) mo[g8 * (D + 2) + D] = st.m;
    }
    __syncthreads();

    const bool whole = (slot0 == 0 && slot1 == wb);
    const int64_t up = prefix[b] + (int64_t)uis * wb;   // first slot of the unit
    const int64_t kf = cta_of(up), kl = cta_of(up + wb - 1);
    const int64_t myslot = (k == kf && cta_start(k) < up) ? 2 * k + 1 : 2 * k;
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
    if (!whole) {
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        const int old = atomicAdd(&tickets[unit], 1);
        ctl->last = (old == (int)(kl - kf));
      }
      __syncthreads();
      if (ctl->last) {
        __threadfence();
        for (int idx = tid; idx < nh * D; idx += kThreads) {
          const int h = idx / D, c = idx % D;
          float M = -INFINITY;
          for (int64_t kk = kf; kk <= kl; ++kk) {
            const int64_t sl = (kk == kf && cta_start(kk) < up) ? 2 * kk + 1 : 2 * kk;
            M = fmaxf(M, __ldcg(partials + sl * w.slot_floats + h * (D + 2) + D));
          }
          float Lsum = 0.f, O = 0.f;
          for (int64_t kk = kf; kk <= kl; ++kk) {
            const int64_t sl = (kk == kf && cta_start(kk) < up) ? 2 * kk + 1 : 2 * kk;
            const float* ps = partials + sl * w.slot_floats + h * (D + 2);
            const float f = fast_exp2(__ldcg(ps + D) - M);
            Lsum += __ldcg(ps + D + 1) * f;
            O += __ldcg(ps + c) * f;
          }
          reinterpret_cast<__half*>(a.out)[((int64_t)b * g.hq + hbase + h) * D + c] =
              __float2half_rn(O / Lsum);
        }
        if (tid == 0) tickets[unit] = 0;
      }
    }
    fence_proxy_async_smem();   // generic accesses before the next bulk copies
    __syncthreads();            // merge area and ctl are reused by the next piece
    pos += slot1 - slot0;
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
  return cudaGetLastError();
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
