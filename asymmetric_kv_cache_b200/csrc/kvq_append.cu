// Append kernel of libkvq: per-channel key quantization, per-token value
// quantization, bit packing into LAYOUT v2, the fp16 tail and its flush.
//
// "[Framework] The Asymmetric Key-Value Cache Compression", §III: keys are
// quantized per channel (outliers stay in their column), values per token,
// and the newest tokens stay in fp16.  One launch serves prefill (many whole
// groups straight from the input), per-step decode appends (one token into
// the tail) and the flush of a tail that fills a group.
//
// Grid: x = tasks (flattened over sequences), y = kv head; 128 threads.
// A task is either one group to quantize (tokens taken from the old tail
// and/or the input) or, when no group completes, the copy of the new tokens
// into the tail.  With a recent window of R tokens a group is quantized once
// R newer tokens follow it (same page, §III and §V), and the tail is a ring
// of W = R + G token slots (token p in slot p mod W), so tokens that stay in
// the tail never move.  A slot whose old token a group task reads is
// rewritten, if a new tail token maps to it, by that same task after its
// read; every other new tail token is written by the sequence's first task.
// So no slot is read and written by two CTAs.  With a sink window of S
// tokens (InnerQ abstract, page "WUSH-KV: KV Cache Quantization with
// Data-Adaptive Transforms") the first S tokens of a sequence go to an fp16
// sink area instead, and all of the above applies to the positions after
// it (q = p - S).
//
// Every CTA reads the sequence's current length from the device copy when
// it starts and counts itself on the sequence's ticket (an atomic in the
// cache buffer, no waiting); the CTA that counts last stores the new length
// at its end and re-arms the ticket.  All reads of the old length therefore
// precede its update.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

template <int D, int G, int KB, int VB>
struct AppCfg {
  static constexpr int J = D / G;
  static constexpr int QV = (1 << VB) - 1;
  static constexpr int FV = 16 / VB;                  // value-code pairs per 32-bit word
  static constexpr int VWORDS_PER_LANE = D * VB / 64;  // per 16-token tile
  static constexpr int VWORDS = G * D * VB / 32;       // (key words: key_codes)
  // dynamic shared memory: fp16 K and V of the group (token rows padded by
  // 16 bytes, so that rows fall 4 banks apart), the fp16 metadata in slot
  // order, and per key channel / per (token, value group) the fp32
  // parameters of the code computation {z, 1/s, s}
  static constexpr int DP = D + 8;   // halves per staged row
  static constexpr int SM_K = 0;
  static constexpr int SM_V = SM_K + 2 * G * DP;
  static constexpr int SM_KS = SM_V + 2 * G * DP;
  static constexpr int SM_KZ = SM_KS + 2 * D;
  static constexpr int SM_VS = SM_KZ + 2 * D;
  static constexpr int SM_VZ = SM_VS + 2 * G * J;
  static constexpr int SM_KP = (SM_VZ + 2 * G * J + 15) / 16 * 16;
  static constexpr int SM_VP = SM_KP + 16 * D;
  // per row slice and key channel pair: fp16x2 {min, max} (key_stats_part)
  static constexpr int SM_KR = SM_VP + 16 * G * J;
  static constexpr int SM_TOTAL = SM_KR + 8 * (128 / (D / 2)) * (D / 2);
};

// Eight consecutive input elements (16-byte aligned) rounded to fp16
// (nearest even), packed in a uint4.
__device__ __forceinline__ uint4 load8_fp16(const void* base, int64_t idx, int dtype) {
  if (dtype == KVQ_FP16) return *reinterpret_cast<const uint4*>(reinterpret_cast<const __half*>(base) + idx);
  uint32_t h[4];
  if (dtype == KVQ_BF16) {
    const uint4 r = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      const __half2 hh = __floats2half2_rn(f.x, f.y);
      h[i] = *reinterpret_cast<const uint32_t*>(&hh);
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4);
    const __half2 h0 = __floats2half2_rn(a.x, a.y), h1 = __floats2half2_rn(a.z, a.w);
    const __half2 h2 = __floats2half2_rn(b.x, b.y), h3 = __floats2half2_rn(b.z, b.w);
    h[0] = *reinterpret_cast<const uint32_t*>(&h0);
    h[1] = *reinterpret_cast<const uint32_t*>(&h1);
    h[2] = *reinterpret_cast<const uint32_t*>(&h2);
    h[3] = *reinterpret_cast<const uint32_t*>(&h3);
  }
  return make_uint4(h[0], h[1], h[2], h[3]);
}

// Eight consecutive input elements as fp32 (exact for fp16 / bf16 / fp32).
__device__ __forceinline__ void load8_f32(const void* base, int64_t idx, int dtype, float (&y)[8]) {
  if (dtype == KVQ_FP32) {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4);
    y[0] = a.x; y[1] = a.y; y[2] = a.z; y[3] = a.w; y[4] = b.x; y[5] = b.y; y[6] = b.z; y[7] = b.w;
    return;
  }
  const uint4 r = dtype == KVQ_FP16
                      ? *reinterpret_cast<const uint4*>(reinterpret_cast<const __half*>(base) + idx)
                      : *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = dtype == KVQ_FP16
                         ? __half22float2(*reinterpret_cast<const __half2*>(&w[i]))
                         : __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    y[2 * i] = f.x;
    y[2 * i + 1] = f.y;
  }
}

// Sixteen-byte chunk cc (channels 8cc .. 8cc + 7) of an input token row as
// the cache stores it: rounded to fp16, after the rotation when `rot`.
// Rotation ("[Framework] The Asymmetric Key-Value Cache Compression", §IV
// stage 1: Y = X H, fast Walsh-Hadamard transform): the unnormalized
// transform in fp32, stages h = 1, 2, ..., D/2 in that order, each pair
// (j, j + h) of a block of 2h channels becoming (a + b, a - b), then times
// fp32(1 / sqrt(D)) and rounded to fp16 - every step an IEEE fp32 operation
// on the same operands in the same order for every element, so the result
// is reproducible bit for bit.  A row is spread over D / 8 consecutive
// lanes (chunk cc in lane cc of its lane group); stages h < 8 run inside a
// lane, h >= 8 exchange with lane cc ^ (h / 8).  Every lane of the warp
// must call this together (the exchanges are warp-wide); `use` = false
// lanes load nothing and return zeros.
template <int D>
__device__ __forceinline__ uint4 row_chunk16(const void* base, int64_t idx, int dtype, int cc,
                                             bool use, bool rot) {
  if (!rot) return use ? load8_fp16(base, idx, dtype) : make_uint4(0u, 0u, 0u, 0u);
  float y[8];
  if (use) {
    load8_f32(base, idx, dtype, y);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = 0.f;
  }
  fwht_lanes<D, 8>(y, cc);
  const float sc = rot_scale<D>();
  uint32_t h2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    h2[i] = h2_as_u32(__floats2half2_rn(__fmul_rn(y[2 * i], sc), __fmul_rn(y[2 * i + 1], sc)));
  return make_uint4(h2[0], h2[1], h2[2], h2[3]);
}

// Channels 8cc .. 8cc+7 of tail token u from the value tail, whose token
// pairs are interleaved ([u/2][c][u%2]).
__device__ __forceinline__ uint4 tail_v8(const __half* tailv, int u, int cc, int D) {
  const uint4* src = reinterpret_cast<const uint4*>(tailv + ((u >> 1) * D + 8 * cc) * 2);
  const uint4 a = src[0], b = src[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)   // halves (2i, u&1) and (2i+1, u&1)
    o[i] = (u & 1) ? __byte_perm(w[2 * i], w[2 * i + 1], 0x7632) : __byte_perm(w[2 * i], w[2 * i + 1], 0x5410);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Write eight fp16 values (one 16-byte chunk of token t) into the tails.
__device__ __forceinline__ void store_tail8(__half* tailk, __half* tailv, int t, int cc, int D,
                                            uint4 k8, uint4 v8) {
  *reinterpret_cast<uint4*>(tailk + t * D + 8 * cc) = k8;
  const __half* hv = reinterpret_cast<const __half*>(&v8);
#pragma unroll
  for (int i = 0; i < 8; ++i) tailv[((t >> 1) * D + 8 * cc + i) * 2 + (t & 1)] = hv[i];
}

// Quantize one value: clamp(rne((x - z) / s), 0, Q) in fp32 with the stored
// fp16 s, z widened; s == 0 gives 0.  IEEE division, no contraction.
__device__ __forceinline__ int quant_code(float x, float zf, float sf, int Q) {
  if (sf == 0.0f) return 0;
  const float t = __fdiv_rn(__fsub_rn(x, zf), sf);
  int c = __float2int_rn(t);
  c = c < 0 ? 0 : c;
  return c > Q ? Q : c;
}

// Code computation in pairs (sm_100 packed fp32x2 arithmetic, IEEE round
// to nearest per element, so each element is exactly the scalar result):
// d = x - z (exact: both are fp16 values), t = d * (1/s) with 1/s correctly
// rounded, rne(t) by adding 1.5 * 2^23 (whose mantissa then holds the
// integer).  t is within 3e-6 of the correctly rounded quotient d / s used
// by the definition, so the two round to the same integer unless d / s lies
// within 6.1e-5 of a half-integer; such a pair is flagged and recomputed with
// IEEE division.  z is the group minimum, so d >= 0 and the code needs no
// lower clamp; the upper clamp to Q stays (a subnormal s is rounded coarsely,
// and d / s can then pass Q + 1/2).  s == 0 has 1/s stored as 0: code 0.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void codes2(float x0, float x1, float z0, float z1, float r0, float r1,
                                       uint32_t Q, uint32_t& c0, uint32_t& c1, bool& near_tie) {
  uint64_t d, t, y, k, e;
  const uint64_t magic = f32x2(12582912.0f, 12582912.0f);
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f32x2(x0, x1)), "l"(f32x2(z0, z1)));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(d), "l"(f32x2(r0, r1)));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(t), "l"(magic));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(k) : "l"(y), "l"(magic));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(e) : "l"(t), "l"(k));
  c0 = min((uint32_t)y & 0xFFu, Q);
  c1 = min((uint32_t)(y >> 32) & 0xFFu, Q);
  // |e| >= 0.5 - 2^-14 in either half (e in [-0.5, 0.5])
  const uint32_t a0 = (uint32_t)e & 0x7FFFFFFFu, a1 = (uint32_t)(e >> 32) & 0x7FFFFFFFu;
  near_tie |= (a0 >= 0x3EFFF800u) | (a1 >= 0x3EFFF800u);   // 0.5 - 2048 ulp
}

// Key statistics of a staged group (fp16 rows of DP halves, G tokens), in
// two phases over the 128 threads.  Part: thread (slice rs, channel pair
// cp) takes the fp16x2 min and max (exact) over its G / NS rows into
// part[rs][cp] = {min, max}.  Final (after a barrier; thread c < D): the
// channel's min and max over the slices, the stored fp16 scale
// fp16((max - min) / QK) and min, their fp32 {z, 1/s, s} for the codes,
// and the metadata in slot order i*(D/4) + 4kt + 2v + e.
template <int D, int G>
__device__ __forceinline__ void key_stats_part(const __half* __restrict__ sk,
                                               uint2* __restrict__ part, int tid) {
  constexpr int DP = D + 8;
  constexpr int NS = 128 / (D / 2);   // row slices
  constexpr int RS = G / NS;          // rows per slice
  const __half2* sk2 = reinterpret_cast<const __half2*>(sk);
  const int cp = tid % (D / 2), rs = tid / (D / 2);
  const __half2* col = sk2 + rs * RS * (DP / 2) + cp;
  __half2 mn = col[0], mx = mn;
#pragma unroll
  for (int r = 1; r < RS; ++r) {
    const __half2 x = col[r * (DP / 2)];
    mn = __hmin2(mn, x);
    mx = __hmax2(mx, x);
  }
  part[rs * (D / 2) + cp] = make_uint2(h2_as_u32(mn), h2_as_u32(mx));
}
template <int D, int G, int QK>
__device__ __forceinline__ void key_stats_final(const uint2* __restrict__ part,
                                                float4* __restrict__ kp, __half* __restrict__ ks,
                                                __half* __restrict__ kz, int c) {
  constexpr int NS = 128 / (D / 2);
  const int cp = c >> 1, e = c & 1;
  float mnf = INFINITY, mxf = -INFINITY;
#pragma unroll
  for (int rs = 0; rs < NS; ++rs) {
    const uint2 pm = part[rs * (D / 2) + cp];
    const __half2 mn = *reinterpret_cast<const __half2*>(&pm.x);
    const __half2 mx = *reinterpret_cast<const __half2*>(&pm.y);
    mnf = fminf(mnf, e ? __high2float(mn) : __low2float(mn));
    mxf = fmaxf(mxf, e ? __high2float(mx) : __low2float(mx));
  }
  const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mxf, mnf), (float)QK));
  const __half z16 = __float2half_rn(mnf);
  const float sf = __half2float(s16);
  kp[c] = make_float4(__half2float(z16), sf == 0.0f ? 0.0f : __frcp_rn(sf), sf, 0.0f);
  // metadata slot i*(D/4) + 4kt + 2v + e
  const int kt = c >> 4, v = (c >> 3) & 1, i = (c >> 1) & 3;
  const int slot = i * (D / 4) + 4 * kt + 2 * v + e;
  ks[slot] = s16;
  kz[slot] = z16;
}

// A key-code word recomputed with IEEE division (the rare words whose fast
// quotients lie near a rounding boundary): token t, word w of lane group i.
// Out of line, so that the hot loops stay small in the instruction cache.
template <int D, int KBq>
__device__ __noinline__ uint32_t key_word_exact(const __half* __restrict__ sk,
                                                const float4* __restrict__ kp, int t, int w, int i) {
  constexpr int DP = D + 8;
  constexpr int QK = (1 << KBq) - 1;
  constexpr int FK = 16 / KBq;
  uint32_t word = 0;
#pragma unroll 1
  for (int f = 0; f < FK; ++f) {
    const int p = w * FK + f;
    const int c = 16 * (p >> 1) + 8 * (p & 1) + 2 * i;
#pragma unroll 1
    for (int e = 0; e < 2; ++e) {
      const float4 pc = kp[c + e];
      const uint32_t code = (uint32_t)quant_code(__half2float(sk[t * DP + c + e]), pc.x, pc.z, QK);
      word |= code << (KBq * (e * FK + f));
    }
  }
  return word;
}

// The same for a value-code word: token tile kv, word w, lane (gg, i).
template <int D, int G, int VB>
__device__ __noinline__ uint32_t value_word_exact(const __half* __restrict__ sv,
                                                  const float4* __restrict__ vp, int kv, int w,
                                                  int gg, int i) {
  constexpr int DP = D + 8;
  constexpr int J = D / G;
  constexpr int QV = (1 << VB) - 1;
  constexpr int FV = 16 / VB;
  uint32_t word = 0;
#pragma unroll 1
  for (int fl = 0; fl < FV; ++fl) {
    const int kh = fl / (FV / 2), rem = fl % (FV / 2);
    const int u = rem >> 1, hr = rem & 1;
    const int mt = w * (FV / 4) + u;
    const int c = 16 * mt + 8 * hr + gg;
#pragma unroll 1
    for (int e = 0; e < 2; ++e) {
      const int t = 16 * kv + 8 * kh + 2 * i + e;
      const float4 pc = vp[t * J + c / G];
      const uint32_t code = (uint32_t)quant_code(__half2float(sv[t * DP + c]), pc.x, pc.z, QV);
      word |= code << (VB * (e * FV + fl));
    }
  }
  return word;
}

// Key codes of a staged group at KBq bits, packed word by word into the
// fragment order of the key-code section kw (see kvq.h).  128 threads.
template <int D, int G, int KBq>
__device__ __forceinline__ void key_codes(const __half* __restrict__ sk, const float4* __restrict__ kp,
                                          uint32_t* __restrict__ kw, int tid) {
  constexpr int DP = D + 8;
  constexpr int QK = (1 << KBq) - 1;
  constexpr int FK = 16 / KBq;               // code pairs per 32-bit word
  constexpr int KWPL = D * KBq / 128;        // key words per lane per 8-token tile
  constexpr int KWORDS = G * D * KBq / 32;
  const __half2* sk2 = reinterpret_cast<const __half2*>(sk);
  {
    // Thread items wi = tid + 128k: lane = wi % 32 varies fastest (a warp
    // reads 8 tokens x 4 channel pairs: 32 distinct banks of the padded
    // rows), then the word w of the lane, then the token tile.  A thread's
    // items share w and the lane, hence one set of channels: their (z, 1/s)
    // are loaded once.
    static_assert(4 % KWPL == 0, "key words of a thread share their channels");
    const int lane = tid % 32;
    const int w = (tid / 32) % KWPL;
    const int i = lane & 3;
    float zk[FK][2], rk[FK][2];
#pragma unroll
    for (int f = 0; f < FK; ++f) {
      const int p = w * FK + f;
      const int c = 16 * (p >> 1) + 8 * (p & 1) + 2 * i;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float4 pc = kp[c + e];
        zk[f][e] = pc.x;
        rk[f][e] = pc.y;
      }
    }
    static_assert(KWORDS % 128 == 0, "whole passes of the 128 threads");
#pragma unroll 1
    for (int pass = 0; pass < KWORDS / 128; ++pass) {
      const int wi = tid + 128 * pass;
      const int nt = wi / (KWPL * 32);
      const int t = 8 * nt + (lane >> 2);
      const int widx = (nt * 32 + lane) * KWPL + w;   // layout word
      uint32_t word = 0;
      bool tie = false;
#pragma unroll
      for (int f = 0; f < FK; ++f) {
        // field f of the low half and of the high half: channels c, c + 1
        const int p = w * FK + f;
        const int c = 16 * (p >> 1) + 8 * (p & 1) + 2 * i;
        const float2 x = __half22float2(sk2[(t * DP + c) >> 1]);
        uint32_t c0, c1;
        codes2(x.x, x.y, zk[f][0], zk[f][1], rk[f][0], rk[f][1], QK, c0, c1, tie);
        word |= ((c0 & QK) << (KBq * f)) | ((c1 & QK) << (KBq * (FK + f)));
      }
      if (tie) word = key_word_exact<D, KBq>(sk, kp, t, w, i);   // rare
      kw[widx] = word;
    }
  }
}

// PLAIN: fp16 inputs into a cache with no recent window, no sink window, no
// rotation and one key width (the common case, compiled without the code of
// the others).
template <int D, int G, int KB, int VB, bool PLAIN>
__global__ void __launch_bounds__(128) append_kernel(const Geom g, unsigned char* __restrict__ cache,
                                                     const void* __restrict__ kin,
                                                     const void* __restrict__ vin, const int dtype_arg,
                                                     const AppendSeqs s) {
  using C = AppCfg<D, G, KB, VB>;
  extern __shared__ __align__(16) unsigned char sm[];
  const int dtype = PLAIN ? (int)KVQ_FP16 : dtype_arg;
  const int g_sink = PLAIN ? 0 : g.sink;
  const int g_window = PLAIN ? 0 : g.window;
  const int g_akvq = PLAIN ? 0 : g.akvq_delta;
  __half* sk = reinterpret_cast<__half*>(sm + C::SM_K);
  __half* sv = reinterpret_cast<__half*>(sm + C::SM_V);
  __half* ks = reinterpret_cast<__half*>(sm + C::SM_KS);
  __half* kz = reinterpret_cast<__half*>(sm + C::SM_KZ);
  __half* vs = reinterpret_cast<__half*>(sm + C::SM_VS);
  __half* vz = reinterpret_cast<__half*>(sm + C::SM_VZ);

  // a decode launched next as a programmatic dependent may start launching
  // now; it waits for this grid's completion before it reads the cache
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x;
  const int task = blockIdx.x;
  const int kvh = blockIdx.y;
  // sequence owning this task: largest b with task_prefix[b] <= task
  int lo = 0, hi = s.n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.task_prefix[mid] <= task) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int tau = task - s.task_prefix[b];
  const int seq = s.seq0 + b;
  int32_t* lens = reinterpret_cast<int32_t*>(cache + g.lens_off);
  int32_t* tickets = reinterpret_cast<int32_t*>(cache + g.counters_off);
  const int nn = s.n_new[b];
  const int seq_ctas = (s.task_prefix[b + 1] - s.task_prefix[b]) * gridDim.y;
  // The sequence's current length: read once (thread 0, acquire), then
  // counted on the sequence's ticket.  The CTA that counts last has seen
  // every other CTA of the sequence read the length, so it may publish the
  // new one (below, after its acquire count: no later read of the old value
  // can see it); nothing else of this launch reads the length.  No fence
  // orders the cache writes: the next kernel on the stream sees them all.
  __shared__ int32_t len_s;
  int ticket_old = -1;
  // launched as a programmatic dependent of the previous kernel on the
  // stream (the decode of the previous step, typically): the planning above
  // reads only kernel parameters; nothing in memory is read or written
  // before the previous grid has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    const int l0 = ld_acquire_gpu(lens + seq);
    len_s = l0;
    ticket_old = atomic_add_acquire_gpu(tickets + seq, 1);
  }
  __syncthreads();
  const int len0 = len_s;
  const int W = PLAIN ? G : g.tail_slots;   // ring slots of the tail: R + G
  const int n1 = len0 + nn;
  // positions after the sink (q = p - S): a0 before, a1 after this append;
  // the first nsink new tokens (input rows 0 .. nsink-1) go to the sink
  const int a0 = max(len0 - g_sink, 0);
  const int a1 = max(n1 - g_sink, 0);
  const int nsink = PLAIN ? 0 : max(min(n1, g_sink) - len0, 0);
  const int N0 = G * quantized_groups(a0, G, g_window);
  const int T0 = a0 - N0;          // tail length before
  const int N1 = G * quantized_groups(a1, G, g_window);
  const int F = (N1 - N0) / G;     // groups completed by this append
  const int64_t row0 = s.row_off[b];
  const int64_t unit = (int64_t)seq * g.hkv + kvh;
  __half* tailk = reinterpret_cast<__half*>(cache + g.tails_off + unit * g.tail_bytes);
  __half* tailv = tailk + (int64_t)W * D;
  const int base0 = N0 % W;        // ring slot of post-sink position N0
  auto in_idx = [&](int64_t r, int c) { return ((row0 + r) * g.hkv + kvh) * D + c; };
  // A replayed capture can ask for more than the capacity, which the host
  // could not check: such an append writes nothing and the length stays.
  const bool fits = (int64_t)len0 + nn <= g.max_tokens;
  // the CTA that counted last publishes the new length and re-arms the ticket
  auto finish = [&]() {
    if (tid == 0 && ticket_old == seq_ctas - 1) {
      if (fits) lens[seq] = len0 + nn;
      tickets[seq] = 0;
    }
  };
  if (!fits) {
    finish();
    return;
  }

  constexpr int CPR = D / 8;   // 16-byte fp16 chunks per token row
  // new sink tokens: input row j -> sink slot len0 + j (nobody reads them here)
  const bool rot = PLAIN ? false : g.rotate != 0;
  // The loops over input rows below run whole warps (row_chunk16 exchanges
  // across a warp when the cache rotates); a lane past the end loads nothing.
  auto write_sink = [&]() {
    __half* sinkk = reinterpret_cast<__half*>(cache + g.sinks_off + unit * g.sink_bytes);
    __half* sinkv = sinkk + (int64_t)g.sink_slots * D;
    for (int c0 = tid - tid % 32; c0 < nsink * CPR; c0 += blockDim.x) {
      const int ci = c0 + tid % 32;
      const bool act = ci < nsink * CPR;
      const int j = act ? ci / CPR : 0, cc = ci % CPR;
      const uint4 k8 = row_chunk16<D>(kin, in_idx(j, 8 * cc), dtype, cc, act, rot);
      const uint4 v8 = row_chunk16<D>(vin, in_idx(j, 8 * cc), dtype, cc, act, rot);
      if (act) store_tail8(sinkk, sinkv, len0 + j, cc, D, k8, v8);
    }
  };
  // Position-adaptive key bits: the tasks after the append's own (max(F, 1))
  // requantize the 4-bit key groups that this append moves from the recent
  // region into the middle ("Asymmetric Key-Value Quantization: 2-Bit
  // Values and 4-Bit Keys under Long-Context Drift", §3.2, with the aging
  // rule of this library): keys dequantized to fp16(fp32(s) * code +
  // fp32(z)), quantized again at 2 bits; the value sections move unchanged
  // to their places in the 2-bit block.  The host reserves one such task
  // per sequence for appends of fewer than G tokens (at most one group ages
  // then); a task with no group to age does nothing.
  if constexpr (KB == 4) {
    if (g_akvq && tau >= (F > 0 ? F : 1)) {
      int first;
      const int A = akvq_aging(len0, n1, N0 / G, G, g_akvq, &first);
      const int r = tau - (F > 0 ? F : 1);
      if (r < A) {
        unsigned char* blk = cache + g.blocks_off +
                             (unit * g.max_groups + first + r) * (int64_t)g.block_bytes;
        const unsigned char* kc4 = blk + g.sec_kcodes;
        const __half* ks4 = reinterpret_cast<const __half*>(blk + g.sec_kscale);
        const __half* kz4 = reinterpret_cast<const __half*>(blk + g.sec_kmin);
        constexpr int LB = D * 4 / 32;   // key-code bytes per lane per 8-token tile
        for (int idx = tid; idx < G * D; idx += 128) {
          // code (t, c) of the 4-bit key section (layout in kvq.h)
          const int t = idx / D, c = idx % D;
          const int nt = t >> 3, rr = t & 7, kt = c >> 4, v = (c >> 3) & 1, i = (c >> 1) & 3,
                    e = c & 1;
          const int p = 2 * kt + v;
          const uint32_t word = *reinterpret_cast<const uint32_t*>(
              kc4 + nt * 32 * LB + (4 * rr + i) * LB + 4 * (p / 4));
          const uint32_t code = (word >> (4 * (p % 4 + 4 * e))) & 15u;
          const int slot = i * (D / 4) + 4 * kt + 2 * v + e;
          const float x = __fadd_rn(__fmul_rn(__half2float(ks4[slot]), (float)code),
                                    __half2float(kz4[slot]));
          sk[t * C::DP + c] = __float2half_rn(x);
        }
        // the value sections, kept in the (unused) value staging area
        unsigned char* vkeep = reinterpret_cast<unsigned char*>(sv);
        constexpr int VBYTES = G * D * VB / 8 + 4 * G * C::J;   // codes, scales, mins
        static_assert(VBYTES % 16 == 0 && VBYTES <= 2 * G * (D + 8), "value sections fit the area");
        for (int i = tid * 16; i < VBYTES; i += 128 * 16)
          *reinterpret_cast<uint4*>(vkeep + i) = *reinterpret_cast<const uint4*>(blk + g.sec_vcodes + i);
        __syncthreads();   // every read of the old block is done
        float4* kp = reinterpret_cast<float4*>(sm + C::SM_KP);
        uint2* kr = reinterpret_cast<uint2*>(sm + C::SM_KR);
        key_stats_part<D, G>(sk, kr, tid);
        __syncthreads();
        if (tid < D) key_stats_final<D, G, 3>(kr, kp, ks, kz, tid);
        __syncthreads();
        key_codes<D, G, 2>(sk, kp, reinterpret_cast<uint32_t*>(blk), tid);
        for (int i = tid; i < D / 2; i += 128) {
          reinterpret_cast<uint32_t*>(blk + g.a2_kscale)[i] = reinterpret_cast<const uint32_t*>(ks)[i];
          reinterpret_cast<uint32_t*>(blk + g.a2_kmin)[i] = reinterpret_cast<const uint32_t*>(kz)[i];
        }
        for (int i = tid * 16; i < VBYTES; i += 128 * 16)
          *reinterpret_cast<uint4*>(blk + g.a2_vcodes + i) = *reinterpret_cast<const uint4*>(vkeep + i);
      }
      finish();
      return;
    }
  }
  if (F == 0) {
    // no group completes: post-sink position a0 + j (input row nsink + j) goes
    // to ring slot (a0 + j) mod W, which holds no tail token (the tail
    // stays below W)
    write_sink();
    const int sl0 = (base0 + T0) % W;
    for (int c0 = tid - tid % 32; c0 < (a1 - a0) * CPR; c0 += blockDim.x) {
      const int ci = c0 + tid % 32;
      const bool act = ci < (a1 - a0) * CPR;
      const int j = act ? ci / CPR : 0, cc = ci % CPR;
      const uint4 k8 = row_chunk16<D>(kin, in_idx(nsink + j, 8 * cc), dtype, cc, act, rot);
      const uint4 v8 = row_chunk16<D>(vin, in_idx(nsink + j, 8 * cc), dtype, cc, act, rot);
      int sl = sl0 + j;
      sl -= (sl >= W) ? W : 0;
      if (act) store_tail8(tailk, tailv, sl, cc, D, k8, v8);
    }
    finish();
    return;
  }
  if (tau >= F) {   // launch planned for more groups than complete (cannot
    finish();       // happen when the host mirror matches the device lengths)
    return;
  }

  // ---- load the group: post-sink position N0 + u (u = tau*G + r) is old
  // tail token u (ring slot (N0 + u) mod W) or input row nsink + u - T0;
  // 16-byte chunks, every load of a thread issued before its stores
  {
    constexpr int NCH = G * CPR / 128;   // chunks per thread (K and V each)
    uint4 kx[NCH], vx[NCH];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int ci = tid + 128 * j, r = ci / CPR, cc = ci % CPR;
      const int u = tau * G + r;
      const bool from_tail = u < T0;   // the same for the D / 8 lanes of the row
      // every lane takes part in the (possibly rotating) input load
      kx[j] = row_chunk16<D>(kin, in_idx(nsink + (from_tail ? 0 : u - T0), 8 * cc), dtype, cc,
                             !from_tail, rot);
      vx[j] = row_chunk16<D>(vin, in_idx(nsink + (from_tail ? 0 : u - T0), 8 * cc), dtype, cc,
                             !from_tail, rot);
      if (from_tail) {   // the old tail already holds cache tokens
        int sl = base0 + u;
        sl -= (sl >= W) ? W : 0;
        kx[j] = *reinterpret_cast<const uint4*>(tailk + sl * D + 8 * cc);
        vx[j] = tail_v8(tailv, sl, cc, D);
      }
    }
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int ci = tid + 128 * j, r = ci / CPR, cc = ci % CPR;
      reinterpret_cast<uint4*>(sk + r * C::DP)[cc] = kx[j];
      reinterpret_cast<uint4*>(sv + r * C::DP)[cc] = vx[j];
    }
  }
  __syncthreads();

  // key width of this group: the cache's, or with position-adaptive bits
  // the width of its region once this append is done
  const int kbits = (KB == 4 && g_akvq) ? akvq_key_bits(N0 / G + tau, n1, G, g_akvq) : KB;

  // ---- statistics.  Keys: partial fp16x2 min/max per (row slice, channel
  // pair) by every thread, then one channel per thread after a barrier.
  // Values: one (token, group of G channels) item per thread, 16-byte
  // loads.  fp16 min/max of fp16 values is exact.
  float4* kp = reinterpret_cast<float4*>(sm + C::SM_KP);   // [c]: {z, 1/s, s, -}
  float4* vp = reinterpret_cast<float4*>(sm + C::SM_VP);   // [r * J + j]
  uint2* kr = reinterpret_cast<uint2*>(sm + C::SM_KR);
  key_stats_part<D, G>(sk, kr, tid);
  __syncthreads();
  if (tid < D) {
    if (kbits == KB) key_stats_final<D, G, (1 << KB) - 1>(kr, kp, ks, kz, tid);
    else key_stats_final<D, G, 3>(kr, kp, ks, kz, tid);
  }
  {
    static_assert(G * C::J <= 128, "one value item per thread");
    for (int q = tid; q < G * C::J; q += 128) {
      const int r = q / C::J, j = q % C::J;
      const uint4* row = reinterpret_cast<const uint4*>(sv + r * C::DP + j * G);
      constexpr int NV = G / 8;
      uint4 w0 = row[r % NV];
      __half2 mn = *reinterpret_cast<__half2*>(&w0.x), mx = mn;
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const uint4 w = row[(u + r) % NV];   // rotate the start: fewer bank conflicts
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const __half2 x = *reinterpret_cast<const __half2*>(&ws[h]);
          mn = __hmin2(mn, x);
          mx = __hmax2(mx, x);
        }
      }
      const float mnf = fminf(__low2float(mn), __high2float(mn));
      const float mxf = fmaxf(__low2float(mx), __high2float(mx));
      const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mxf, mnf), (float)C::QV));
      const __half z16 = __float2half_rn(mnf);
      const float sf = __half2float(s16);
      vp[q] = make_float4(__half2float(z16), sf == 0.0f ? 0.0f : __frcp_rn(sf), sf, 0.0f);
      // metadata slot ((4kv + i)*J + j)*4 + 2kh + e
      const int kv = r >> 4, kh = (r >> 3) & 1, i = (r >> 1) & 3, e = r & 1;
      const int slot = ((4 * kv + i) * C::J + j) * 4 + 2 * kh + e;
      vs[slot] = s16;
      vz[slot] = z16;
    }
  }
  __syncthreads();

  // ---- codes, quantized and packed word by word into the group block
  unsigned char* blk = cache + g.blocks_off +
                       (unit * g.max_groups + (N0 / G + tau)) * (int64_t)g.block_bytes;
  if (kbits == KB) key_codes<D, G, KB>(sk, kp, reinterpret_cast<uint32_t*>(blk + g.sec_kcodes), tid);
  else key_codes<D, G, 2>(sk, kp, reinterpret_cast<uint32_t*>(blk), tid);
  uint32_t* vw = reinterpret_cast<uint32_t*>(blk + (kbits == KB ? g.sec_vcodes : g.a2_vcodes));
  static_assert(C::VWORDS % 128 == 0, "whole passes of the 128 threads");
#pragma unroll 1
  for (int pass = 0; pass < C::VWORDS / 128; ++pass) {
    const int wi = tid + 128 * pass;
    // lane fastest (a warp reads 4 token pairs x 8 channels: distinct banks
    // of the padded rows), then the lane's word w, then the token tile
    const int lane = wi % 32;
    const int w = (wi / 32) % C::VWORDS_PER_LANE;
    const int kv = wi / (C::VWORDS_PER_LANE * 32);
    const int widx = (kv * 32 + lane) * C::VWORDS_PER_LANE + w;   // layout word
    const int gg = lane >> 2, i = lane & 3;
    uint32_t word = 0;
    bool tie = false;
    // the word's channels 16 mt .. 16 mt + 15 lie in one value group j; its
    // four tokens (kh, e) have one (z, 1/s) each
    const int jw = (16 * (w * (C::FV / 4))) / G;
    float4 pv[2][2];
#pragma unroll
    for (int kh = 0; kh < 2; ++kh)
#pragma unroll
      for (int e = 0; e < 2; ++e) pv[kh][e] = vp[(16 * kv + 8 * kh + 2 * i + e) * C::J + jw];
#pragma unroll
    for (int fl = 0; fl < C::FV; ++fl) {
      // field fl of the low half (token t) and of the high half (token t + 1)
      const int kh = fl / (C::FV / 2), rem = fl % (C::FV / 2);
      const int u = rem >> 1, hr = rem & 1;
      const int mt = w * (C::FV / 4) + u;
      const int c = 16 * mt + 8 * hr + gg;
      const int t = 16 * kv + 8 * kh + 2 * i;
      const float4 p0 = pv[kh][0], p1 = pv[kh][1];
      uint32_t c0, c1;
      codes2(__half2float(sv[t * C::DP + c]), __half2float(sv[(t + 1) * C::DP + c]), p0.x, p1.x,
             p0.y, p1.y, C::QV, c0, c1, tie);
      word |= ((c0 & C::QV) << (VB * fl)) | ((c1 & C::QV) << (VB * (C::FV + fl)));
    }
    if (tie) word = value_word_exact<D, G, VB>(sv, vp, kv, w, gg, i);   // rare
    vw[widx] = word;
  }
  // metadata sections are copied verbatim (already in slot order)
  {
    const uint32_t* src;
    uint32_t* dst;
    const bool full = kbits == KB;   // else a 2-bit key group (position-adaptive bits)
    src = reinterpret_cast<const uint32_t*>(ks);
    dst = reinterpret_cast<uint32_t*>(blk + (full ? g.sec_kscale : g.a2_kscale));
    for (int i = tid; i < D / 2; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint32_t*>(kz);
    dst = reinterpret_cast<uint32_t*>(blk + (full ? g.sec_kmin : g.a2_kmin));
    for (int i = tid; i < D / 2; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint32_t*>(vs);
    dst = reinterpret_cast<uint32_t*>(blk + (full ? g.sec_vscale : g.a2_vscale));
    for (int i = tid; i < G * C::J / 2; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint32_t*>(vz);
    dst = reinterpret_cast<uint32_t*>(blk + (full ? g.sec_vmin : g.a2_vmin));
    for (int i = tid; i < G * C::J / 2; i += blockDim.x) dst[i] = src[i];
  }

  // ---- the new tail: post-sink positions [A, a1), all new tokens (input
  // rows nsink + q - a0).  Ring residue rr = (q - N0) mod W: rr < T0 is the
  // slot of old tail token N0 + rr, which this append quantizes in task
  // rr / G (that task read it before the barrier above), so that task
  // writes the slot; residues T0 .. W-1 hold no old tail token and task 0
  // writes them.  Each residue occurs at most once in [A, a1) (the new tail
  // is shorter than W).  Task 0 also writes the new sink tokens.
  if (tau == 0) write_sink();
  {
    const int A = max(N1, a0);
    const int r_lo = tau * G;
    const int r_hi = min(T0, r_lo + G);
    auto write_residues = [&](int lo, int hi) {
      for (int c0 = tid - tid % 32; c0 < (hi - lo) * CPR; c0 += blockDim.x) {
        const int ci = c0 + tid % 32;
        const int rr = lo + (ci < (hi - lo) * CPR ? ci / CPR : 0), cc = ci % CPR;
        // the post-sink position q >= A with q = N0 + rr (mod W)
        int off = (N0 + rr - A) % W;
        off += (off < 0) ? W : 0;
        const int q = A + off;
        const bool act = ci < (hi - lo) * CPR && q < a1;
        const int64_t r = act ? (int64_t)nsink + q - a0 : 0;
        const uint4 k8 = row_chunk16<D>(kin, in_idx(r, 8 * cc), dtype, cc, act, rot);
        const uint4 v8 = row_chunk16<D>(vin, in_idx(r, 8 * cc), dtype, cc, act, rot);
        if (act) {
          int sl = base0 + rr;
          sl -= (sl >= W) ? W : 0;
          store_tail8(tailk, tailv, sl, cc, D, k8, v8);
        }
      }
    };
    if (r_lo < r_hi) write_residues(r_lo, r_hi);
    if (tau == 0) write_residues(T0, W);
  }
  finish();
}

template <int D, int G, int KB, int VB>
cudaError_t launch_append_t(const Geom& g, unsigned char* cache, const void* k, const void* v,
                            int dtype, const AppendSeqs& seqs, int n_tasks, cudaStream_t stream) {
  using C = AppCfg<D, G, KB, VB>;
  const bool plain = dtype == KVQ_FP16 && g.window == 0 && g.sink == 0 && g.rotate == 0 &&
                     g.akvq_delta == 0;
  auto kern = plain ? append_kernel<D, G, KB, VB, true> : append_kernel<D, G, KB, VB, false>;
  static bool configured[2] = {false, false};   // attribute set once, before any capture
  if (!configured[plain]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SM_TOTAL);
    if (e != cudaSuccess) return e;
    configured[plain] = true;
  }
  // a programmatic dependent of the previous kernel: its CTAs may be
  // resident while that kernel runs, and wait for it (griddepcontrol.wait)
  // before touching memory
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)n_tasks, (unsigned)g.hkv);
  lc.blockDim = dim3(128);
  lc.dynamicSmemBytes = C::SM_TOTAL;
  lc.stream = stream;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  la[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = la;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, g, cache, k, v, dtype, seqs);
}

}  // namespace

cudaError_t launch_append(const Geom& g, unsigned char* cache, const void* k, const void* v,
                          int dtype, const AppendSeqs& seqs, int n_tasks, cudaStream_t stream) {
#define KVQ_APPEND_CASE(D_, G_, KB_, VB_)                                              \
  if (g.d == D_ && g.G == G_ && g.kb == KB_ && g.vb == VB_)                            \
    return launch_append_t<D_, G_, KB_, VB_>(g, cache, k, v, dtype, seqs, n_tasks, stream);
#define KVQ_APPEND_BITS(D_, G_) \
  KVQ_APPEND_CASE(D_, G_, 4, 2) KVQ_APPEND_CASE(D_, G_, 2, 2) \
  KVQ_APPEND_CASE(D_, G_, 4, 4) KVQ_APPEND_CASE(D_, G_, 2, 4)
  KVQ_APPEND_BITS(128, 32)
  KVQ_APPEND_BITS(128, 64)
  KVQ_APPEND_BITS(64, 32)
  KVQ_APPEND_BITS(64, 64)
#undef KVQ_APPEND_BITS
#undef KVQ_APPEND_CASE
  return cudaErrorInvalidValue;
}

}  // namespace kvq
