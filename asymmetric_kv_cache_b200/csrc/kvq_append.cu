// Append kernel of libkvq: per-channel key quantization, per-token value
// quantization, bit packing into LAYOUT v1, the fp16 tail and its flush.
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
// into the tail.  The task that quantizes the first completed group of a
// sequence also writes that sequence's new tail, after it has read the old
// one, so no other CTA touches the tail concurrently.
//
// Every CTA reads the sequence's current length from the device copy when
// it starts; the last CTA of the sequence to finish (atomic ticket in the
// cache buffer, no waiting) stores the new length and re-arms the ticket.
// All reads of the old length therefore precede its update.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

template <int D, int G, int KB, int VB>
struct AppCfg {
  static constexpr int J = D / G;
  static constexpr int QK = (1 << KB) - 1;
  static constexpr int QV = (1 << VB) - 1;
  static constexpr int FK = 16 / KB;           // code pairs per 32-bit word
  static constexpr int FV = 16 / VB;
  static constexpr int KWORDS_PER_LANE = D * KB / 128;   // per 8-token tile
  static constexpr int VWORDS_PER_LANE = D * VB / 64;    // per 16-token tile
  static constexpr int KWORDS = G * D * KB / 32;
  static constexpr int VWORDS = G * D * VB / 32;
  // dynamic shared memory: fp16 K and V of the group, their codes, metadata
  static constexpr int SM_K = 0;
  static constexpr int SM_V = SM_K + 2 * G * D;
  static constexpr int SM_KC = SM_V + 2 * G * D;
  static constexpr int SM_VC = SM_KC + G * D;
  static constexpr int SM_KS = SM_VC + G * D;
  static constexpr int SM_KZ = SM_KS + 2 * D;
  static constexpr int SM_VS = SM_KZ + 2 * D;
  static constexpr int SM_VZ = SM_VS + 2 * G * J;
  static constexpr int SM_TOTAL = SM_VZ + 2 * G * J;
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

template <int D, int G, int KB, int VB>
__global__ void __launch_bounds__(128) append_kernel(const Geom g, unsigned char* __restrict__ cache,
                                                     const void* __restrict__ kin,
                                                     const void* __restrict__ vin, const int dtype,
                                                     const AppendSeqs s) {
  using C = AppCfg<D, G, KB, VB>;
  extern __shared__ __align__(16) unsigned char sm[];
  __half* sk = reinterpret_cast<__half*>(sm + C::SM_K);
  __half* sv = reinterpret_cast<__half*>(sm + C::SM_V);
  uint8_t* kc = sm + C::SM_KC;
  uint8_t* vc = sm + C::SM_VC;
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
  const int len0 = *reinterpret_cast<volatile int32_t*>(lens + seq);
  const int nn = s.n_new[b];
  const int seq_ctas = (s.task_prefix[b + 1] - s.task_prefix[b]) * gridDim.y;
  const int T0 = len0 % G;
  const int N0 = len0 - T0;
  const int F = (T0 + nn) / G;     // groups completed by this append
  const int T1 = (T0 + nn) % G;    // tail length afterwards
  const int64_t row0 = s.row_off[b];
  const int64_t unit = (int64_t)seq * g.hkv + kvh;
  __half* tailk = reinterpret_cast<__half*>(cache + g.tails_off + unit * g.tail_bytes);
  __half* tailv = tailk + G * D;
  auto in_idx = [&](int64_t r, int c) { return ((row0 + r) * g.hkv + kvh) * D + c; };
  // A replayed capture can ask for more than the capacity, which the host
  // could not check: such an append writes nothing and the length stays.
  const bool fits = (int64_t)len0 + nn <= g.max_tokens;
  // the last CTA of this sequence to finish publishes the new length
  auto finish = [&]() {
    __syncthreads();
    if (tid == 0 && atomic_add_acq_rel_gpu(tickets + seq, 1) == seq_ctas - 1) {
      if (fits) lens[seq] = len0 + nn;
      tickets[seq] = 0;
    }
  };
  if (!fits) {
    finish();
    return;
  }

  constexpr int CPR = D / 8;   // 16-byte fp16 chunks per token row
  if (F == 0) {
    // no group completes: new tokens go to tail slots T0 .. T0 + nn - 1
    for (int ci = tid; ci < nn * CPR; ci += blockDim.x) {
      const int j = ci / CPR, cc = ci % CPR;
      store_tail8(tailk, tailv, T0 + j, cc, D, load8_fp16(kin, in_idx(j, 8 * cc), dtype),
                  load8_fp16(vin, in_idx(j, 8 * cc), dtype));
    }
    finish();
    return;
  }
  if (tau >= F) {   // launch planned for more groups than complete (cannot
    finish();       // happen when the host mirror matches the device lengths)
    return;
  }

  // ---- load the group: virtual token u = tau*G + r of [old tail ++ input],
  // 16-byte chunks, every load of a thread issued before its stores
  {
    constexpr int NCH = G * CPR / 128;   // chunks per thread (K and V each)
    uint4 kx[NCH], vx[NCH];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int ci = tid + 128 * j, r = ci / CPR, cc = ci % CPR;
      const int u = tau * G + r;
      if (u < T0) {
        kx[j] = *reinterpret_cast<const uint4*>(tailk + u * D + 8 * cc);
        vx[j] = tail_v8(tailv, u, cc, D);
      } else {
        kx[j] = load8_fp16(kin, in_idx(u - T0, 8 * cc), dtype);
        vx[j] = load8_fp16(vin, in_idx(u - T0, 8 * cc), dtype);
      }
    }
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int ci = tid + 128 * j;
      reinterpret_cast<uint4*>(sk)[ci] = kx[j];
      reinterpret_cast<uint4*>(sv)[ci] = vx[j];
    }
  }
  __syncthreads();

  // ---- keys: one (scale, min) per channel over the G tokens
  for (int c = tid; c < D; c += blockDim.x) {
    float mn = __half2float(sk[c]), mx = mn;
    for (int r = 1; r < G; ++r) {
      const float x = __half2float(sk[r * D + c]);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)C::QK));
    const __half z16 = __float2half_rn(mn);
    const float sf = __half2float(s16), zf = __half2float(z16);
    for (int r = 0; r < G; ++r) kc[r * D + c] = (uint8_t)quant_code(__half2float(sk[r * D + c]), zf, sf, C::QK);
    // metadata slot i*(D/4) + 4kt + 2v + e
    const int kt = c >> 4, v = (c >> 3) & 1, i = (c >> 1) & 3, e = c & 1;
    const int slot = i * (D / 4) + 4 * kt + 2 * v + e;
    ks[slot] = s16;
    kz[slot] = z16;
  }
  // ---- values: one (scale, min) per (token, group of G channels)
  for (int q = tid; q < G * C::J; q += blockDim.x) {
    const int r = q / C::J, j = q % C::J;
    const __half* row = sv + r * D + j * G;
    // start each thread at a different channel to spread shared-memory banks
    float mn = __half2float(row[r % G]), mx = mn;
    for (int k = 1; k < G; ++k) {
      const float x = __half2float(row[(k + r) % G]);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)C::QV));
    const __half z16 = __float2half_rn(mn);
    const float sf = __half2float(s16), zf = __half2float(z16);
    for (int k = 0; k < G; ++k) {
      const int kk = (k + r) % G;
      vc[r * D + j * G + kk] = (uint8_t)quant_code(__half2float(row[kk]), zf, sf, C::QV);
    }
    // metadata slot ((4kv + i)*J + j)*4 + 2kh + e
    const int kv = r >> 4, kh = (r >> 3) & 1, i = (r >> 1) & 3, e = r & 1;
    const int slot = ((4 * kv + i) * C::J + j) * 4 + 2 * kh + e;
    vs[slot] = s16;
    vz[slot] = z16;
  }
  __syncthreads();

  // ---- pack into the group block
  unsigned char* blk = cache + g.blocks_off +
                       (unit * g.max_groups + (N0 / G + tau)) * (int64_t)g.block_bytes;
  uint32_t* kw = reinterpret_cast<uint32_t*>(blk + g.sec_kcodes);
  for (int wi = tid; wi < C::KWORDS; wi += blockDim.x) {
    const int w = wi % C::KWORDS_PER_LANE;
    const int lane = (wi / C::KWORDS_PER_LANE) % 32;
    const int nt = wi / (C::KWORDS_PER_LANE * 32);
    const int t = 8 * nt + (lane >> 2), i = lane & 3;
    uint32_t word = 0;
#pragma unroll
    for (int fp = 0; fp < 32 / KB; ++fp) {
      const int e = fp / C::FK, f = fp % C::FK;
      const int p = w * C::FK + f;
      const int c = 16 * (p >> 1) + 8 * (p & 1) + 2 * i + e;
      word |= (uint32_t)kc[t * D + c] << (KB * fp);
    }
    kw[wi] = word;
  }
  uint32_t* vw = reinterpret_cast<uint32_t*>(blk + g.sec_vcodes);
  for (int wi = tid; wi < C::VWORDS; wi += blockDim.x) {
    const int w = wi % C::VWORDS_PER_LANE;
    const int lane = (wi / C::VWORDS_PER_LANE) % 32;
    const int kv = wi / (C::VWORDS_PER_LANE * 32);
    const int gg = lane >> 2, i = lane & 3;
    uint32_t word = 0;
#pragma unroll
    for (int fp = 0; fp < 32 / VB; ++fp) {
      const int e = fp / C::FV, fl = fp % C::FV;
      const int kh = fl / (C::FV / 2), rem = fl % (C::FV / 2);
      const int u = rem >> 1, hr = rem & 1;
      const int mt = w * (C::FV / 4) + u;
      const int c = 16 * mt + 8 * hr + gg;
      const int t = 16 * kv + 8 * kh + 2 * i + e;
      word |= (uint32_t)vc[t * D + c] << (VB * fp);
    }
    vw[wi] = word;
  }
  // metadata sections are copied verbatim (already in slot order)
  {
    const uint32_t* src;
    uint32_t* dst;
    src = reinterpret_cast<const uint32_t*>(ks);
    dst = reinterpret_cast<uint32_t*>(blk + g.sec_kscale);
    for (int i = tid; i < D / 2; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint32_t*>(kz);
    dst = reinterpret_cast<uint32_t*>(blk + g.sec_kmin);
    for (int i = tid; i < D / 2; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint32_t*>(vs);
    dst = reinterpret_cast<uint32_t*>(blk + g.sec_vscale);
    for (int i = tid; i < G * C::J / 2; i += blockDim.x) dst[i] = src[i];
    src = reinterpret_cast<const uint32_t*>(vz);
    dst = reinterpret_cast<uint32_t*>(blk + g.sec_vmin);
    for (int i = tid; i < G * C::J / 2; i += blockDim.x) dst[i] = src[i];
  }

  if (tau == 0) {
    // the new tail: virtual tokens F*G .. F*G + T1 - 1, all from the input
    // (the old tail was fully read above, before the barrier)
    for (int ci = tid; ci < T1 * CPR; ci += blockDim.x) {
      const int t = ci / CPR, cc = ci % CPR;
      const int64_t r = (int64_t)F * G + t - T0;
      store_tail8(tailk, tailv, t, cc, D, load8_fp16(kin, in_idx(r, 8 * cc), dtype),
                  load8_fp16(vin, in_idx(r, 8 * cc), dtype));
    }
  }
  finish();
}

template <int D, int G, int KB, int VB>
cudaError_t launch_append_t(const Geom& g, unsigned char* cache, const void* k, const void* v,
                            int dtype, const AppendSeqs& seqs, int n_tasks, cudaStream_t stream) {
  using C = AppCfg<D, G, KB, VB>;
  auto kern = append_kernel<D, G, KB, VB>;
  static bool configured = false;   // attribute set once, before any capture
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SM_TOTAL);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(n_tasks, g.hkv);
  kern<<<grid, 128, C::SM_TOTAL, stream>>>(g, cache, k, v, dtype, seqs);
  return cudaGetLastError();
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
