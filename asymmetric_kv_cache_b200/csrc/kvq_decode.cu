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
// same number of slots whatever the lengths are); the grid is one CTA per SM.
// Inside a CTA the 12-16 warps claim the groups of the current unit piece
// one at a time from a shared counter (so warps that the schedulers favour
// simply take more groups and all finish together), each with its own
// online softmax, and merge through shared memory at the end of the piece.
// A unit cut by CTA boundaries writes per-piece partials (m, l, o): the
// last of its CTAs merges them (acquire-release ticket; wide CTAs with at
// most 32 pieces per unit), else the combine kernel does.  With a rotating
// cache the query rows are rotated before the fp16 split and every final
// output row is rotated back; with position-adaptive key widths each group
// is copied and read at its own width.
//
// Per group (one 32/64-token slot) a warp:
//   * waits for the group block, brought into its own shared-memory ring by
//     a 1-D bulk (TMA) copy issued NST groups ahead;
//   * folds the per-channel key scales into the query: q'_c = q_c s_c, so
//     q . k_hat = sum_c q'_c code_c + sum_c q_c z_c, the second sum (the
//     key-min bias, one per group and head) on the tensor core as well;
//   * runs S = q' codes^T on m16n8k16 tiles whose 16 rows are the 8 query
//     heads of the GQA group twice: rows 0-7 carry q' rounded to fp16 and
//     rows 8-15 the rounding residual, so the logits keep ~22 bits of q'
//     at no extra tile; the 8 columns are 8 tokens, so a lane ends up with
//     two tokens of one head per tile;
//   * updates the running max / rescales, exponentiates (exp2 domain) and
//     packs P to fp16: the accumulator layout of S is already the B-operand
//     layout of the value product;
//   * runs O^T += V_code^T (p s_v) on tiles whose rows are channels and whose
//     columns are heads, with the per-token value scale folded into p for
//     each channel group, and sum_t p_t z_t (value mins) and sum_t p_t (the
//     softmax denominator) on one more tile.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>

#include "kvq_decode_kernels.cuh"

namespace kvq {
namespace {

#include "kvq_decode_tc.cuh"

// ---------------------------------------------------------------------------
// fp16 decode baseline (comparison).  The same attention over an
// unquantized fp16 cache K, V laid out [n_seq][Hkv][max_tokens][d]: 512 B
// per token-head at d = 128, four times the K4/V2 bytes ("non-quantized
// baseline" of the InnerQ abstract on the "WUSH-KV" page; the first page's
// FlashDecoding baseline, §IV).  Same split: stream-K over one wide CTA per
// SM, units of (sequence, kv head, <= 8 heads), slots of 16 tokens claimed
// dynamically by the warps, fp16 high/low query on the tensor core, online
// softmax, shared-memory merge, combine_kernel for split units.  Chunks are
// staged by cp.async into padded rows (conflict-free fragment reads); the
// V^T fragments come from token-major rows through ldmatrix.trans.
template <int D>
struct F16Cfg {
  static constexpr int NW = 8;
  static constexpr int THREADS = NW * 32;
  static constexpr int CH = 16;                 // tokens per slot
  static constexpr int ROW = 2 * D + 16;        // padded bytes per token row
  static constexpr int STAGE = 2 * CH * ROW;    // K rows then V rows
  static constexpr int NST = 2;
  static constexpr int RING = NW * NST * STAGE;
  static constexpr int KT = D / 16, MT = D / 16;
  static constexpr int QA_OFF = RING;
  static constexpr int QA_BYTES = KT * 32 * 16;
  static_assert(kHeadsPerSlice * D * 4 <= QA_BYTES, "raw query rows fit the fragment area");
  static constexpr int MERGE_FLOATS = NW * kHeadsPerSlice * (D + 2);
  static constexpr int WTS_OFF = MERGE_FLOATS;
  static_assert((MERGE_FLOATS + (NW + 2) * kHeadsPerSlice) * 4 <= RING, "merge area fits");
  static constexpr int BAR_OFF = QA_OFF + QA_BYTES;
  static constexpr int SMEM_FIXED = BAR_OFF + 64;
};

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copy tokens [t0, t0 + 16) of one (sequence, kv head) row block into a
// stage (rows past `T` zero-filled); one commit group.
template <int D>
__device__ __forceinline__ void f16_stage(unsigned char* __restrict__ st,
                                          const __half* __restrict__ k,
                                          const __half* __restrict__ v, int t0, int T, int lane) {
  using F = F16Cfg<D>;
  constexpr int SEGS = F::CH * (D / 8);   // 16-byte pieces per matrix
  for (int seg = lane; seg < 2 * SEGS; seg += 32) {
    const int m = seg / SEGS, r = (seg % SEGS) / (D / 8), cs = seg % (D / 8);
    const int t = t0 + r;
    const __half* src = (m ? v : k) + (t < T ? (int64_t)t * D + cs * 8 : 0);
    cp_async16(st + m * F::CH * F::ROW + r * F::ROW + cs * 16, src, t < T ? 16u : 0u);
  }
  cp_async_commit();
}

// Attention over one staged 16-token slot (tokens t0.. of the unit; those
// at or past T masked out).
template <int D, bool PK>
__device__ __forceinline__ void f16_slot(WarpState<D, 4, 2, 32, PK>& st,
                                         const unsigned char* __restrict__ buf, int t0, int T,
                                         const uint4* __restrict__ qsm, int lane) {
  using F = F16Cfg<D>;
  const int g8 = lane >> 2, i4 = lane & 3;
  const unsigned char* kb = buf;
  const unsigned char* vbuf = buf + F::CH * F::ROW;
  uint32_t pt[2];
  if constexpr (PK) {
    // S^T = K q^T: rows 16 tokens, columns q_hi (n < 4) / q_lo (n >= 4): the
    // lanes' x words
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const unsigned char* k0 = kb + g8 * F::ROW + 4 * i4;
    const unsigned char* k1 = k0 + 8 * F::ROW;
#pragma unroll
    for (int kt = 0; kt < F::KT; ++kt) {
      const uint4 q4 = qsm[kt * 32 + lane];
      mma16816(acc, *reinterpret_cast<const uint32_t*>(k0 + 32 * kt),
               *reinterpret_cast<const uint32_t*>(k1 + 32 * kt),
               *reinterpret_cast<const uint32_t*>(k0 + 32 * kt + 16),
               *reinterpret_cast<const uint32_t*>(k1 + 32 * kt + 16), q4.y, q4.w);
    }
    float s[1][4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float x = acc[r] + __shfl_xor_sync(0xffffffffu, acc[r], 2);
      s[0][r] = (t0 + g8 + (r < 2 ? 0 : 8) < T) ? x : -INFINITY;
    }
    uint32_t p2[1][2];
    softmax_pk<D, 1, 4, 2, 32>(st, s, p2);
    pt[0] = p2[0][0];
    pt[1] = p2[0][1];
  } else {
    // S = q K^T: rows q high / low parts, columns 8 tokens per tile
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const unsigned char* k0 = kb + g8 * F::ROW + 4 * i4;
#pragma unroll
    for (int kt = 0; kt < F::KT; ++kt) {
      const uint4 q4 = qsm[kt * 32 + lane];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const unsigned char* kr = k0 + 8 * nt * F::ROW + 32 * kt;
        mma16816(acc[nt], q4.x, q4.y, q4.z, q4.w, *reinterpret_cast<const uint32_t*>(kr),
                 *reinterpret_cast<const uint32_t*>(kr + 16));
      }
    }
    float s[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int t = t0 + 8 * nt + 2 * i4;
      s[nt][0] = (t < T) ? acc[nt][0] + acc[nt][2] : -INFINITY;
      s[nt][1] = (t + 1 < T) ? acc[nt][1] + acc[nt][3] : -INFINITY;
    }
    softmax_update<D, 2, 4, 2, 32>(st, s, pt, i4);
  }
  // denominator: row 0 of the Z tile
  const uint32_t ones = (g8 == 0) ? 0x3C003C00u : 0u;
  mma16816(st.z, ones, 0u, ones, 0u, pt[0], pt[1]);
  // O^T += V^T P^T, V^T fragments by transposed matrix loads of the
  // token-major rows; rows past T are zero (their p is 0)
  const int r8 = lane & 7, mj = lane >> 3;
  const unsigned char* vrow = vbuf + (r8 + 8 * (mj >> 1)) * F::ROW + 16 * (mj & 1);
#pragma unroll
  for (int mt = 0; mt < F::MT; ++mt) {
    uint32_t a[4];
    ldmatrix_x4_trans(a, vrow + 32 * mt);
    mma16816(st.o[mt], a[0], a[1], a[2], a[3], pt[0], pt[1]);
  }
}

template <int D, bool PK>
__global__ void __launch_bounds__(F16Cfg<D>::THREADS, 1)
    f16_decode_kernel(const Geom g, const WsLayout w, const DecodeArgs a,
                      const __half* __restrict__ kc, const __half* __restrict__ vc,
                      const int32_t* __restrict__ lens_all, int max_tokens) {
  using F = F16Cfg<D>;
  constexpr int NW = F::NW;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int32_t wsum[NW];
  __shared__ int32_t claim;
  uint64_t* qbar = reinterpret_cast<uint64_t*>(smem + F::BAR_OFF);
  uint4* qsm = reinterpret_cast<uint4*>(smem + F::QA_OFF);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + F::SMEM_FIXED);
  int32_t* slen = prefix + (a.n_seq + 1);
  float* merge = reinterpret_cast<float*>(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, i4 = lane & 3;
  const int n_seq = a.n_seq;
  const int per_seq_units = g.hkv * g.slices;
  const int32_t* lens = lens_all + a.seq0;
  int32_t* err = reinterpret_cast<int32_t*>(a.ws + w.err_off);
  float* partials = reinterpret_cast<float*>(a.ws + w.partials_off);

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");   // as in decode_kernel
  if (tid == 0) {
    mbar_init(qbar, 1);
    fence_mbar_init();
    prefix[0] = 0;
    claim = 0;
  }
  {
    const int chunk = (n_seq + F::THREADS - 1) / F::THREADS;
    const int b0 = tid * chunk, b1 = min(n_seq, b0 + chunk);
    int32_t run = 0;
    // lengths outside [0, max_tokens] are clamped: never an access past the rows
    for (int bb = b0; bb < b1; ++bb)
      run += per_seq_units * ((min(max(lens[bb], 0), max_tokens) + F::CH - 1) / F::CH);
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
      const int L = min(max(lens[bb], 0), max_tokens);
      acc += per_seq_units * ((L + F::CH - 1) / F::CH);
      prefix[bb + 1] = acc;
      slen[bb] = L;
    }
  }
  __syncthreads();
  const int T = prefix[n_seq];
  const int grid = gridDim.x;
  const int k = blockIdx.x;
  int start, end;
  cta_range(k, T, grid, &start, &end);
  if (start == end && tid < kHeadsPerSlice) {
    // an empty range (more CTAs than slots): the split record of a unit
    // counts every CTA between its first and its last slot, so publish an
    // empty piece (m = -inf, l = 0) that the combine skips
    float* ps = partials + (int64_t)(2 * k) * w.slot_floats + tid * (D + 4);
    ps[D] = -INFINITY;
    ps[D + 1] = 0.f;
  }
  int head = 0;
  uint32_t qphase = 0;
  unsigned char* wst = smem + warp * F::NST * F::STAGE;

  for (int pos = start; pos < end;) {
    WarpState<D, 4, 2, 32, PK> st;
#pragma unroll
    for (int mt = 0; mt < F::MT; ++mt) st.o[mt][0] = st.o[mt][1] = st.o[mt][2] = st.o[mt][3] = 0.f;
    st.z[0] = st.z[1] = st.z[2] = st.z[3] = 0.f;
#pragma unroll
    for (int r = 0; r < (PK ? 2 : 1); ++r) st.m[r] = -INFINITY;
    // the piece: slots [s0, s1) of unit (b, kvh, slice), slot = 16 tokens
    const int b = find_seq(prefix, n_seq, pos);
    const int L = slen[b];
    const int wb = (L + F::CH - 1) / F::CH;
    const int local = pos - prefix[b];
    const int uis = local / wb;
    const int s0 = local - uis * wb, s1 = min(wb, s0 + (end - pos));
    const int kvh = uis / g.slices, slice = uis - kvh * g.slices;
    const int hbase = kvh * g.gqa + slice * kHeadsPerSlice;
    const int nh = min(kHeadsPerSlice, g.gqa - slice * kHeadsPerSlice);
    const int64_t row0 = ((int64_t)(a.seq0 + b) * g.hkv + kvh) * max_tokens;
    const __half* kr = kc + row0 * D;
    const __half* vr = vc + row0 * D;
    if (tid == 0) {
      const int esz = a.q_dtype == KVQ_FP32 ? 4 : 2;
      const uint32_t qbytes = (uint32_t)(nh * D * esz);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(qbar, qbytes);
      bulk_copy_g2s(qsm, static_cast<const unsigned char*>(a.q) + ((int64_t)b * g.hq + hbase) * D * esz,
                    qbytes, qbar);
    }
    const int nsl = s1 - s0;
    auto claim_into = [&](int stg) -> int {
      int c = -1;
      if (lane == 0) c = atomicAdd(&claim, 1);
      c = __shfl_sync(0xffffffffu, c, 0);
      if (c >= nsl) return -1;
      f16_stage<D>(wst + stg * F::STAGE, kr, vr, (s0 + c) * F::CH, L, lane);
      return c;
    };
    int cur = claim_into(head);
    int nxt = cur >= 0 ? claim_into(head ^ 1) : -1;
    {
      constexpr int NCW = (NW < D / 16) ? NW : D / 16;   // converting warps
      if (warp < NCW) {
        bool got = mbar_wait_bounded(qbar, qphase & 1);
        got = __all_sync(0xffffffffu, got);
        if (!got && lane == 0) atomicExch(err, KVQ_ERR_DEVICE);
        convert_query<D, PK, NCW>(a.q_dtype, nh, got, warp, lane, qsm,
                                  reinterpret_cast<const unsigned char*>(qsm));
      }
    }
    ++qphase;
    __syncthreads();
    while (cur >= 0) {
      if (nxt >= 0) cp_async_wait<1>(); else cp_async_wait<0>();
      __syncwarp();
      f16_slot<D, PK>(st, wst + head * F::STAGE, (s0 + cur) * F::CH, L, qsm, lane);
      __syncwarp();
      const int nn = nxt >= 0 ? claim_into(head) : -1;
      cur = nxt;
      nxt = nn;
      head ^= 1;
    }
    cp_async_wait<0>();

    // ---- merge the warps
    __syncthreads();
    if (tid == 0) claim = 0;
    {
      float* mo = merge + (warp * kHeadsPerSlice) * (D + 2);
      const float l0 = __shfl_sync(0xffffffffu, st.z[0], i4);   // row 0: the sums
      const float l1 = __shfl_sync(0xffffffffu, st.z[1], i4);
      if (!PK || i4 < 2) {
#pragma unroll
        for (int mt = 0; mt < F::MT; ++mt) {
          const int c0 = 16 * mt + g8, c1 = c0 + 8;
          mo[(2 * i4) * (D + 2) + c0] = st.o[mt][0];
          mo[(2 * i4 + 1) * (D + 2) + c0] = st.o[mt][1];
          mo[(2 * i4) * (D + 2) + c1] = st.o[mt][2];
          mo[(2 * i4 + 1) * (D + 2) + c1] = st.o[mt][3];
        }
      }
      if constexpr (PK) {
        if (g8 == 0 && i4 < 2) {
          mo[(2 * i4) * (D + 2) + D] = st.m[0];
          mo[(2 * i4 + 1) * (D + 2) + D] = st.m[1];
        }
      } else {
        if (i4 == 0) mo[g8 * (D + 2) + D] = st.m[0];
      }
      if (g8 == 0) {
        mo[(2 * i4) * (D + 2) + D + 1] = l0;
        mo[(2 * i4 + 1) * (D + 2) + D + 1] = l1;
      }
    }
    __syncthreads();
    const bool whole = (s0 == 0 && s1 == wb);
    float* wts = merge + F::WTS_OFF;
    merge_weights<D, NW>(merge, wts, whole, tid);
    const int myslot = piece_partial_slot(k, pos, start);
    if (s0 == 0 && tid == 0) {
      const int kl = cta_of_slot((int64_t)pos + wb - 1, T, grid);
      const int unit = b * per_seq_units + uis;
      *reinterpret_cast<int2*>(a.ws + w.units_off + 8LL * unit) = make_int2(myslot, kl - k + 1);
    }
    __syncthreads();
    for (int idx = tid; idx < nh * D; idx += F::THREADS) {
      const int h = idx / D, c = idx % D;
      const float* f = wts + h * NW;
      const float* mo = merge + h * (D + 2) + c;
      constexpr int WS = kHeadsPerSlice * (D + 2);
      float O = 0.f;
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) O += f[ww] * mo[ww * WS];
      if (whole) {
        reinterpret_cast<__half*>(a.out)[((int64_t)b * g.hq + hbase + h) * D + c] =
            __float2half_rn(O);
      } else {
        float* ps = partials + myslot * w.slot_floats + h * (D + 4);
        ps[c] = O;
        if (c == 0) {
          ps[D] = wts[NW * kHeadsPerSlice + h];
          ps[D + 1] = wts[(NW + 1) * kHeadsPerSlice + h];
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    pos += s1 - s0;
  }
}

template <int D>
size_t f16_smem_bytes(int n_seq) {
  return F16Cfg<D>::SMEM_FIXED + 4 * (size_t)(2 * n_seq + 1);
}

template <int D, bool PK>
cudaError_t f16_launch_t(const Geom& g, const WsLayout& w, const DecodeArgs& a,
                         const __half* kc, const __half* vc, const int32_t* lens,
                         int max_tokens, int grid, cudaStream_t stream) {
  using F = F16Cfg<D>;
  auto kern = f16_decode_kernel<D, PK>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)f16_smem_bytes<D>(kSeqsPerLaunch));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  {
    cudaLaunchConfig_t dc = {};
    dc.gridDim = dim3((unsigned)grid);
    dc.blockDim = dim3(F::THREADS);
    dc.dynamicSmemBytes = f16_smem_bytes<D>(a.n_seq);
    dc.stream = stream;
    cudaLaunchAttribute da[1];
    da[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    da[0].val.programmaticStreamSerializationAllowed = 1;
    dc.attrs = da;
    dc.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&dc, kern, g, w, a, kc, vc, lens, max_tokens);
    if (e != cudaSuccess) return e;
  }
  const int units = a.n_seq * g.hkv * g.slices;
  const int npc_est = grid / units + 1;
  const int wpi = npc_est <= 4 ? 1 : npc_est <= 8 ? 2 : npc_est <= 16 ? 4 : 8;
  const int heads = g.gqa < kHeadsPerSlice ? g.gqa : kHeadsPerSlice;
  const int n_items = units * heads;
  const int ipb = kCombineWarps / wpi;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)((n_items + ipb - 1) / ipb));
  lc.blockDim = dim3(kCombineThreads);
  lc.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, combine_kernel<D>, g, w, a, wpi, heads, n_items);
}

}  // namespace

cudaError_t decode_max_ctas(const Geom& g, bool wide, int* max_ctas) {
#define KVQ_CASE(D_, KB_, VB_, G_)                                  \
  if (g.d == D_ && g.kb == KB_ && g.vb == VB_ && g.G == G_)         \
    return decode_max_ctas_##D_##_##KB_##_##VB_##_##G_(g, wide, max_ctas);
  KVQ_DECODE_FOR_EACH(KVQ_CASE)
#undef KVQ_CASE
  return cudaErrorInvalidValue;
}

// The tcgen05 kernel (kvq_decode_tc.cuh) is opt-in: KVQ_DECODE_TC=1 selects
// it for the shapes it covers.  Measured on B200 it is about 2x slower than
// the mma.sync kernel on these shapes (the contraction per group is too
// small for the tensor core to matter; unpacking and the role hand-offs
// dominate), so the mma.sync kernel is the default.
bool decode_tc_eligible(const Geom& g) {
  if (!(g.d == 128 && g.G == 32 && g.vb == 2 && (g.kb == 2 || g.kb == 4) && g.gqa <= 4 &&
        g.slices == 1 && g.window == 0 && g.sink == 0 && g.rotate == 0 && g.akvq_delta == 0))
    return false;
  const char* env = std::getenv("KVQ_DECODE_TC");
  return env && env[0] == '1';
}

cudaError_t launch_decode(const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid,
                          bool wide, cudaStream_t stream) {
  if (wide && decode_tc_eligible(g))
    return g.kb == 4 ? launch_tc_t<4>(g, w, a, grid, stream) : launch_tc_t<2>(g, w, a, grid, stream);
#define KVQ_CASE(D_, KB_, VB_, G_)                                  \
  if (g.d == D_ && g.kb == KB_ && g.vb == VB_ && g.G == G_)         \
    return launch_decode_##D_##_##KB_##_##VB_##_##G_(g, w, a, grid, wide, stream);
  KVQ_DECODE_FOR_EACH(KVQ_CASE)
#undef KVQ_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_fp16(const Geom& g, const WsLayout& w, const DecodeArgs& a,
                               const void* k, const void* v, const int32_t* lens,
                               int max_tokens, int grid, cudaStream_t stream) {
  const __half* kc = static_cast<const __half*>(k);
  const __half* vc = static_cast<const __half*>(v);
  if (g.d == 128)
    return g.gqa <= 4 ? f16_launch_t<128, true>(g, w, a, kc, vc, lens, max_tokens, grid, stream)
                      : f16_launch_t<128, false>(g, w, a, kc, vc, lens, max_tokens, grid, stream);
  if (g.d == 64)
    return g.gqa <= 4 ? f16_launch_t<64, true>(g, w, a, kc, vc, lens, max_tokens, grid, stream)
                      : f16_launch_t<64, false>(g, w, a, kc, vc, lens, max_tokens, grid, stream);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Decode without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// plugins whose host framework owns every device allocation and offers no
// workspace hook, and deployments that forbid allocation after start-up
// (a fixed memory footprint, no allocator on the serving path).  For them
// the scratch the decode kernel needs (error word, per-unit split records
// and tickets, split partials) lives in this fixed file-scope device array
// instead of a caller buffer.  Every GPU that loads the library holds it
// until the process exits.  All such calls share it: calls that overlap on
// the GPU race on it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
// device address of the array, per device (0 until looked up); written
// once per device with the same value by whichever thread looks first
std::atomic<uintptr_t> g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

// Set-up, once per device, with that device current: the address the
// kernels must be given (in host code the array's name is only a host-side
// stand-in, not a device address).
cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  uintptr_t p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    p = reinterpret_cast<uintptr_t>(addr);
    g_noalloc_ptr[dev].store(p, std::memory_order_release);
  }
  *ptr = reinterpret_cast<void*>(p);
  return cudaSuccess;
}

}  // namespace kvq
