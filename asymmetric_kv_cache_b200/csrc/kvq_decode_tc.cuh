// Decode on the 5th-generation tensor cores (tcgen05) for d = 128, 32-token
// groups, 2-bit values and GQA groups of at most 4 heads (the Llama-3-8B
// shaped layer and the 128k-token long context).  Included by
// kvq_decode.cu after kvq_decode_kernels.cuh (it uses that header's Geom,
// DecCfg, Piece, query conversion, fp16-tail code, merge helpers and split
// records).  Same attention as decode_kernel (per-channel key and per-token
// value dequantization, "[Framework] The Asymmetric Key-Value Cache
// Compression", §III; online softmax and the split merge of that page's
// flash-decoding baseline, §IV), same
// stream-K split and partial format, so combine_kernel and
// finish_split_unit serve both.
//
// A tile is 4 groups = 128 tokens, the M of one tcgen05.mma.  Per tile:
//   S[t, (g, h, part)] = sum_c A_K[t, c] B_q[c, (g, h, part)]
//     A_K (tensor memory, 128 lanes = tokens): key codes as 1024 + m*code,
//       m = 2^(field offset), written by the key warps (one LOP3 per pair);
//     B_q (shared memory, K-major): q * s_k / m as fp16 high part and
//       residual for each of the tile's 4 groups (N = 4 x 8 columns, a
//       group's tokens read only their own 8), built by the builder warps;
//     a second K-block set against a constant -1024 A block cancels the
//       offset inside the same accumulation (the tensor core sums exactly
//       the fp16 B values the code block saw);
//   the key warps add the key-min bias sum_c q_c z_c (mma.sync by the
//   builders, per group and head), run the online softmax across the tile
//   (one running max per head), and write B_P[t, (j, h)] = fp16(p s_v)
//   (shared memory, MN-major: a token's 16 values are one 32-byte row);
//   O_tile[c, (j, h)] = sum_t A_V[c, t] B_P[t, (j, h)]
//     A_V (tensor memory, 128 lanes = channels): value codes unpacked
//       exactly, written by the value warps; channel c reads its own group
//       j = c / 32;
//   the value warps fold O_tile into per-channel registers with the tile's
//   rescale factors, and the value-min terms sum_t p z_v are per-token
//   partial sums of the key warps, reduced once per piece.
// Warps: 0-3 keys + softmax (tensor-memory lanes 32w..), 4-7 values + O,
// 8 bulk-copy producer, 9 MMA issue (one elected lane), 10-11 B_q builders,
// 12 the unit's fp16 tail (the mma.sync tail code) when the piece has it.
// Every wait on an mbarrier is bounded (kWaitSpinLimit polls); one that runs
// out sets the workspace error word.

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// arrive on `bar` once every tcgen05 operation this thread issued so far is complete
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D (tensor memory) (+)= A (tensor memory) * B (shared-memory descriptor)
__device__ __forceinline__ void tc_mma(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile(
      "{\n.reg .pred e;\n.reg .b32 r;\nelect.sync r|e, 0xffffffff;\nselp.u32 %0, 1, 0, e;\n}\n"
      : "=r"(p));
  return p != 0;
}
__device__ __forceinline__ void tc_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
#define KVQ_R4(b) "r"(r[b]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3])
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      KVQ_R4(0), KVQ_R4(4), KVQ_R4(8), KVQ_R4(12)
      : "memory");
}
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      KVQ_R4(0), KVQ_R4(4), KVQ_R4(8), KVQ_R4(12), KVQ_R4(16), KVQ_R4(20), KVQ_R4(24),
      KVQ_R4(28)
      : "memory");
}
#undef KVQ_R4
__device__ __forceinline__ void tc_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tc_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}
// Shared-memory matrix descriptor, no swizzle: core matrices of 8 rows x 16
// bytes stored contiguously; lbo = byte distance between core matrices along
// K (K-major) or along K-groups of 8 (MN-major), sbo = the other direction.
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor: fp16 A and B, fp32 accumulator, A K-major, B
// K-major (b_mn = 0) or MN-major (b_mn = 1), M x N.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, int b_mn) {
  return (1u << 4) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// Max over the warp of a float (no NaN): an order-preserving map to int.
__device__ __forceinline__ float warp_max_f(float x) {
  const int i = __float_as_int(x);
  int k = i >= 0 ? i : (i ^ 0x7FFFFFFF);
  k = __reduce_max_sync(0xffffffffu, k);
  return __int_as_float(k >= 0 ? k : (k ^ 0x7FFFFFFF));
}

template <int KB>
struct TcCfg {
  static constexpr int D = 128, G = 32, VB = 2;
  using C = DecCfg<D, KB, VB, G, true>;
  static constexpr int BLK = C::BLK;
  static constexpr int TILE = 4;            // groups per tile: 128 tokens
  static constexpr int NS = 16;             // ring stages (group blocks), four tiles
  static constexpr int WV = 4, WP = 8, WM = 9, WB = 10, WT = 12, NWARP = 13;
  static constexpr int THREADS = NWARP * 32;
  // tensor-memory columns: A_K[2] (64 each: 128 fp16 channels), the -1024
  // block, A_V[2] (64 each: 128 fp16 tokens), S[2] (32), O[PD] (16)
  static constexpr uint32_t T_AK = 0, T_CONST = 128, T_AV = 192, T_S = 320, T_O = 384;
  // depth of the P -> O hand-off (B_P, O, the rescale factors): the key
  // warps may run PD tiles ahead of the value warps' folding
  static constexpr int PD = 4;
  static constexpr uint32_t T_COLS = 512;
  // B_q: per group 16 K-chunks (8 channels each) of 8 rows x 16 B, chunks
  // 144 B apart (a 16-byte pad keeps the builders' row stores conflict-free)
  static constexpr int BQ_LBO = 144, BQ_SBO = 16 * BQ_LBO, BQ_BUF = TILE * BQ_SBO;
  // B_P (MN-major): 8-token groups 256 B apart, 8-column halves 128 B apart
  static constexpr int BP_LBO = 256, BP_SBO = 128, BP_BUF = 16 * BP_LBO;
  static constexpr int RING_OFF = 0;
  static constexpr int BQ_OFF = NS * BLK;
  static constexpr int BP_OFF = BQ_OFF + 2 * BQ_BUF;
  static constexpr int QS_OFF = BP_OFF + PD * BP_BUF;
  static constexpr int QS_BYTES = C::QA_BYTES;
  static constexpr int TAIL_OFF = QS_OFF + QS_BYTES;
  static constexpr int TAIL_BYTES = 2 * TailStage<D>::BYTES;
  static constexpr int MERGE_OFF = TAIL_OFF + TAIL_BYTES;
  static constexpr int MERGE_FLOATS = 2 * kHeadsPerSlice * (D + 2);   // two areas
  static constexpr int WTS_OFF = MERGE_FLOATS;                        // within merge
  static constexpr int MISC_OFF = MERGE_OFF + (MERGE_FLOATS + 4 * kHeadsPerSlice) * 4;
  // misc floats: bias[2][4][4], tile max[2][4][4], alpha[4][4], l[4][4],
  // value-min sums[4][16], running max[4]
  static constexpr int F_BIAS = 0, F_RED = 32, F_ALPHA = 64, F_L = 80, F_Z = 96, F_M = 160;
  static constexpr int MISC_FLOATS = 164;
  static constexpr int BAR_OFF = MISC_OFF + ((MISC_FLOATS * 4 + 15) / 16) * 16;
  static constexpr int B_FULL = 0, B_EMPTY = NS, B_AKF = 2 * NS, B_BQF = B_AKF + 2,
                       B_SF = B_BQF + 2, B_SE = B_SF + 2, B_PF = B_SE + 2, B_AVF = B_PF + PD,
                       B_OF = B_AVF + 2, B_OE = B_OF + PD, B_Q = B_OE + PD, NBAR = B_Q + 1;
  static constexpr int SMEM_FIXED = BAR_OFF + NBAR * 8;
  // arrivals that free a ring stage: its key warp, the 4 value warps, its builder
  static constexpr int EMPTY_COUNT = 1 + 4 + 1;
  static_assert(C::LWK * C::FK == 16, "16 code pairs per lane and 8-token tile");
  static_assert(C::LWV == 4 && C::FV == 8, "2-bit values: 4 words per lane and k-tile");
  static_assert(BQ_OFF % 16 == 0 && BP_OFF % 16 == 0 && QS_OFF % 16 == 0 && TAIL_OFF % 16 == 0,
                "16-byte aligned areas");
};

// Wait for phase `parity` of bar with the warp suspended in hardware
// between checks (a suspend-time hint of 20 us per try, woken early when the
// phase completes) instead of spinning: the specialized warps of this kernel
// wait often, and spinning ones take issue slots from the working warps of
// their sub-partition.  At most 2^14 tries (a few tenths of a second).
__device__ __forceinline__ bool mbar_wait_suspend(uint64_t* bar, uint32_t parity) {
  for (int it = 0; it < (1 << 14); ++it) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\n"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
        "selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Bounded wait that folds a timeout into the warp-uniform `ok` and the
// workspace error word.
__device__ __forceinline__ void tc_wait(uint64_t* bar, uint32_t parity, bool& ok,
                                        int32_t* err, int lane) {
  if (!ok) return;
  bool got = mbar_wait_suspend(bar, parity);
  got = __all_sync(0xffffffffu, got);
  if (!got) {
    ok = false;
    if (lane == 0) atomicExch(err, KVQ_ERR_DEVICE);
  }
}

template <int KB>
__global__ void __launch_bounds__(TcCfg<KB>::THREADS, 1)
    decode_tc_kernel(const Geom g, const WsLayout w, const DecodeArgs a) {
  using T = TcCfg<KB>;
  using C = typename T::C;
  constexpr int D = 128, G = 32, VB = 2;
  extern __shared__ __align__(1024) unsigned char tc_smem[];
  unsigned char* const smem = tc_smem;
  __shared__ int32_t wsum[T::NWARP];
  __shared__ int32_t ticket_flag[3];
  __shared__ uint32_t tmem_base_s;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BAR_OFF);
  uint4* qsm = reinterpret_cast<uint4*>(smem + T::QS_OFF);
  float* misc = reinterpret_cast<float*>(smem + T::MISC_OFF);
  float* merge = reinterpret_cast<float*>(smem + T::MERGE_OFF);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + T::SMEM_FIXED);
  int32_t* slen = prefix + (a.n_seq + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, i4 = lane & 3;
  const int n_seq = a.n_seq;
  const int per_seq_units = g.hkv * g.slices;
  const int32_t* lens = reinterpret_cast<const int32_t*>(a.cache + g.lens_off) + a.seq0;
  int32_t* err = reinterpret_cast<int32_t*>(a.ws + w.err_off);
  float* partials = reinterpret_cast<float*>(a.ws + w.partials_off);
  const unsigned char* blocks = a.cache + g.blocks_off;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(&bars[T::B_FULL + s], 1);
      mbar_init(&bars[T::B_EMPTY + s], T::EMPTY_COUNT);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[T::B_AKF + b], 4);
      mbar_init(&bars[T::B_BQF + b], 2);
      mbar_init(&bars[T::B_SF + b], 1);
      mbar_init(&bars[T::B_SE + b], 4);
      mbar_init(&bars[T::B_AVF + b], 4);
    }
    for (int x = 0; x < T::PD; ++x) {
      mbar_init(&bars[T::B_PF + x], 4);
      mbar_init(&bars[T::B_OF + x], 1);
      mbar_init(&bars[T::B_OE + x], 4);
    }
    mbar_init(&bars[T::B_Q], 1);
    fence_mbar_init();
  }
  if (warp == T::WM) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base_s)),
                 "r"(T::T_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // ---- slot prefix over sequences (as decode_kernel)
  if (tid == 0) prefix[0] = 0;
  {
    const int chunk = (n_seq + T::THREADS - 1) / T::THREADS;
    const int b0 = tid * chunk, b1 = min(n_seq, b0 + chunk);
    int32_t run = 0;
    for (int bb = b0; bb < b1; ++bb) {
      const int L = lens[bb];
      run += per_seq_units * (L / G + (L % G ? 1 : 0));
    }
    int32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    int32_t base = 0;
    for (int ww = 0; ww < warp; ++ww) base += wsum[ww];
    int32_t acc = base + incl - run;
    for (int bb = b0; bb < b1; ++bb) {
      const int L = lens[bb];
      acc += per_seq_units * (L / G + (L % G ? 1 : 0));
      prefix[bb + 1] = acc;
      slen[bb] = L;
    }
  }
  const uint32_t tm = tmem_base_s;
  // the constant -1024 block (key warps: their 32 lanes each)
  if (warp < 4) {
    uint32_t r[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] = 0xE400E400u;
    const uint32_t la = (uint32_t)(32 * warp) << 16;
    tc_st32(tm + la + T::T_CONST, r);
    tc_st32(tm + la + T::T_CONST + 32, r);
    tc_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int Tsl = prefix[n_seq];
  const int grid = gridDim.x;
  const int k = blockIdx.x;
  int start, end;
  cta_range(k, Tsl, grid, &start, &end);
  if (start == end) {   // as in decode_kernel: an empty piece, counted on its unit's ticket
    if (tid < kHeadsPerSlice) {
      float* ps = partials + (int64_t)(2 * k) * w.slot_floats + tid * (D + 4);
      ps[D] = -INFINITY;
      ps[D + 1] = 0.f;
    }
    if (a.inline_merge && start < Tsl) {
      const Piece p = make_piece(g, prefix, slen, n_seq, start, start + 1);
      if (p.slot0 > 0)
        finish_split_unit<D, T::THREADS>(g, w, a, p.unit, (int64_t)start - p.slot0, p.wb, Tsl,
                                         grid, p.b, p.hbase, p.nh, reinterpret_cast<float*>(smem),
                                         T::NS * T::BLK / (4 * 3 * kHeadsPerSlice), ticket_flag,
                                         tid, false, nullptr);
    }
  }

  bool ok = true;
  int tile_base = 0, grp_base = 0;
  uint32_t qphase = 0;
  for (int pos = start; pos < end;) {
    int ngr, nh, Tb;
    int64_t gb;
    bool has_tail;
    {
      const Piece p = make_piece(g, prefix, slen, n_seq, pos, end);
      gb = ((int64_t)(a.seq0 + p.b) * g.hkv + p.kvh) * g.max_groups + p.slot0;
      ngr = max(0, min(p.slot1, p.ng) - p.slot0);
      nh = p.nh;
      Tb = p.Tb;
      has_tail = p.Tb > 0 && p.slot1 == p.wb && p.slot0 <= p.ng;
      if (tid == 0) {
        const int esz = a.q_dtype == KVQ_FP32 ? 4 : 2;
        const uint32_t qbytes = (uint32_t)(p.nh * D * esz);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[T::B_Q], qbytes);
        bulk_copy_g2s(qsm,
                      static_cast<const unsigned char*>(a.q) +
                          ((int64_t)p.b * g.hq + p.hbase) * D * esz,
                      qbytes, &bars[T::B_Q]);
      }
      if (warp == T::WT && has_tail) {
        const __half* tk = reinterpret_cast<const __half*>(
            a.cache + g.tails_off + ((int64_t)(a.seq0 + p.b) * g.hkv + p.kvh) * g.tail_bytes);
        for (int kv = 0; kv * 16 < p.Tb; ++kv)
          stage_tail_chunk<D>(smem + T::TAIL_OFF + kv * TailStage<D>::BYTES, tk, tk + G * D,
                              p.Tb, kv, lane);
      }
    }
    const int ntiles = (ngr + T::TILE - 1) / T::TILE;
    // the producer starts the piece's copies at once; the key warps turn
    // the query rows into fragments meanwhile
    // (the first NS of them: their stages' previous uses belong to pieces
    // that are complete; the rest wait for the consumers below)
    auto produce = [&](int gq0, int gq1) {
      if (lane == 0) {
        for (int gq = gq0; gq < gq1 && ok; ++gq) {
          const int gg = grp_base + gq, s = gg % T::NS;
          if (gg >= T::NS) {
            if (!mbar_wait_suspend(&bars[T::B_EMPTY + s], ((gg / T::NS) + 1) & 1)) {
              ok = false;
              atomicExch(err, KVQ_ERR_DEVICE);
              break;
            }
          }
          mbar_arrive_expect_tx(&bars[T::B_FULL + s], T::BLK);
          bulk_copy_g2s(smem + s * T::BLK, blocks + (gb + gq) * T::BLK, T::BLK,
                        &bars[T::B_FULL + s]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    };
    if (warp == T::WP) produce(0, min(ngr, T::NS));
    if (warp < 4) {
      bool got = mbar_wait_bounded(&bars[T::B_Q], qphase & 1);
      got = __all_sync(0xffffffffu, got);
      if (!got && lane == 0) atomicExch(err, KVQ_ERR_DEVICE);
      convert_query<D, true, 4>(a.q_dtype, nh, got, warp, lane, qsm,
                                reinterpret_cast<const unsigned char*>(qsm));
    }
    ++qphase;
    __syncthreads();

    if (warp < 4) {
      // ================= key warps: dequant keys, softmax =================
      const int q = warp;
      const uint32_t la = (uint32_t)(32 * q) << 16;
      float mrun[4], lsum[4], zs[4][4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        mrun[h] = -INFINITY;
        lsum[h] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) zs[h][j] = 0.f;
      }
      for (int i = 0; i <= ntiles; ++i) {
        if (i < ntiles) {
          // key codes of token `lane` of group 4i + q into A_K[b]
          const int tg = tile_base + i, b = tg & 1, gq = T::TILE * i + q;
          if (gq < ngr) {
            const int gg = grp_base + gq, s = gg % T::NS;
            tc_wait(&bars[T::B_FULL + s], (gg / T::NS) & 1, ok, err, lane);
            const uint4* kr = reinterpret_cast<const uint4*>(smem + s * T::BLK + C::SEC_KCODES) +
                              lane * C::LWK;
            uint32_t wd[4 * C::LWK];
#pragma unroll
            for (int x = 0; x < C::LWK; ++x) {
              const uint4 v = kr[x];
              wd[4 * x] = v.x; wd[4 * x + 1] = v.y; wd[4 * x + 2] = v.z; wd[4 * x + 3] = v.w;
            }
            // TMEM pair column col: i4 = col / 16, code pair p = col % 16 of
            // that lane's words (word p / FK, field p % FK)
            static_for<2>([&](auto hf_) {
              constexpr int hf = decltype(hf_)::value;
              uint32_t r[32];
              static_for<32>([&](auto c_) {
                constexpr int col = 32 * hf + decltype(c_)::value;
                constexpr int ii = col / 16, pp = col % 16;
                r[decltype(c_)::value] =
                    code_offset<KB, pp % C::FK>(wd[ii * C::LWK + pp / C::FK]);
              });
              if (ok) tc_st32(tm + la + T::T_AK + 64 * b + 32 * hf, r);
            });
            tc_wait_st();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[T::B_AKF + b]);
        }
        if (i >= 1) {
          // ---- softmax of tile i - 1
          const int ti = i - 1, tg = tile_base + ti, b = tg & 1;
          const uint32_t ph = (tg >> 1) & 1;
          const int gq = T::TILE * ti + q;
          const bool valid = gq < ngr;
          const int gg = grp_base + gq, s = gg % T::NS;
          tc_wait(&bars[T::B_BQF + b], ph, ok, err, lane);
          tc_wait(&bars[T::B_SF + b], ph, ok, err, lane);
          tc_fence_after();
          uint32_t v[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          if (ok) {
            tc_ld8(tm + la + T::T_S + 32 * b + 8 * q, v);
            tc_wait_ld();
          }
          // the builders overwrite the tile's bias after this arrive
          const float4 bias = *reinterpret_cast<const float4*>(misc + T::F_BIAS + b * 16 + q * 4);
          const float bh[4] = {bias.x, bias.y, bias.z, bias.w};
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[T::B_SE + b]);
          float sv[4], wm[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            sv[h] = (valid && h < nh && ok)
                        ? (__uint_as_float(v[h]) + __uint_as_float(v[4 + h])) + bh[h]
                        : -INFINITY;
            wm[h] = warp_max_f(sv[h]);
          }
          if (lane == 0)
            *reinterpret_cast<float4*>(misc + T::F_RED + b * 16 + q * 4) =
                make_float4(wm[0], wm[1], wm[2], wm[3]);
          asm volatile("bar.sync 2, 128;" ::: "memory");
          float al[4], pv[4];
          bool resc = false;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            float tmx = misc[T::F_RED + b * 16 + h];
#pragma unroll
            for (int qq = 1; qq < 4; ++qq) tmx = fmaxf(tmx, misc[T::F_RED + b * 16 + qq * 4 + h]);
            const float mn = fmaxf(mrun[h], tmx);
            al[h] = (mn == -INFINITY || mn == mrun[h]) ? 1.f : fast_exp2(mrun[h] - mn);
            resc |= al[h] != 1.f;
            mrun[h] = mn;
            pv[h] = (sv[h] == -INFINITY) ? 0.f : fast_exp2(sv[h] - mn);
          }
          if (resc) {   // the same on every key thread
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              lsum[h] *= al[h];
#pragma unroll
              for (int j = 0; j < 4; ++j) zs[h][j] *= al[h];
            }
          }
          uint4 row0 = make_uint4(0u, 0u, 0u, 0u), row1 = row0;
          if (valid) {
            // token `lane`'s value scale and min of group j: slot
            // ((4 kv + i) J + j) 4 + 2 kh + e (the value-side fragment order)
            const int kv = lane >> 4, kh = (lane >> 3) & 1, ii = (lane >> 1) & 3, e = lane & 1;
            const unsigned short* vsh = reinterpret_cast<const unsigned short*>(
                                            smem + s * T::BLK + C::SEC_VSCALE) +
                                        (4 * kv + ii) * C::J * 4 + 2 * kh + e;
            const unsigned short* vzh = reinterpret_cast<const unsigned short*>(
                                            smem + s * T::BLK + C::SEC_VMIN) +
                                        (4 * kv + ii) * C::J * 4 + 2 * kh + e;
            float zv[4];
            uint32_t sj[4];   // (s_j, s_j)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              zv[j] = __half2float(__ushort_as_half(vzh[4 * j]));
              const uint32_t x = vsh[4 * j];
              sj[j] = x | (x << 16);
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              lsum[h] += pv[h];
#pragma unroll
              for (int j = 0; j < 4; ++j) zs[h][j] = fmaf(pv[h], zv[j], zs[h][j]);
            }
            const uint32_t p01 = pack_h2(pv[0], pv[1]), p23 = pack_h2(pv[2], pv[3]);
            row0 = make_uint4(hmul2_b(p01, sj[0]), hmul2_b(p23, sj[0]), hmul2_b(p01, sj[1]),
                              hmul2_b(p23, sj[1]));
            row1 = make_uint4(hmul2_b(p01, sj[2]), hmul2_b(p23, sj[2]), hmul2_b(p01, sj[3]),
                              hmul2_b(p23, sj[3]));
          }
          // B_P, O and the rescale slot of tile tg are free once the value
          // warps have folded tile tg - PD (after its PV completed).  Waiting
          // for that rather than the PV's commit also keeps this P-full
          // phase from running two phases ahead of the value warps' wait.
          const int px = tg % T::PD;
          if (tg >= T::PD) tc_wait(&bars[T::B_OE + px], ((tg - T::PD) / T::PD) & 1, ok, err, lane);
          if (q == 0 && lane == 0)
            *reinterpret_cast<float4*>(misc + T::F_ALPHA + px * 4) =
                make_float4(al[0], al[1], al[2], al[3]);
          const int kk = 32 * q + lane;   // the token's K index within the tile
          unsigned char* bp = smem + T::BP_OFF + px * T::BP_BUF + (kk >> 3) * T::BP_LBO + (kk & 7) * 16;
          *reinterpret_cast<uint4*>(bp) = row0;
          *reinterpret_cast<uint4*>(bp + T::BP_SBO) = row1;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bars[T::B_PF + px]);
            if (valid) mbar_arrive(&bars[T::B_EMPTY + s]);
          }
        }
      }
      // per-piece sums over the key threads
#pragma unroll
      for (int h = 0; h < 4; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) zs[h][j] += __shfl_xor_sync(0xffffffffu, zs[h][j], o);
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          misc[T::F_L + q * 4 + h] = lsum[h];
#pragma unroll
          for (int j = 0; j < 4; ++j) misc[T::F_Z + q * 16 + h * 4 + j] = zs[h][j];
          if (q == 0) misc[T::F_M + h] = mrun[h];
        }
      }
    } else if (warp < 8) {
      // ================= value warps: dequant values, fold O =================
      const int qv = warp - 4, c = 32 * qv + lane;
      const uint32_t la = (uint32_t)(32 * qv) << 16;
      // channel c = 16 mt + g + 8 hr: word wd = mt / 2 of lane (g, i4), field
      // 2 (mt % 2) + hr in the low byte of each half (tokens 2i4, 2i4 + 1 of
      // the k-tile) and the same field in the high byte (tokens + 8)
      const int mt = c >> 4, rr = c & 15, gw = rr & 7, hr = rr >> 3;
      const int wdi = mt >> 1, f0 = 2 * (mt & 1) + hr;
      const uint32_t mask = 0x00030003u << (2 * f0);
      const uint32_t scl = h2_pow2_neg(2 * f0);
      const uint32_t off = (0x8000u | ((uint32_t)(25 - 2 * f0) << 10)) * 0x00010001u;   // -2^(10-e)
      float oacc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i <= ntiles + 1; ++i) {
        if (i >= 2) {
          // fold O of tile i - 2
          // (its PV is also what frees A_V for tile i)
          const int tg = tile_base + i - 2, px = tg % T::PD;
          const uint32_t ph = (tg / T::PD) & 1;
          tc_wait(&bars[T::B_PF + px], ph, ok, err, lane);
          tc_wait(&bars[T::B_OF + px], ph, ok, err, lane);
          tc_fence_after();
          uint32_t v[4] = {0u, 0u, 0u, 0u};
          if (ok) {
            tc_ld4(tm + la + T::T_O + 16 * px + 4 * qv, v);
            tc_wait_ld();
          }
          const float4 al = *reinterpret_cast<const float4*>(misc + T::F_ALPHA + px * 4);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[T::B_OE + px]);
          oacc[0] = fmaf(oacc[0], al.x, __uint_as_float(v[0]));
          oacc[1] = fmaf(oacc[1], al.y, __uint_as_float(v[1]));
          oacc[2] = fmaf(oacc[2], al.z, __uint_as_float(v[2]));
          oacc[3] = fmaf(oacc[3], al.w, __uint_as_float(v[3]));
        }
        if (i < ntiles) {
          const int tg = tile_base + i, b = tg & 1;
          for (int q = 0; q < T::TILE; ++q) {
            const int gq = T::TILE * i + q;
            uint32_t r[16];
            if (gq < ngr) {
              const int gg = grp_base + gq, s = gg % T::NS;
              tc_wait(&bars[T::B_FULL + s], (gg / T::NS) & 1, ok, err, lane);
              const uint32_t* vw = reinterpret_cast<const uint32_t*>(smem + s * T::BLK + C::SEC_VCODES);
#pragma unroll
              for (int kv = 0; kv < 2; ++kv) {
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                  const uint32_t wv = vw[(kv * 32 + 4 * gw + ii) * C::LWV + wdi];
                  uint32_t x0, x1;
                  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(x0) : "r"(wv), "r"(mask), "r"(kH2One024));
                  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(x1) : "r"(wv >> 8), "r"(mask), "r"(kH2One024));
                  r[8 * kv + ii] = hfma2_b(x0, scl, off);
                  r[8 * kv + ii + 4] = hfma2_b(x1, scl, off);
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) r[j] = 0u;
            }
            if (ok) tc_st16(tm + la + T::T_AV + 64 * b + 16 * q, r);
          }
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bars[T::B_AVF + b]);
            for (int q = 0; q < T::TILE; ++q) {
              const int gq = T::TILE * i + q;
              if (gq < ngr) mbar_arrive(&bars[T::B_EMPTY + (grp_base + gq) % T::NS]);
            }
          }
        }
      }
      // value-min terms and the head's max and sum join the O of channel c
      asm volatile("bar.sync 3, %0;" ::"n"(T::THREADS) : "memory");   // (A): key sums in misc
      {
        float* mo = merge;   // area 0
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float z = 0.f;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) z += misc[T::F_Z + qq * 16 + h * 4 + qv];
          mo[h * (D + 2) + c] = oacc[h] + z;
        }
        if (qv == 0 && lane < kHeadsPerSlice) {
          const int h = lane;
          float l = 0.f;
          if (h < 4)
            for (int qq = 0; qq < 4; ++qq) l += misc[T::F_L + qq * 4 + h];
          mo[h * (D + 2) + D] = h < 4 ? misc[T::F_M + h] : -INFINITY;
          mo[h * (D + 2) + D + 1] = l;
        }
      }
    } else if (warp == T::WP) {
      // ================= bulk-copy producer: the rest of the piece =================
      produce(T::NS, ngr);
    } else if (warp == T::WM) {
      // ================= MMA issue =================
      // Operands are computed by the whole warp (warp-uniform values) and one
      // elected lane issues: an issue from divergent code, with operands
      // outside the uniform datapath, costs ~10x per instruction.
      constexpr uint32_t ID_QK = umma_idesc(128, 32, 0), ID_PV = umma_idesc(128, 16, 1);
      const uint32_t sb = smem_u32(smem);
      const uint64_t dq0 = umma_sdesc(sb + T::BQ_OFF, T::BQ_LBO, T::BQ_SBO);
      const uint64_t dp0 = umma_sdesc(sb + T::BP_OFF, T::BP_LBO, T::BP_SBO);
      for (int i = 0; i <= ntiles; ++i) {
        if (i < ntiles) {
          const int tg = tile_base + i, b = tg & 1;
          const uint32_t ph = (tg >> 1) & 1;
          tc_wait(&bars[T::B_AKF + b], ph, ok, err, lane);
          tc_wait(&bars[T::B_BQF + b], ph, ok, err, lane);
          if (tg >= 2) tc_wait(&bars[T::B_SE + b], ((tg - 2) >> 1) & 1, ok, err, lane);
          tc_fence_after();
          const uint64_t dq = dq0 + (uint64_t)((b * T::BQ_BUF) >> 4);
          const uint32_t dS = tm + T::T_S + 32 * b, aK = tm + T::T_AK + 64 * b;
          const uint32_t aC = tm + T::T_CONST;
          if (ok) {
            if (elect_one()) {
#pragma unroll
              for (int kb = 0; kb < 8; ++kb)
                tc_mma(dS, aK + 8 * kb, dq + (uint64_t)((kb * 2 * T::BQ_LBO) >> 4), ID_QK,
                       kb > 0 ? 1u : 0u);
#pragma unroll
              for (int kb = 0; kb < 8; ++kb)
                tc_mma(dS, aC + 8 * kb, dq + (uint64_t)((kb * 2 * T::BQ_LBO) >> 4), ID_QK, 1u);
              tc_commit(&bars[T::B_SF + b]);
            }
          }
          __syncwarp();
        }
        if (i >= 1) {
          const int tg = tile_base + i - 1, b = tg & 1, px = tg % T::PD;
          tc_wait(&bars[T::B_PF + px], (tg / T::PD) & 1, ok, err, lane);
          tc_wait(&bars[T::B_AVF + b], (tg >> 1) & 1, ok, err, lane);
          if (tg >= T::PD) tc_wait(&bars[T::B_OE + px], ((tg - T::PD) / T::PD) & 1, ok, err, lane);
          tc_fence_after();
          const uint64_t dp = dp0 + (uint64_t)((px * T::BP_BUF) >> 4);
          const uint32_t dO = tm + T::T_O + 16 * px, aV = tm + T::T_AV + 64 * b;
          if (ok) {
            if (elect_one()) {
#pragma unroll
              for (int kb = 0; kb < 8; ++kb)
                tc_mma(dO, aV + 8 * kb, dp + (uint64_t)((kb * 2 * T::BP_LBO) >> 4), ID_PV,
                       kb > 0 ? 1u : 0u);
              tc_commit(&bars[T::B_OF + px]);
            }
          }
          __syncwarp();
        }
      }
    } else if (warp == T::WB || warp == T::WB + 1) {
      // ================= B_q builders (groups 2x, 2x + 1 of each tile) =================
      const int x = warp - T::WB;
      const int k8 = lane >> 1, hp = lane & 1;
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(qsm);
      uint32_t qh[2][4], ql[2][4], mul[4];
      int kwi[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int col = 4 * k8 + u, ii = col >> 4, pp = col & 15;
        const int kt = pp >> 1, half = pp & 1, f = pp % C::FK;
        // the pair's word in the (channel-permuted) key scale array:
        // slots 32 ii + 4 kt + 2 half + {0, 1}
        kwi[u] = 16 * ii + 2 * kt + half;
        mul[u] = h2_pow2_neg(KB * (f % (8 / KB)));
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int h = 2 * hp + hh;
          qh[hh][u] = qw[(kt * 32 + 4 * (h + 4) + ii) * 4 + 2 * half];
          ql[hh][u] = qw[(kt * 32 + 4 * (h + 4) + ii) * 4 + 2 * half + 1];
        }
      }
      // bias fragments: columns 0-3 the heads' high parts, 4-7 their low parts
      uint32_t qb[C::KT][2];
      {
#pragma unroll
        for (int kt = 0; kt < C::KT; ++kt) {   // the lanes' x words
          const uint4 q4 = qsm[kt * 32 + lane];
          qb[kt][0] = q4.y;
          qb[kt][1] = q4.w;
        }
      }
      for (int i = 0; i < ntiles; ++i) {
        const int tg = tile_base + i, b = tg & 1;
        // B_q[b] and the bias slots are free once the key warps are done
        // with tile tg - 2 (they read S after its MMAs completed)
        if (tg >= 2) tc_wait(&bars[T::B_SE + b], ((tg - 2) >> 1) & 1, ok, err, lane);
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const int q = 2 * x + qq, gq = T::TILE * i + q;
          if (gq < ngr) {
            const int gg = grp_base + gq, s = gg % T::NS;
            tc_wait(&bars[T::B_FULL + s], (gg / T::NS) & 1, ok, err, lane);
            const uint32_t* ksw = reinterpret_cast<const uint32_t*>(smem + s * T::BLK + C::SEC_KSCALE);
            uint32_t sp[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) sp[u] = hmul2_b(ksw[kwi[u]], mul[u]);
            unsigned char* dst = smem + T::BQ_OFF + b * T::BQ_BUF + q * T::BQ_SBO + k8 * T::BQ_LBO;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t hi[4], lo[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                hi[u] = hmul2_b(qh[hh][u], sp[u]);
                lo[u] = hfma2_b(ql[hh][u], sp[u], hfma2_negc_b(qh[hh][u], sp[u], hi[u]));
              }
              const int h = 2 * hp + hh;
              *reinterpret_cast<uint4*>(dst + h * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
              *reinterpret_cast<uint4*>(dst + (h + 4) * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
          }
        }
        // key-min bias of the two groups: rows g8 < 2 of the A operand
        {
          const int q = 2 * x + (g8 & 1), gq = T::TILE * i + q;
          const bool row = g8 < 2 && gq < ngr;
          const uint32_t* kzw = reinterpret_cast<const uint32_t*>(
              smem + ((grp_base + (row ? gq : 0)) % T::NS) * T::BLK + C::SEC_KMIN);
          float bacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kt = 0; kt < C::KT; ++kt) {
            const uint32_t a0 = row ? kzw[16 * i4 + 2 * kt] : 0u;       // channels 16kt + 2i4 + {0,1}
            const uint32_t a2 = row ? kzw[16 * i4 + 2 * kt + 1] : 0u;   // and + 8
            mma16816(bacc, a0, 0u, a2, 0u, qb[kt][0], qb[kt][1]);
          }
          // head columns 2i4, 2i4 + 1 (i4 < 2) plus their low parts (i4 + 2)
          const float x0 = bacc[0] + __shfl_xor_sync(0xffffffffu, bacc[0], 2);
          const float x1 = bacc[1] + __shfl_xor_sync(0xffffffffu, bacc[1], 2);
          if (row && i4 < 2) {
            misc[T::F_BIAS + b * 16 + q * 4 + 2 * i4] = x0;
            misc[T::F_BIAS + b * 16 + q * 4 + 2 * i4 + 1] = x1;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars[T::B_BQF + b]);
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            const int gq = T::TILE * i + 2 * x + qq;
            if (gq < ngr) mbar_arrive(&bars[T::B_EMPTY + (grp_base + gq) % T::NS]);
          }
        }
      }
    } else if (warp == T::WT) {
      // ================= the unit's fp16 tail (mma.sync) =================
      WarpState<D, KB, VB, G, true> st;
#pragma unroll
      for (int m2 = 0; m2 < C::MT; ++m2) st.o[m2][0] = st.o[m2][1] = st.o[m2][2] = st.o[m2][3] = 0.f;
      st.z[0] = st.z[1] = st.z[2] = st.z[3] = 0.f;
      st.m[0] = st.m[1] = -INFINITY;
      if (has_tail) {
        cp_async_wait_all();
        __syncwarp();
        for (int kv = 0; kv * 16 < Tb; ++kv)
          tail_chunk_pk<D, KB, VB, G>(st, smem + T::TAIL_OFF + kv * TailStage<D>::BYTES, Tb, kv,
                                      qsm, lane);
      }
      // area 1 of the merge: (o, m, l) of heads 0-3 as in decode_kernel
      float* mo = merge + kHeadsPerSlice * (D + 2);
      float zl0[C::J], zl1[C::J];
#pragma unroll
      for (int j = 0; j < C::J; ++j) {
        zl0[j] = __shfl_sync(0xffffffffu, st.z[0], 4 * j + i4);
        zl1[j] = __shfl_sync(0xffffffffu, st.z[1], 4 * j + i4);
      }
      const float l0 = __shfl_sync(0xffffffffu, st.z[0], 4 * C::J + i4);
      const float l1 = __shfl_sync(0xffffffffu, st.z[1], 4 * C::J + i4);
      if (i4 < 2) {
#pragma unroll
        for (int m2 = 0; m2 < C::MT; ++m2) {
          const int c0 = 16 * m2 + g8, c1 = c0 + 8;
          const int j = (16 * m2) / G;
          mo[(2 * i4) * (D + 2) + c0] = st.o[m2][0] + zl0[j];
          mo[(2 * i4 + 1) * (D + 2) + c0] = st.o[m2][1] + zl1[j];
          mo[(2 * i4) * (D + 2) + c1] = st.o[m2][2] + zl0[j];
          mo[(2 * i4 + 1) * (D + 2) + c1] = st.o[m2][3] + zl1[j];
        }
      }
      if (g8 == 0 && i4 < 2) {
        mo[(2 * i4) * (D + 2) + D] = st.m[0];
        mo[(2 * i4 + 1) * (D + 2) + D] = st.m[1];
        mo[(2 * i4) * (D + 2) + D + 1] = l0;
        mo[(2 * i4 + 1) * (D + 2) + D + 1] = l1;
      }
      if (g8 == 0 && i4 >= 2) {   // heads 4-7 carry no weight
        mo[(2 * i4) * (D + 2) + D] = -INFINITY;
        mo[(2 * i4 + 1) * (D + 2) + D] = -INFINITY;
        mo[(2 * i4) * (D + 2) + D + 1] = 0.f;
        mo[(2 * i4 + 1) * (D + 2) + D + 1] = 0.f;
      }
    }
    // producer, MMA, builder and tail warps meet the value warps' barrier (A)
    if (warp < 4 || warp >= 8) asm volatile("bar.sync 3, %0;" ::"n"(T::THREADS) : "memory");   // (A)
    __syncthreads();   // merge areas complete

    const Piece p = make_piece(g, prefix, slen, n_seq, pos, end);
    const int b = p.b, slot0 = p.slot0, slot1 = p.slot1, wb = p.wb, unit = p.unit;
    const int hbase = p.hbase;
    const bool whole = (slot0 == 0 && slot1 == wb);
    float* wts = merge + T::WTS_OFF;
    merge_weights<D, 2>(merge, wts, whole, tid);
    const int myslot = piece_partial_slot(k, pos, start);
    if (slot0 == 0 && tid == 0) {
      const int kl = cta_of_slot((int64_t)pos + wb - 1, Tsl, grid);
      *reinterpret_cast<int2*>(a.ws + w.units_off + 8LL * unit) = make_int2(myslot, kl - k + 1);
    }
    __syncthreads();
    for (int idx = tid; idx < nh * D; idx += T::THREADS) {
      const int h = idx / D, c = idx % D;
      const float* f = wts + h * 2;
      const float* mo = merge + h * (D + 2) + c;
      constexpr int WS = kHeadsPerSlice * (D + 2);
      const float O = f[0] * mo[0] + f[1] * mo[WS];
      if (whole) {
        reinterpret_cast<__half*>(a.out)[((int64_t)b * g.hq + hbase + h) * D + c] =
            __float2half_rn(O);
      } else {
        float* ps = partials + myslot * w.slot_floats + h * (D + 4);
        ps[c] = O;
        if (c == 0) {
          ps[D] = wts[2 * kHeadsPerSlice + h];
          ps[D + 1] = wts[3 * kHeadsPerSlice + h];
        }
      }
    }
    if (!whole && a.inline_merge)
      finish_split_unit<D, T::THREADS>(g, w, a, unit, (int64_t)pos - slot0, wb, Tsl, grid, b,
                                       hbase, nh, reinterpret_cast<float*>(smem),
                                       T::NS * T::BLK / (4 * 3 * kHeadsPerSlice), ticket_flag,
                                       tid, false, nullptr);
    fence_proxy_async_smem();
    __syncthreads();
    tile_base += ntiles;
    grp_base += ngr;
    pos += slot1 - slot0;
  }
  // every MMA was waited on (the last S and O of each piece); free the columns
  tc_fence_before();
  __syncthreads();
  if (warp == T::WM) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm),
                 "r"(T::T_COLS)
                 : "memory");
  }
}

template <int KB>
size_t tc_smem_bytes(int n_seq) {
  return TcCfg<KB>::SMEM_FIXED + 4 * (size_t)(2 * n_seq + 1);
}

template <int KB>
cudaError_t launch_tc_t(const Geom& g, const WsLayout& w, const DecodeArgs& a, int grid,
                        cudaStream_t stream) {
  using T = TcCfg<KB>;
  if (g.block_bytes != T::BLK || g.sec_vmin != T::C::SEC_VMIN ||
      g.sec_kscale != T::C::SEC_KSCALE)
    return cudaErrorInvalidValue;
  auto kern = decode_tc_kernel<KB>;
  static bool configured = false;   // attribute set once, before any capture
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc_smem_bytes<KB>(kSeqsPerLaunch));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  {
    cudaLaunchConfig_t dc = {};
    dc.gridDim = dim3((unsigned)grid);
    dc.blockDim = dim3(T::THREADS);
    dc.dynamicSmemBytes = tc_smem_bytes<KB>(a.n_seq);
    dc.stream = stream;
    cudaLaunchAttribute da[1];
    da[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    da[0].val.programmaticStreamSerializationAllowed = 1;
    dc.attrs = da;
    dc.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&dc, kern, g, w, a);
    if (e != cudaSuccess) return e;
  }
  if (a.inline_merge) return cudaSuccess;
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
  return cudaLaunchKernelEx(&lc, combine_kernel<128>, g, w, a, wpi, heads, n_items);
}
