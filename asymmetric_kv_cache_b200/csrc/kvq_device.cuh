// Device helpers for the libkvq kernels (sm_100a): bulk (TMA) copies into
// shared memory with mbarrier completion, bounded waits, the fp16 tensor-core
// tile, and exact unpacking of 2/4-bit codes into fp16 pairs.
#pragma once

#include <cstdint>
#include <type_traits>
#include <utility>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace kvq {

// Iteration cap of every spin on an mbarrier.  A wait that runs out sets the
// workspace error word and the kernel abandons its remaining work instead of
// hanging; no correct launch ever gets near the cap.
constexpr uint32_t kWaitSpinLimit = 1u << 24;

// Debug builds (-DKVQ_DEBUG, libkvq_debug.so) check the index of every
// cache, workspace, query and output access of the decode kernels against
// its buffer before making it; a check that fails records KVQ_ERR_DEVICE
// with the check's number (bits 8 and up) in the workspace error word and
// the access is skipped.  Release builds compile the checks away.
#ifdef KVQ_DEBUG
constexpr bool kDebug = true;
#else
constexpr bool kDebug = false;
#endif

__device__ __forceinline__ bool debug_ok(bool cond, int32_t* err, int code) {
  if (kDebug && !cond) {
    atomicCAS(err, 0, 10 | (code << 8));   // 10 = KVQ_ERR_DEVICE; the first failure wins
    return false;
  }
  return true;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the asynchronous (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier shared-memory accesses before later bulk-copy
// writes into the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One arrival on bar (release: this thread's earlier accesses are visible
// to whoever observes the phase complete).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 1-D bulk copy global -> shared (this CTA), completion counted on bar.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// A bulk copy of `bytes` from src, which must lie in [lo, hi): debug builds
// skip a copy that would leave the range (the barrier phase still completes,
// with no data) and record the failed check.
__device__ __forceinline__ void checked_bulk_copy(void* dst, const unsigned char* src,
                                                  uint32_t bytes, uint64_t* bar,
                                                  const unsigned char* lo, const unsigned char* hi,
                                                  int32_t* err, int code) {
  if (!debug_ok(src >= lo && src + bytes <= hi, err, code)) {
    mbar_arrive(bar);
    return;
  }
  mbar_arrive_expect_tx(bar, bytes);
  bulk_copy_g2s(dst, src, bytes, bar);
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of bar.  Returns false if the cap ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitSpinLimit; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  return false;
}

// D += A * B on one m16n8k16 tile, fp16 inputs, fp32 accumulate.
// A row-major 16x16 (4 regs of half2), B column-major 16x8 (2 regs).
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 matrix of 16-bit elements held one row-pair per lane
// (lane 4r + c holds row r, columns 2c and 2c+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

// Pack two fp32 values into an fp16 pair (round to nearest even); lo -> bits 0..15.
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  return h2_as_u32(__floats2half2_rn(lo, hi));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Ticket increment with acquire-release semantics at GPU scope: the stores
// that precede it (the CTA's, when a CTA barrier comes first) are visible to
// whoever reads the incremented value, and it is ordered before the caller's
// later accesses.
__device__ __forceinline__ int atomic_add_acquire_gpu(int* p, int v) {
  int old;
  asm volatile("atom.add.acquire.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int atomic_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// fp16x2 arithmetic on packed 32-bit registers (round to nearest even).
__device__ __forceinline__ uint32_t hfma2_b(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// a * b - c (the negation folds into the multiply-add)
__device__ __forceinline__ uint32_t hfma2_negc_b(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("{\n.reg .b32 t;\nneg.f16x2 t, %3;\nfma.rn.f16x2 %0, %1, %2, t;\n}"
      : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t hmul2_b(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Code pair of field f of a packed word as the fp16 pair (1024 + m*code_lo,
// 1024 + m*code_hi), m = 2^(BITS * (f mod 8/BITS)) (code_mul<BITS, f>()):
// the field OR-ed into the mantissa of 1024.0.  One LOP3 (plus a shared
// byte shift for the upper fields); the 1024 offset and the factor m are
// removed on the other side of the tensor-core product.
template <int BITS, int F_IDX>
__device__ __forceinline__ uint32_t code_offset(uint32_t w) {
  static_assert(BITS == 2 || BITS == 4, "2- or 4-bit codes");
  constexpr int kPerByte = 8 / BITS;
  constexpr int kShift = (F_IDX >= kPerByte) ? 8 : 0;
  constexpr int kF = F_IDX % kPerByte;
  constexpr uint32_t kLowMask = (BITS == 4) ? 0x000F000Fu : 0x00030003u;
  const uint32_t mask = kLowMask << (BITS * kF);
  const uint32_t one024 = 0x64006400u;
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w >> kShift), "r"(mask), "r"(one024));
  return d;
}
template <int BITS, int F_IDX>
__host__ __device__ constexpr int code_log2_mul() {
  return BITS * (F_IDX % (8 / BITS));
}
// fp16x2 bit pattern of (2^-e, 2^-e).
__host__ __device__ constexpr uint32_t h2_pow2_neg(int e) {
  return ((uint32_t)(15 - e) << 10) | ((uint32_t)(15 - e) << 26);
}
constexpr uint32_t kH2One024 = 0x64006400u;   // (1024, 1024)

// Exact fp16 pair (code_lo, code_hi) of field f of a packed word: the
// offset pair 1024 + m*code (code_offset) times 1/m minus 1024/m in one
// fused fp16x2 multiply-add (small integers times powers of two: exact).
template <int BITS, int F_IDX>
__device__ __forceinline__ uint32_t unpack_pair(uint32_t w) {
  constexpr int e = code_log2_mul<BITS, F_IDX>();
  constexpr uint32_t kOff = 0x8000u | ((uint32_t)(25 - e) << 10);   // -2^(10-e)
  return hfma2_b(code_offset<BITS, F_IDX>(w), h2_pow2_neg(e), kOff | (kOff << 16));
}

// Walsh-Hadamard rotation ("[Framework] The Asymmetric Key-Value Cache
// Compression", §IV stage 1: Y = X H, H an orthogonal +-1 matrix applied by
// the fast Walsh-Hadamard transform).  A row of D values is spread over D / V
// consecutive lanes, V consecutive values per lane (lane index l within the
// row).  Unnormalized transform in IEEE fp32: stages h = 1, 2, ..., D / 2 in
// that order, each pair (j, j + h) of a block of 2h values becoming (a + b,
// a - b); stages h < V inside a lane, the others with lane l ^ (h / V).
// Every lane of the warp must call it together.
template <int D, int V>
__device__ __forceinline__ void fwht_lanes(float (&y)[V], int l) {
#pragma unroll
  for (int h = 1; h < V; h <<= 1) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (j & h) continue;
      const float a = y[j], b = y[j + h];
      y[j] = __fadd_rn(a, b);
      y[j + h] = __fsub_rn(a, b);
    }
  }
#pragma unroll
  for (int hl = 1; hl < D / V; hl <<= 1) {
    const bool upper = (l & hl) != 0;   // this lane holds the b of each pair
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const float p = __shfl_xor_sync(0xffffffffu, y[j], hl);
      y[j] = upper ? __fsub_rn(p, y[j]) : __fadd_rn(y[j], p);
    }
  }
}
// fp32(1 / sqrt(D)), the normalization of the rotation (rounded once).
template <int D>
__host__ __device__ constexpr float rot_scale() {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  return D == 64 ? 0.125f : 0.0883883461356163f;   // 2^-3.5 = 0.08838834764.. -> fp32
}

// Compile-time loop: f(std::integral_constant<int, i>) for i = 0 .. N-1.
template <class F, int... I>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
  static_for_impl(f, std::make_integer_sequence<int, N>{});
}

// N consecutive 32-bit words from shared memory with the widest aligned loads.
template <int N>
__device__ __forceinline__ void lds_words(const uint32_t* p, uint32_t (&w)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(p + i);
      w[i] = v.x; w[i + 1] = v.y; w[i + 2] = v.z; w[i + 3] = v.w;
    }
  } else if constexpr (N % 2 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 2) {
      const uint2 v = *reinterpret_cast<const uint2*>(p + i);
      w[i] = v.x; w[i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) w[i] = p[i];
  }
}

// 16-byte asynchronous global -> shared copy; src_bytes < 16 zero-fills the
// rest (0 reads nothing).  dst, src 16-byte aligned.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ float load_as_float(const void* base, int64_t idx, int dtype) {
  // dtype: 0 fp16, 1 bf16, 2 fp32 (kvq_dtype)
  if (dtype == 0) return __half2float(reinterpret_cast<const __half*>(base)[idx]);
  if (dtype == 1) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  return reinterpret_cast<const float*>(base)[idx];
}

}  // namespace kvq
