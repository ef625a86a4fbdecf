// Host side of the libkvq C ABI: argument validation (before any launch),
// LAYOUT v2 geometry, the host mirror of sequence lengths and launch
// planning.  Every numeric step of the method runs in the CUDA kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "kvq.h"
#include "kvq_internal.h"
#include "kvq_split.h"

struct kvq_cache {
  kvq_config cfg;
  kvq::Geom geom;
  kvq::WsLayout ws;
  unsigned char* buf;
  size_t buf_bytes;
  std::vector<int32_t> lens;   // host mirror of the device lengths
  int max_ctas[2];             // decode CTA caps, narrow / wide (0 until queried)
};

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
kvq_status fail(kvq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

kvq_status ok() {
  g_last_error.clear();
  return KVQ_OK;
}

kvq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KVQ_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

kvq_status validate_config(const kvq_config* c) {
  if (!c) return fail(KVQ_ERR_NULL, "config is NULL");
  if (c->layout_version != 0 && c->layout_version != KVQ_LAYOUT_VERSION)
    return fail(KVQ_ERR_CONFIG, "layout_version %d unsupported (library has %d)",
                c->layout_version, KVQ_LAYOUT_VERSION);
  if (c->k_bits != 2 && c->k_bits != 4)
    return fail(KVQ_ERR_CONFIG, "k_bits must be 2 or 4 (got %d)", c->k_bits);
  if (c->v_bits != 2 && c->v_bits != 4)
    return fail(KVQ_ERR_CONFIG, "v_bits must be 2 or 4 (got %d)", c->v_bits);
  if (c->group != 32 && c->group != 64)
    return fail(KVQ_ERR_CONFIG, "group must be 32 or 64 (got %d)", c->group);
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(KVQ_ERR_CONFIG, "head_dim must be 64 or 128 (got %d)", c->head_dim);
  if (c->head_dim % c->group != 0)
    return fail(KVQ_ERR_CONFIG, "head_dim %d is not a multiple of group %d", c->head_dim, c->group);
  if (c->n_kv_heads < 1 || c->n_q_heads < 1)
    return fail(KVQ_ERR_CONFIG, "head counts must be >= 1 (q %d, kv %d)", c->n_q_heads, c->n_kv_heads);
  if (c->n_q_heads % c->n_kv_heads != 0)
    return fail(KVQ_ERR_CONFIG, "n_q_heads %d is not a multiple of n_kv_heads %d", c->n_q_heads,
                c->n_kv_heads);
  if (c->max_seqs < 1 || c->max_tokens < 1)
    return fail(KVQ_ERR_CONFIG, "max_seqs and max_tokens must be >= 1 (got %d, %d)", c->max_seqs,
                c->max_tokens);
  if (c->window < 0 || c->window > 1024 || c->window % 16 != 0)
    return fail(KVQ_ERR_CONFIG, "window must be a multiple of 16 in [0, 1024] (got %d)", c->window);
  if (c->sink < 0 || c->sink > 1024)
    return fail(KVQ_ERR_CONFIG, "sink must be in [0, 1024] (got %d)", c->sink);
  if (c->rotate != 0 && c->rotate != 1)
    return fail(KVQ_ERR_CONFIG, "rotate must be 0 or 1 (got %d)", c->rotate);
  if (c->akvq_delta != 0) {
    if (c->akvq_delta < 0 || c->akvq_delta > (1 << 20) || c->akvq_delta % c->group != 0)
      return fail(KVQ_ERR_CONFIG, "akvq_delta must be a multiple of group in [0, 2^20] (got %d)",
                  c->akvq_delta);
    if (c->k_bits != 4 || c->window != 0 || c->sink != 0)
      return fail(KVQ_ERR_CONFIG, "akvq_delta needs k_bits = 4 and window = sink = 0");
  }
  // decode addresses slots (groups + tail) of all units with 32-bit prefixes
  const int64_t slices = (c->n_q_heads / c->n_kv_heads + kvq::kHeadsPerSlice - 1) / kvq::kHeadsPerSlice;
  const int64_t slots = (int64_t)c->max_seqs * c->n_kv_heads * slices * (c->max_tokens / c->group + 1);
  if (slots >= (int64_t)1 << 31)
    return fail(KVQ_ERR_CONFIG, "max_seqs * n_kv_heads * groups too large (%lld slots)", (long long)slots);
  return KVQ_OK;
}

kvq_status dtype_ok(int32_t dt) {
  if (dt != KVQ_FP16 && dt != KVQ_BF16 && dt != KVQ_FP32)
    return fail(KVQ_ERR_DTYPE, "unsupported dtype %d", dt);
  return KVQ_OK;
}

void fill_layout(const kvq::Geom& g, kvq_layout* o) {
  o->total_bytes = g.total_bytes;
  o->lens_offset = g.lens_off;
  o->counters_offset = g.counters_off;
  o->blocks_offset = g.blocks_off;
  o->block_bytes = g.block_bytes;
  o->max_groups = g.max_groups;
  o->tails_offset = g.tails_off;
  o->tail_bytes = g.tail_bytes;
  o->tail_slots = (uint64_t)g.tail_slots;
  o->sinks_offset = (uint64_t)g.sinks_off;
  o->sink_bytes = (uint64_t)g.sink_bytes;
  o->sink_slots = (uint64_t)g.sink_slots;
  o->kcodes_offset = g.sec_kcodes;
  o->kscale_offset = g.sec_kscale;
  o->kmin_offset = g.sec_kmin;
  o->vcodes_offset = g.sec_vcodes;
  o->vscale_offset = g.sec_vscale;
  o->vmin_offset = g.sec_vmin;
  o->akvq_block_bytes = g.a2_bytes;
  o->akvq_kscale_offset = g.a2_kscale;
  o->akvq_kmin_offset = g.a2_kmin;
  o->akvq_vcodes_offset = g.a2_vcodes;
  o->akvq_vscale_offset = g.a2_vscale;
  o->akvq_vmin_offset = g.a2_vmin;
}

}  // namespace

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_NULL: return "KVQ_ERR_NULL: a required pointer is NULL";
    case KVQ_ERR_CONFIG: return "KVQ_ERR_CONFIG: unsupported configuration";
    case KVQ_ERR_BUFFER_TOO_SMALL: return "KVQ_ERR_BUFFER_TOO_SMALL: buffer too small";
    case KVQ_ERR_CAPACITY: return "KVQ_ERR_CAPACITY: capacity exceeded";
    case KVQ_ERR_EMPTY: return "KVQ_ERR_EMPTY: decode over an empty sequence";
    case KVQ_ERR_DTYPE: return "KVQ_ERR_DTYPE: unsupported element type";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA: CUDA call failed";
    case KVQ_ERR_ALIGN: return "KVQ_ERR_ALIGN: misaligned pointer";
    case KVQ_ERR_ARG: return "KVQ_ERR_ARG: invalid argument";
    case KVQ_ERR_DEVICE: return "KVQ_ERR_DEVICE: a kernel gave up a bounded wait";
    default: return "KVQ_ERR_?: unknown status";
  }
}

const char* kvq_last_error(void) { return g_last_error.c_str(); }

kvq_status kvq_layout_for(const kvq_config* cfg, kvq_layout* out) {
  if (!out) return fail(KVQ_ERR_NULL, "layout output is NULL");
  kvq_status s = validate_config(cfg);
  if (s != KVQ_OK) return s;
  kvq::Geom g;
  kvq::make_geom(*cfg, &g);
  fill_layout(g, out);
  return ok();
}

kvq_status kvq_cache_required_bytes(const kvq_config* cfg, size_t* cache_bytes,
                                    size_t* workspace_bytes) {
  kvq_status s = validate_config(cfg);
  if (s != KVQ_OK) return s;
  kvq::Geom g;
  kvq::make_geom(*cfg, &g);
  kvq::WsLayout w;
  kvq::make_ws_layout(g, &w);
  if (cache_bytes) *cache_bytes = (size_t)g.total_bytes;
  if (workspace_bytes) *workspace_bytes = (size_t)w.total;
  return ok();
}

kvq_status kvq_cache_create(const kvq_config* cfg, void* dev_buf, size_t bytes, kvq_cache** out) {
  if (!out) return fail(KVQ_ERR_NULL, "output handle pointer is NULL");
  *out = nullptr;
  kvq_status s = validate_config(cfg);
  if (s != KVQ_OK) return s;
  if (!dev_buf) return fail(KVQ_ERR_NULL, "device buffer is NULL");
  if (!aligned(dev_buf, 256)) return fail(KVQ_ERR_ALIGN, "cache buffer must be 256-byte aligned");
  kvq::Geom g;
  kvq::make_geom(*cfg, &g);
  if ((int64_t)bytes < g.total_bytes)
    return fail(KVQ_ERR_BUFFER_TOO_SMALL, "cache buffer has %zu bytes, needs %lld", bytes,
                (long long)g.total_bytes);
  // lengths and append tickets are contiguous: [lens | pad | counters]
  cudaError_t e = cudaMemset(static_cast<unsigned char*>(dev_buf) + g.lens_off, 0,
                             (size_t)(g.counters_off - g.lens_off) + 4 * (size_t)cfg->max_seqs);
  if (e != cudaSuccess) return cuda_fail(e, "zeroing the length and ticket arrays");
  kvq_cache* c = new (std::nothrow) kvq_cache();
  if (!c) return fail(KVQ_ERR_ARG, "out of host memory");
  c->cfg = *cfg;
  c->cfg.layout_version = KVQ_LAYOUT_VERSION;
  c->geom = g;
  kvq::make_ws_layout(g, &c->ws);
  c->buf = static_cast<unsigned char*>(dev_buf);
  c->buf_bytes = bytes;
  c->lens.assign(cfg->max_seqs, 0);
  c->max_ctas[0] = c->max_ctas[1] = 0;
  *out = c;
  return ok();
}

kvq_status kvq_cache_destroy(kvq_cache* cache) {
  delete cache;
  return ok();
}

kvq_status kvq_reset(kvq_cache* cache, void* stream) {
  if (!cache) return fail(KVQ_ERR_NULL, "cache is NULL");
  cudaError_t e = cudaMemsetAsync(cache->buf + cache->geom.lens_off, 0,
                                  (size_t)(cache->geom.counters_off - cache->geom.lens_off) +
                                      4 * (size_t)cache->cfg.max_seqs,
                                  (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_reset");
  std::fill(cache->lens.begin(), cache->lens.end(), 0);
  return ok();
}

kvq_status kvq_append(kvq_cache* cache, const void* k, const void* v, kvq_dtype dtype,
                      const int32_t* n_new, int32_t n_seq, void* stream) {
  if (!cache) return fail(KVQ_ERR_NULL, "cache is NULL");
  if (n_seq < 0) return fail(KVQ_ERR_ARG, "n_seq %d < 0", n_seq);
  if (n_seq > cache->cfg.max_seqs)
    return fail(KVQ_ERR_CAPACITY, "n_seq %d > max_seqs %d", n_seq, cache->cfg.max_seqs);
  if (n_seq > 0 && !n_new) return fail(KVQ_ERR_NULL, "n_new is NULL");
  kvq_status s = dtype_ok(dtype);
  if (s != KVQ_OK) return s;
  int64_t total = 0;
  for (int b = 0; b < n_seq; ++b) {
    if (n_new[b] < 0) return fail(KVQ_ERR_ARG, "n_new[%d] = %d < 0", b, n_new[b]);
    if ((int64_t)cache->lens[b] + n_new[b] > cache->cfg.max_tokens)
      return fail(KVQ_ERR_CAPACITY, "sequence %d would hold %lld tokens > max_tokens %d", b,
                  (long long)cache->lens[b] + n_new[b], cache->cfg.max_tokens);
    total += n_new[b];
  }
  if (total == 0) return ok();
  if (!k || !v) return fail(KVQ_ERR_NULL, "k or v is NULL");
  if (!aligned(k, 16) || !aligned(v, 16)) return fail(KVQ_ERR_ALIGN, "k and v must be 16-byte aligned");

  const kvq::Geom& g = cache->geom;
  // one launch per chunk of sequences (their arguments ride in the kernel
  // parameters); rows of the concatenated input are counted across chunks
  static thread_local kvq::AppendSeqs seqs;
  int64_t row = 0;
  for (int s0 = 0; s0 < n_seq; s0 += kvq::kAppendMaxSeqs) {
    const int n = std::min(kvq::kAppendMaxSeqs, n_seq - s0);
    seqs.n = n;
    seqs.seq0 = s0;
    int tasks = 0;
    for (int i = 0; i < n; ++i) {
      const int b = s0 + i;
      const int len0 = cache->lens[b], nn = n_new[b];
      // groups this append completes (the kernel recomputes them from the
      // device lengths; for nn < G at most one, whatever the length)
      const int F = kvq::quantized_groups_s(len0 + nn, g.G, g.window, g.sink) -
                    kvq::quantized_groups_s(len0, g.G, g.window, g.sink);
      seqs.task_prefix[i] = tasks;
      seqs.row_off[i] = (int32_t)row;
      seqs.n_new[i] = nn;
      tasks += nn > 0 ? std::max(F, 1) : 0;
      if (g.akvq_delta && nn > 0) {
        // requantization tasks of the groups that age into the middle: one
        // reserved below G new tokens (the launch shape then does not depend
        // on the lengths), else the exact count
        int first;
        tasks += nn < g.G ? 1
                          : kvq::akvq_aging(len0, len0 + nn, len0 / g.G, g.G, g.akvq_delta, &first);
      }
      row += nn;
    }
    seqs.task_prefix[n] = tasks;
    if (row > INT32_MAX) return fail(KVQ_ERR_ARG, "more than 2^31 appended rows in one call");
    if (tasks == 0) continue;
    cudaError_t e = kvq::launch_append(g, cache->buf, k, v, dtype, seqs, tasks, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
  }
  for (int b = 0; b < n_seq; ++b) cache->lens[b] += n_new[b];
  return ok();
}

namespace {
// One decode + combine pair per chunk of at most kSeqsPerLaunch sequences
// (stream order keeps the chunks from overlapping on the workspace).
cudaError_t launch_decode_chunks(const kvq::Geom& g, const kvq::WsLayout& w,
                                 const int32_t* lens, const void* q, int q_dtype, void* out,
                                 unsigned char* ws, int n_seq, int* max_ctas, int64_t max_grid,
                                 const unsigned char* cache_buf, cudaStream_t stream) {
  for (int wide = 0; wide < 2; ++wide) {
    if (max_ctas[wide] == 0) {
      cudaError_t e = kvq::decode_max_ctas(g, wide != 0, &max_ctas[wide]);
      if (e != cudaSuccess) return e;
    }
  }
  int env_cap = 0;
  if (const char* env = std::getenv("KVQ_DECODE_MAX_CTAS")) env_cap = std::atoi(env);
  const int64_t qrow = (int64_t)g.hq * g.d * (q_dtype == KVQ_FP32 ? 4 : 2);
  const int64_t orow = (int64_t)g.hq * g.d * 2;
  for (int s0 = 0; s0 < n_seq; s0 += kvq::kSeqsPerLaunch) {
    const int ns = std::min(kvq::kSeqsPerLaunch, n_seq - s0);
    // wide CTAs (one per SM) while there are at most as many units as SMs
    const bool wide = (int64_t)ns * g.hkv * g.slices <= max_ctas[1];
    int cap = max_ctas[wide ? 1 : 0];
    if (env_cap > 0) cap = std::min(cap, env_cap);
    int64_t slots = 0;
    for (int b = s0; b < s0 + ns; ++b)
      slots += (int64_t)g.hkv * g.slices * kvq::unit_slots_s(lens[b], g.G, g.window, g.sink);
    const int64_t grid = std::min(max_grid, kvq::choose_grid(g, lens + s0, ns, slots, cap));
    kvq::DecodeArgs a;
    a.cache = cache_buf;
    a.q = static_cast<const unsigned char*>(q) + s0 * qrow;
    a.q_dtype = q_dtype;
    a.out = static_cast<unsigned char*>(out) + s0 * orow;
    a.ws = ws;
    a.n_seq = ns;
    a.seq0 = s0;
    // wide CTAs (one unit piece each) with up to 32 pieces per split unit:
    // the last CTA of each unit merges them in one round of L2 loads (no
    // combine kernel).  Otherwise the combine kernel: a narrow CTA moves on
    // to its next piece, which an in-kernel merge would delay.
    const int64_t units = (int64_t)ns * g.hkv * g.slices;
    a.inline_merge = kvq::use_inline_merge(wide, grid, units) ? 1 : 0;
    cudaError_t e = kvq::launch_decode(g, w, a, (int)grid, wide, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}
}  // namespace

kvq_status kvq_decode(kvq_cache* cache, const void* q, kvq_dtype q_dtype, void* out,
                      int32_t n_seq, void* workspace, size_t ws_bytes, void* stream) {
  if (!cache) return fail(KVQ_ERR_NULL, "cache is NULL");
  if (!q || !out || !workspace) return fail(KVQ_ERR_NULL, "q, out or workspace is NULL");
  if (n_seq < 1) return fail(KVQ_ERR_ARG, "n_seq %d < 1", n_seq);
  if (n_seq > cache->cfg.max_seqs)
    return fail(KVQ_ERR_CAPACITY, "n_seq %d > max_seqs %d", n_seq, cache->cfg.max_seqs);
  if (n_seq > kvq::kMaxSeqsDecode)
    return fail(KVQ_ERR_CAPACITY, "n_seq %d > %d sequences per decode call", n_seq,
                kvq::kMaxSeqsDecode);
  kvq_status s = dtype_ok(q_dtype);
  if (s != KVQ_OK) return s;
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(KVQ_ERR_ALIGN, "q and out must be 16-byte aligned");
  if (!aligned(workspace, 256)) return fail(KVQ_ERR_ALIGN, "workspace must be 256-byte aligned");
  if ((int64_t)ws_bytes < cache->ws.total)
    return fail(KVQ_ERR_BUFFER_TOO_SMALL, "workspace has %zu bytes, needs %lld", ws_bytes,
                (long long)cache->ws.total);
  const kvq::Geom& g = cache->geom;
  for (int b = 0; b < n_seq; ++b)
    if (cache->lens[b] <= 0) return fail(KVQ_ERR_EMPTY, "sequence %d is empty", b);
  cudaError_t e = launch_decode_chunks(g, cache->ws, cache->lens.data(), q, q_dtype, out,
                                       static_cast<unsigned char*>(workspace), n_seq,
                                       cache->max_ctas, kvq::kMaxDecodeCtas, cache->buf,
                                       (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

kvq_status kvq_decode_noalloc(kvq_cache* cache, const void* q, kvq_dtype q_dtype, void* out,
                              int32_t n_seq, void* stream) {
  if (!cache) return fail(KVQ_ERR_NULL, "cache is NULL");
  if (!q || !out) return fail(KVQ_ERR_NULL, "q or out is NULL");
  if (n_seq < 1) return fail(KVQ_ERR_ARG, "n_seq %d < 1", n_seq);
  if (n_seq > cache->cfg.max_seqs)
    return fail(KVQ_ERR_CAPACITY, "n_seq %d > max_seqs %d", n_seq, cache->cfg.max_seqs);
  if (n_seq > kvq::kMaxSeqsDecode)
    return fail(KVQ_ERR_CAPACITY, "n_seq %d > %d sequences per decode call", n_seq,
                kvq::kMaxSeqsDecode);
  kvq_status s = dtype_ok(q_dtype);
  if (s != KVQ_OK) return s;
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(KVQ_ERR_ALIGN, "q and out must be 16-byte aligned");
  const kvq::Geom& g = cache->geom;
  for (int b = 0; b < n_seq; ++b)
    if (cache->lens[b] <= 0) return fail(KVQ_ERR_EMPTY, "sequence %d is empty", b);
  // The fixed scratch holds [error word | split records and tickets of the
  // units of one launch (at most kSeqsPerLaunch sequences) | two partial
  // slots per CTA]; the CTA count is lowered until the partials fit.
  kvq::WsLayout w = cache->ws;
  const int64_t units = (int64_t)std::min(n_seq, kvq::kSeqsPerLaunch) * g.hkv * g.slices;
  w.units = (int32_t)units;
  w.err_off = 0;
  w.units_off = 256;
  w.tickets_off = kvq::align_up(w.units_off + 8LL * units, 256);
  w.partials_off = kvq::align_up(w.tickets_off + 4LL * units, 256);
  const int64_t slot_bytes = 2LL * w.slot_floats * 4;
  const int64_t room = kvq::kNoAllocScratchBytes - w.partials_off;
  if (room < slot_bytes)
    return fail(KVQ_ERR_CAPACITY,
                "kvq_decode_noalloc: the %lld (sequence, kv head, head slice) units of one launch "
                "need more than the %lld-byte fixed scratch; use kvq_decode with a workspace",
                (long long)units, (long long)kvq::kNoAllocScratchBytes);
  const int64_t max_grid = std::min<int64_t>(kvq::kMaxDecodeCtas, room / slot_bytes);
  void* scratch = nullptr;
  cudaError_t e = kvq::noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "looking up the fixed decode scratch");
  // the error word and the tickets must start at zero; the array keeps
  // whatever the previous call left (split records are rewritten by every
  // launch, and the last CTA of a unit puts its ticket back to zero)
  e = cudaMemsetAsync(scratch, 0, (size_t)w.partials_off, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the fixed decode scratch");
  w.total = w.partials_off + max_grid * slot_bytes;
  e = launch_decode_chunks(g, w, cache->lens.data(), q, q_dtype, out,
                           static_cast<unsigned char*>(scratch), n_seq, cache->max_ctas, max_grid,
                           cache->buf, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

namespace {
// Geometry of an fp16 baseline call (slots of 16 tokens; no block layout).
kvq_status fp16_geom(int32_t n_seq, int32_t hq, int32_t hkv, int32_t d, kvq::Geom* g,
                     kvq::WsLayout* w) {
  if (n_seq < 1) return fail(KVQ_ERR_ARG, "n_seq %d < 1", n_seq);
  if (n_seq > kvq::kMaxSeqsDecode)
    return fail(KVQ_ERR_CAPACITY, "n_seq %d > %d sequences per decode call", n_seq,
                kvq::kMaxSeqsDecode);
  if (d != 64 && d != 128) return fail(KVQ_ERR_CONFIG, "head_dim %d not in {64, 128}", d);
  if (hkv < 1 || hq < hkv || hq % hkv) return fail(KVQ_ERR_CONFIG, "heads %d / %d", hq, hkv);
  *g = kvq::Geom{};
  g->d = d;
  g->hq = hq;
  g->hkv = hkv;
  g->gqa = hq / hkv;
  g->slices = (g->gqa + kvq::kHeadsPerSlice - 1) / kvq::kHeadsPerSlice;
  g->max_seqs = n_seq;
  g->G = 16;
  kvq::make_ws_layout(*g, w);
  return KVQ_OK;
}
}  // namespace

kvq_status kvq_fp16_workspace_bytes(int32_t n_seq, int32_t n_q_heads, int32_t n_kv_heads,
                                    int32_t head_dim, size_t* bytes) {
  if (!bytes) return fail(KVQ_ERR_NULL, "bytes is NULL");
  kvq::Geom g;
  kvq::WsLayout w;
  kvq_status s = fp16_geom(n_seq, n_q_heads, n_kv_heads, head_dim, &g, &w);
  if (s != KVQ_OK) return s;
  *bytes = (size_t)w.total;
  return ok();
}

kvq_status kvq_decode_fp16(const void* k, const void* v, const int32_t* lens, int32_t max_tokens,
                           int32_t n_seq, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                           const void* q, kvq_dtype q_dtype, void* out, void* workspace,
                           size_t ws_bytes, void* stream) {
  if (!k || !v || !lens || !q || !out || !workspace)
    return fail(KVQ_ERR_NULL, "a pointer argument is NULL");
  if (max_tokens < 1) return fail(KVQ_ERR_ARG, "max_tokens %d < 1", max_tokens);
  kvq::Geom g;
  kvq::WsLayout w;
  kvq_status s = fp16_geom(n_seq, n_q_heads, n_kv_heads, head_dim, &g, &w);
  if (s != KVQ_OK) return s;
  s = dtype_ok(q_dtype);
  if (s != KVQ_OK) return s;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(q, 16) || !aligned(out, 16) ||
      !aligned(lens, 4))
    return fail(KVQ_ERR_ALIGN, "k, v, q and out must be 16-byte aligned, lens 4-byte");
  if (!aligned(workspace, 256)) return fail(KVQ_ERR_ALIGN, "workspace must be 256-byte aligned");
  if ((int64_t)ws_bytes < w.total)
    return fail(KVQ_ERR_BUFFER_TOO_SMALL, "workspace has %zu bytes, needs %lld", ws_bytes,
                (long long)w.total);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const int64_t qrow = (int64_t)n_q_heads * head_dim * (q_dtype == KVQ_FP32 ? 4 : 2);
  const int64_t orow = (int64_t)n_q_heads * head_dim * 2;
  for (int s0 = 0; s0 < n_seq; s0 += kvq::kSeqsPerLaunch) {
    kvq::DecodeArgs a;
    a.cache = nullptr;
    a.q = static_cast<const unsigned char*>(q) + s0 * qrow;
    a.q_dtype = q_dtype;
    a.out = static_cast<unsigned char*>(out) + s0 * orow;
    a.ws = static_cast<unsigned char*>(workspace);
    a.n_seq = std::min(kvq::kSeqsPerLaunch, n_seq - s0);
    a.seq0 = s0;
    a.inline_merge = 0;
    e = kvq::launch_decode_fp16(g, w, a, k, v, lens, max_tokens, std::min(sms, kvq::kMaxDecodeCtas),
                                (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "fp16 decode launch");
  }
  return ok();
}

size_t kvq_noalloc_scratch_bytes(void) { return (size_t)kvq::kNoAllocScratchBytes; }

kvq_status kvq_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace) return fail(KVQ_ERR_NULL, "workspace is NULL");
  cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_workspace_init");
  return ok();
}

kvq_status kvq_workspace_status(const void* workspace, void* stream) {
  if (!workspace) return fail(KVQ_ERR_NULL, "workspace is NULL");
  int32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the workspace error word");
  if (word != 0)
    return fail(KVQ_ERR_DEVICE,
                "a decode kernel gave up a bounded wait or failed range check %d (word %#x)",
                word >> 8, (unsigned)word);
  return ok();
}

kvq_status kvq_sync_lengths(kvq_cache* cache, void* stream) {
  if (!cache) return fail(KVQ_ERR_NULL, "cache is NULL");
  cudaError_t e = cudaMemcpyAsync(cache->lens.data(), cache->buf + cache->geom.lens_off,
                                  4 * (size_t)cache->cfg.max_seqs, cudaMemcpyDeviceToHost,
                                  (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kvq_sync_lengths");
  return ok();
}

kvq_status kvq_cache_config(const kvq_cache* cache, kvq_config* out) {
  if (!cache || !out) return fail(KVQ_ERR_NULL, "cache or output is NULL");
  *out = cache->cfg;
  return ok();
}

kvq_status kvq_cache_layout(const kvq_cache* cache, kvq_layout* out) {
  if (!cache || !out) return fail(KVQ_ERR_NULL, "cache or output is NULL");
  fill_layout(cache->geom, out);
  return ok();
}

kvq_status kvq_get_lengths(const kvq_cache* cache, int32_t* host_lens, int32_t n) {
  if (!cache || !host_lens) return fail(KVQ_ERR_NULL, "cache or output is NULL");
  if (n < 0 || n > cache->cfg.max_seqs)
    return fail(KVQ_ERR_ARG, "n = %d outside [0, max_seqs = %d]", n, cache->cfg.max_seqs);
  std::memcpy(host_lens, cache->lens.data(), 4 * (size_t)n);
  return ok();
}

}  // extern "C"
