/*
 * kvq.h — C ABI of libkvq: decode-step attention over an asymmetrically
 * quantized KV cache, for NVIDIA B200 (sm_100a).
 *
 * What the library computes
 * -------------------------
 * Keys are quantized per channel and values per token, with uniform
 * asymmetric (min + scale) codes, and the newest tokens stay in fp16:
 *   "[Framework] The Asymmetric Key-Value Cache Compression", §III (Pillar I,
 *   KIVI partitioning): K per channel, V per token, an FP16 window of recent
 *   tokens; "Asymmetric Key-Value Quantization: 2-Bit Values and 4-Bit Keys
 *   under Long-Context Drift", §3.1: keys at 4 bits, values at 2 bits.
 * Decode attention is out_h = sum_t alpha_t v_t,
 * alpha = softmax(q_h . k_t / sqrt(d))  (same report, §1 and §2.1), evaluated
 * over the dequantized groups and the fp16 tail.
 *
 * Quantizer (bit-exact contract).  Every K/V element entering the cache is
 * first rounded to IEEE binary16 (round to nearest even).  For each group,
 * in IEEE fp32 with round-to-nearest-even and no fused multiply-add:
 *     mn, mx = min / max over the group
 *     s      = fp16( (mx - mn) / Q )            Q = 2^bits - 1
 *     z      = fp16( mn )
 *     code   = clamp( rne( (x - z) / s ), 0, Q )   with fp32(s), fp32(z);
 *              code = 0 when s == 0.
 * Key group: G consecutive tokens x one channel (G tokens from position 0 of
 * each sequence).  Value group: G consecutive channels of one token.
 * The newest tokens of each sequence (keys and values) sit in an fp16 tail.
 * With the recent window R = kvq_config.window (same page, §III and §V: the
 * most recent 32 to 128 tokens stay in FP16), a group is quantized once R
 * newer tokens follow it: N = G * floor(max(0, n - R) / G) tokens are
 * quantized and the tail holds the other n - N, between R and R + G - 1 once
 * n >= R; a tail that reaches R + G tokens has its oldest G quantized as the
 * next group ("flush").  R = 0 gives the n mod G tail.  With the sink window
 * S = kvq_config.sink (InnerQ abstract, page "WUSH-KV: KV Cache Quantization
 * with Data-Adaptive Transforms": high-precision windows for recent and for
 * attention-sink tokens) the first S tokens of a sequence stay in fp16 as
 * well; groups are cut from position S on and the rule above applies to the
 * tokens after the sink.  Query head h reads kv head h / (n_q_heads /
 * n_kv_heads).  With kvq_config.rotate ("[Framework] The Asymmetric Key-Value
 * Cache Compression", §IV stage 1: Y = X H with an orthogonal +-1 matrix,
 * fast Walsh-Hadamard transform; "Asymmetric Key-Value Quantization: 2-Bit
 * Values and 4-Bit Keys under Long-Context Drift", §3.1: keys and values
 * rotated before quantization) every K/V token is rotated before all of the
 * above, so the whole cache (groups, tail, sink) holds rotated tokens; q .
 * k is unchanged when q is rotated the same way, and the output is rotated
 * back (H / sqrt(d) is symmetric and its own inverse).
 *
 * Conventions
 * -----------
 *  - Every function returns kvq_status (0 = KVQ_OK); nothing throws.
 *  - All device memory is owned by the caller.  The handle owns host state
 *    only (configuration and a host mirror of the sequence lengths).
 *  - Calls taking a stream (cudaStream_t passed as void*; NULL = legacy
 *    default stream) are asynchronous on that stream; pointers must stay
 *    valid until the stream has passed the call.  Argument errors are
 *    detected on the host, before anything is launched, and leave the
 *    cache unchanged.
 *  - A handle is not thread-safe; distinct handles are independent.
 *
 * LAYOUT v2 of the cache buffer (all region offsets 256-byte aligned; see
 * kvq_layout for the numbers).  Version 1 was a plain layout: separate
 * regions for key codes, key (scale, min) pairs, value codes and value
 * pairs, codes packed little-endian in element order.  Version 2 (the only
 * one this library reads or writes; a configuration asking for 1 is refused
 * with KVQ_ERR_CONFIG) keeps the same bytes per token but interleaves each
 * group's sections into one contiguous block, so that a single bulk copy
 * brings a whole group on chip, and stores the codes in tensor-core fragment
 * order, so that one 128-bit shared-memory load gives a lane its operand.
 *   lens   : int32 [max_seqs]                 device copy of the lengths
 *   tickets: int32 [max_seqs]                 append completion counters (0 at rest)
 *   blocks : [max_seqs][n_kv_heads][max_groups] group blocks of block_bytes
 *   tails  : [max_seqs][n_kv_heads] { K tail fp16 [W][d] token-major,
 *                                     V tail fp16 [W/2][d][2] token pairs }
 *            a ring of W = R + G token slots: the token at sequence
 *            position p sits in slot t = (p - S) mod W while it is in the
 *            tail (t = p - N when R = S = 0).  K tail slot (t, c) is element
 *            t*d + c; V tail slot (t, c) is element ((t/2)*d + c)*2 + t%2.
 *   sinks  : [max_seqs][n_kv_heads] { K fp16 [SW][d], V fp16 [SW/2][d][2] }
 *            SW = S rounded up to a multiple of 16; token p < S in slot p,
 *            same element order as the tail (absent when S = 0).
 * A group block holds, in this order (byte offsets in kvq_layout):
 *   key codes   G*d*kbits/8 bytes
 *   key scales  d fp16, key mins d fp16
 *   value codes G*d*vbits/8 bytes
 *   value scales G*(d/G) fp16, value mins G*(d/G) fp16
 * Code packing (little-endian 32-bit words, F = 16/bits code pairs per
 * word, field f occupies bits [f*bits, (f+1)*bits)):
 *   key (token t, channel c): nt = t/8, r = t%8, kt = c/16, v = (c%16)/8,
 *     i = (c%8)/2, e = c%2; lane = 4r+i; p = 2kt+v;
 *     byte offset = nt*32*LB + lane*LB + 4*(p/F) with LB = d*kbits/32,
 *     field = p%F + F*e.
 *   value (token t, channel c): kv = t/16, kh = (t%16)/8, i = (t%8)/2,
 *     e = t%2, mt = c/16, hr = (c%16)/8, g = c%8; lane = 4g+i;
 *     word = mt/(F/4), u = mt%(F/4); byte offset = kv*32*LB + lane*LB +
 *     4*word with LB = d*vbits/16; field = 2u + hr + (F/2)*kh + F*e.
 *   key scale/min of channel c sit at slot i*(d/4) + 4kt + 2v + e;
 *   value scale/min of (token t, channel group j), J = d/G groups, sit at
 *   slot ((4kv + i)*J + j)*4 + 2kh + e.
 * (These are the tensor-core fragment orders the decode kernel reads with
 * 128-bit loads; the packing is a fixed permutation, so every token still
 * costs a fixed number of bits.)
 * Position-adaptive key bits (kvq_config.akvq_delta > 0, k_bits = 4): slots
 * stay block_bytes apart (the 4-bit block); a group whose keys are at 2 bits
 * holds, from the start of its slot, the block of a 2-bit-key cache (the
 * same sections and packing with kbits = 2: offsets akvq_* in kvq_layout,
 * akvq_block_bytes long); the rest of that slot is unspecified.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_LAYOUT_VERSION 2

/* Exported entry points (the library is built with hidden visibility). */
#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

typedef int32_t kvq_status;
enum {
  KVQ_OK = 0,
  KVQ_ERR_NULL = 1,              /* a required pointer is NULL */
  KVQ_ERR_CONFIG = 2,            /* unsupported bits / group / head_dim / heads */
  KVQ_ERR_BUFFER_TOO_SMALL = 3,  /* cache or workspace buffer too small */
  KVQ_ERR_CAPACITY = 4,          /* append past max_tokens or n_seq > max_seqs */
  KVQ_ERR_EMPTY = 5,             /* decode over a sequence of length 0 */
  KVQ_ERR_DTYPE = 6,             /* unsupported element type */
  KVQ_ERR_CUDA = 7,              /* a CUDA call failed (see kvq_last_error) */
  KVQ_ERR_ALIGN = 8,             /* a pointer is not suitably aligned */
  KVQ_ERR_ARG = 9,               /* other invalid argument (negative count ...) */
  KVQ_ERR_DEVICE = 10            /* a kernel reported a failed internal wait */
};

typedef enum { KVQ_FP16 = 0, KVQ_BF16 = 1, KVQ_FP32 = 2 } kvq_dtype;

typedef struct {
  int32_t k_bits;          /* 2 or 4 */
  int32_t v_bits;          /* 2 or 4 */
  int32_t group;           /* G: 32 or 64 */
  int32_t head_dim;        /* d: 64 or 128 (d % G == 0) */
  int32_t n_q_heads;       /* Hq, a multiple of n_kv_heads */
  int32_t n_kv_heads;      /* Hkv >= 1 */
  int32_t max_seqs;        /* sequences the buffer holds, >= 1 */
  int32_t max_tokens;      /* capacity per sequence, >= 1 */
  int32_t layout_version;  /* must be KVQ_LAYOUT_VERSION (or 0 = current) */
  int32_t window;          /* R: recent tokens kept in fp16 beyond the partial
                              group; a multiple of 16 in [0, 1024]; 0 = the
                              n mod G tail */
  int32_t sink;            /* S: first tokens of each sequence kept in fp16,
                              in [0, 1024]; 0 = none */
  int32_t rotate;          /* 1: every K/V token is rotated by the normalized
                              Walsh-Hadamard matrix H / sqrt(d) before it
                              enters the cache (fp32 butterfly, stages h = 1,
                              2, .., d/2 with (a, b) -> (a + b, a - b), times
                              fp32(1 / sqrt(d)), then fp16); the decode
                              rotates q the same way and rotates its output
                              back.  0: no rotation */
  int32_t akvq_delta;      /* Delta > 0: position-adaptive key bits ("Asymmetric
                              Key-Value Quantization: 2-Bit Values and 4-Bit
                              Keys under Long-Context Drift", §3.2): 4-bit keys
                              (k_bits must be 4) for the early key groups (all
                              positions < Delta) and the recent ones (last
                              position >= n - Delta), 2-bit keys in between; a
                              4-bit group that ages into the middle is
                              requantized to 2 bits from its dequantized keys,
                              fp16(fp32(s) * code + fp32(z)), by the append
                              that moves it there.  A multiple of group, at
                              most 2^20; needs window = sink = 0.  Every group
                              keeps a slot of block_bytes (the 4-bit block);
                              a 2-bit group's block (akvq_block_bytes, the
                              sections at the akvq_* offsets) starts at its
                              slot.  0: off */
} kvq_config;

typedef struct {
  uint64_t total_bytes;    /* cache buffer size */
  uint64_t lens_offset;    /* int32[max_seqs] */
  uint64_t counters_offset;/* int32[max_seqs], zero between calls */
  uint64_t blocks_offset;  /* first group block */
  uint64_t block_bytes;    /* one group block */
  uint64_t max_groups;     /* floor(max_tokens / G) blocks per (seq, kv head) */
  uint64_t tails_offset;   /* first tail */
  uint64_t tail_bytes;     /* K tail + V tail of one (seq, kv head) = 4*W*d */
  uint64_t kcodes_offset, kscale_offset, kmin_offset; /* within a block */
  uint64_t vcodes_offset, vscale_offset, vmin_offset; /* within a block */
  uint64_t tail_slots;     /* W = window + G token slots per tail ring */
  uint64_t sinks_offset;   /* first sink area (0 bytes each when sink = 0) */
  uint64_t sink_bytes;     /* K + V sink of one (seq, kv head) = 4*SW*d */
  uint64_t sink_slots;     /* SW: sink rounded up to a multiple of 16 */
  uint64_t akvq_block_bytes;                          /* a 2-bit key group's block */
  uint64_t akvq_kscale_offset, akvq_kmin_offset;      /* within that block (codes at 0) */
  uint64_t akvq_vcodes_offset, akvq_vscale_offset, akvq_vmin_offset;
} kvq_layout;

typedef struct kvq_cache kvq_cache;

/* Human-readable name of a status code (static string). */
KVQ_API const char* kvq_status_string(kvq_status s);

/* Detail of the last failure on the calling thread ("" if none).  The
 * string stays valid until the next call on that thread. */
KVQ_API const char* kvq_last_error(void);

/* LAYOUT v2 offsets for a configuration (host only, no device work).
 * Errors: KVQ_ERR_NULL, KVQ_ERR_CONFIG. */
KVQ_API kvq_status kvq_layout_for(const kvq_config* cfg, kvq_layout* out);

/* Bytes the caller must provide: the cache buffer and the decode workspace
 * (split partials, per-unit split records and an error word).  Either output
 * pointer may be NULL.  Host only.  Errors: KVQ_ERR_NULL, KVQ_ERR_CONFIG. */
KVQ_API kvq_status kvq_cache_required_bytes(const kvq_config* cfg, size_t* cache_bytes,
                                    size_t* workspace_bytes);

/* Bind a handle to a caller-owned device buffer of at least cache_bytes
 * (256-byte aligned).  Validates the configuration on the host first
 * (KVQ_ERR_NULL, KVQ_ERR_CONFIG, KVQ_ERR_BUFFER_TOO_SMALL, KVQ_ERR_ALIGN),
 * then zeroes the device length and counter arrays synchronously on the
 * current device (KVQ_ERR_CUDA if that fails).  The buffer is not otherwise
 * touched. */
KVQ_API kvq_status kvq_cache_create(const kvq_config* cfg, void* dev_buf, size_t bytes,
                            kvq_cache** out);

/* Free the host handle (never the device buffer).  NULL is accepted. */
KVQ_API kvq_status kvq_cache_destroy(kvq_cache* cache);

/* Set every sequence length to 0 (host mirror and device copy, on stream). */
KVQ_API kvq_status kvq_reset(kvq_cache* cache, void* stream);

/* Append n_new[b] tokens to sequence b, for b in [0, n_seq).
 * Defining passages: "[Framework] The Asymmetric Key-Value Cache
 * Compression", §III (Pillar I: keys grouped per channel along the token
 * axis, values per token, the most recent tokens in FP16), and the InnerQ
 * abstract on the "WUSH-KV: KV Cache Quantization with Data-Adaptive
 * Transforms" page (group-wise quantization of the cache); the quantizer is
 * the bit-exact contract in the header comment above.
 * k, v: device arrays [sum_b n_new[b], n_kv_heads, head_dim] of dtype
 * (fp16, bf16 or fp32), token-major, sequences concatenated in order b;
 * 16-byte aligned; read only.  n_new: host array of n_seq non-negative
 * counts, read before the call returns.
 * Performs prefill quantization (whole groups straight from the input),
 * per-step appends into the fp16 tail and the flush of a tail that reaches
 * R + G tokens (its oldest G become a group), all in one launch.  The launch
 * is a programmatic dependent of the previous kernel on the stream: its
 * CTAs may become resident while that kernel runs, and they wait for it to
 * complete before they read or write any memory (inputs included), so
 * stream order holds as for a plain launch.  The kernel
 * takes the current lengths from the device copy and advances it, so an
 * append captured in a CUDA graph may be replayed provided every n_new[b] <
 * G (the launch shape then does not depend on the lengths); after replays,
 * kvq_sync_lengths refreshes the host mirror.  Values outside the fp16 range
 * are not representable by the cache (their codes are unspecified).
 * Errors (host side, cache unchanged): KVQ_ERR_NULL, KVQ_ERR_ARG,
 * KVQ_ERR_CAPACITY (n_seq > max_seqs or a length would pass max_tokens),
 * KVQ_ERR_DTYPE, KVQ_ERR_ALIGN; KVQ_ERR_CUDA if the launch fails. */
KVQ_API kvq_status kvq_append(kvq_cache* cache, const void* k, const void* v, kvq_dtype dtype,
                      const int32_t* n_new, int32_t n_seq, void* stream);

/* Decode attention for sequences [0, n_seq): for every query head h,
 * out_h = sum_t alpha_t v_t with alpha = softmax(q_h . k_t / sqrt(d)) over
 * all tokens of the sequence ("Asymmetric Key-Value Quantization: 2-Bit
 * Values and 4-Bit Keys under Long-Context Drift", §1 and §2.1), the keys
 * and values dequantized from their groups (s * code + z) or read from the
 * fp16 tail and sink.
 * q: device [n_seq, n_q_heads, d] (fp16, bf16 or fp32, 16-byte aligned),
 * read only; out: device [n_seq, n_q_heads, d] fp16, written.  n_seq: the
 * first n_seq sequences of the cache are decoded (any count up to
 * max_seqs; the survey's interface left it implicit, this library takes it
 * as an argument so that a batch may use fewer slots than the cache holds).
 * workspace: device buffer of at least the workspace_bytes reported by
 * kvq_cache_required_bytes, 256-byte aligned, zero-filled before its first
 * use (kvq_workspace_init).  Calls that share a workspace must not overlap
 * on the GPU.  For each chunk of up to 2048 sequences the call launches the
 * split-K decode kernel (one CTA per SM) and, when units are split across
 * many CTAs, a small combine kernel that merges them (launched as a
 * programmatic dependent of the first).  Inside a CTA the warps claim key
 * groups dynamically, so repeated calls are not bit-identical: the fp16
 * attention weights are rounded relative to a running max that depends on
 * the order a warp meets its groups (outputs move by ~1e-5..1e-4).
 * Errors (host side): KVQ_ERR_NULL, KVQ_ERR_ARG, KVQ_ERR_CAPACITY,
 * KVQ_ERR_EMPTY (some sequence has length 0), KVQ_ERR_DTYPE,
 * KVQ_ERR_ALIGN, KVQ_ERR_BUFFER_TOO_SMALL; KVQ_ERR_CUDA on launch failure.
 * The kernel reads the lengths from the device copy, so a captured decode
 * may be replayed while appends advance them (the launch shape, fixed at
 * capture, stays valid as lengths grow).  A failed internal wait inside the
 * kernel (never expected) is recorded in the workspace and reported by
 * kvq_workspace_status.  The environment variable KVQ_DECODE_MAX_CTAS, if
 * set to a positive integer, caps the number of CTAs (split granularity;
 * results stay within rounding of each other). */
KVQ_API kvq_status kvq_decode(kvq_cache* cache, const void* q, kvq_dtype q_dtype, void* out,
                      int32_t n_seq, void* workspace, size_t ws_bytes, void* stream);

/* kvq_decode for callers that cannot allocate device memory when they
 * decode: plugins whose host framework owns every device allocation and
 * offers no workspace hook, and deployments that forbid allocation after
 * start-up (a fixed memory footprint, no allocator on the serving path).
 * The pages have no counterpart of this call: it only changes where the
 * decode scratch lives.
 * Instead of a caller workspace, the scratch (error word, per-unit split
 * records and tickets, split partials) is a fixed 8 MiB device array inside
 * the library (kvq_noalloc_scratch_bytes()); every GPU that loads the
 * library holds it until exit.  The call allocates nothing: it clears the
 * error word, split records and tickets with cudaMemsetAsync, lowers the
 * number of CTAs until the partials fit, and launches the same decode
 * kernel.  All calls share the array, which keeps the last call's contents,
 * so calls that overlap on the GPU (other streams, other threads) race:
 * serialize them.  The first call on each device also looks up the array's
 * device address (cudaGetSymbolAddress).  Arguments and errors as
 * kvq_decode; KVQ_ERR_CAPACITY
 * (nothing launched) when the units of one launch - min(n_seq, 2048)
 * sequences x n_kv_heads x head slices of 8 query heads - need more split
 * records than the array holds (about 690,000 units).  A failed internal
 * wait (never expected) is recorded only in the array's error word, which
 * the next call clears; use kvq_decode with a workspace where that report
 * matters.  Bit-for-bit results may differ from kvq_decode's when the CTA
 * count differs (split order); both are within the same tolerance of exact
 * attention. */
KVQ_API kvq_status kvq_decode_noalloc(kvq_cache* cache, const void* q, kvq_dtype q_dtype,
                                      void* out, int32_t n_seq, void* stream);

/* fp16 decode baseline (comparison kernel; not part of the quantized path).
 * The same decode attention over an unquantized fp16 cache: k and v device
 * [n_seq][n_kv_heads][max_tokens][head_dim] fp16, 16-byte aligned; lens a
 * DEVICE int32 array [n_seq] of lengths in [1, max_tokens] (the kernel
 * clamps lengths to [0, max_tokens], so no access leaves the arrays; a
 * sequence of length 0 gets an undefined output); q, out as for kvq_decode.  The
 * pages compare the quantized cache against this unquantized baseline
 * ("WUSH-KV" page, InnerQ abstract; FlashDecoding in the first page, §IV):
 * 2 * head_dim * 2 bytes per token-head instead of the packed codes.  Same
 * split-K design (stream-K over one CTA per SM, dynamic 16-token slots,
 * fp16 high/low query on the tensor core, combine kernel).  head_dim 64 or
 * 128, n_q_heads a multiple of n_kv_heads.  workspace: at least
 * kvq_fp16_workspace_bytes(n_seq, ...) bytes, 256-byte aligned,
 * zero-filled before first use.  Errors (host side): KVQ_ERR_NULL,
 * KVQ_ERR_CONFIG (shape), KVQ_ERR_ARG, KVQ_ERR_CAPACITY (n_seq > 8192),
 * KVQ_ERR_DTYPE, KVQ_ERR_ALIGN, KVQ_ERR_BUFFER_TOO_SMALL; KVQ_ERR_CUDA on
 * launch failure. */
KVQ_API kvq_status kvq_fp16_workspace_bytes(int32_t n_seq, int32_t n_q_heads, int32_t n_kv_heads,
                                            int32_t head_dim, size_t* bytes);
KVQ_API kvq_status kvq_decode_fp16(const void* k, const void* v, const int32_t* lens,
                                   int32_t max_tokens, int32_t n_seq, int32_t n_q_heads,
                                   int32_t n_kv_heads, int32_t head_dim, const void* q,
                                   kvq_dtype q_dtype, void* out, void* workspace,
                                   size_t ws_bytes, void* stream);

/* Size in bytes of the fixed scratch array used by kvq_decode_noalloc. */
KVQ_API size_t kvq_noalloc_scratch_bytes(void);

/* Zero-fill a decode workspace on stream (cudaMemsetAsync). */
KVQ_API kvq_status kvq_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Read the workspace error word (synchronous copy on stream): KVQ_OK, or
 * KVQ_ERR_DEVICE if some decode kernel gave up a bounded wait. */
KVQ_API kvq_status kvq_workspace_status(const void* workspace, void* stream);

/* Refresh the host length mirror from the device copy (synchronizes
 * stream).  Needed after replaying captured appends. */
KVQ_API kvq_status kvq_sync_lengths(kvq_cache* cache, void* stream);

/* The configuration, layout and host length mirror of a handle. */
KVQ_API kvq_status kvq_cache_config(const kvq_cache* cache, kvq_config* out);
KVQ_API kvq_status kvq_cache_layout(const kvq_cache* cache, kvq_layout* out);
KVQ_API kvq_status kvq_get_lengths(const kvq_cache* cache, int32_t* host_lens, int32_t n);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
