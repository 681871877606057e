/*
 * kvq.h — C ABI of the key-priority mixed-precision KV-cache library.
 *
 * What it computes
 * ----------------
 * "Quantize What Counts: More for Keys, Less for Values" (summary page,
 * sections "Problem statement" and "Methodology") stores the KV cache of an
 * LLM at reduced precision and gives keys more bits than values (b_k > b_v,
 * e.g. K4V2), because key errors are amplified through the attention map
 * while value errors are not ("Key-Priority Quantization Theorem").
 * The page fixes neither the quantizer nor the kernel.  This library uses the
 * plainest reading that the rest of the page supports:
 *
 *   * group-wise, uniform, asymmetric min-max quantization along head_dim,
 *     one (scale, zero) pair per group of `group` (keys) or `group_v`
 *     (values) consecutive elements, stored
 *     as IEEE binary16 (the page's "group size" knob, section "Results",
 *     "Group-size sensitivity");
 *   * b-bit codes, b in {2, 4, 8}, bit-packed (the page's K4V2 / K2V4 /
 *     K4V4 / K8 allocations, sections "Key contributions" and "Results");
 *   * decode attention that reads the packed cache directly (the inference
 *     step whose memory traffic motivates the page, "Problem statement").
 *
 * Quantizer (per row r = (batch, kv_head, token), per group of G elements,
 * every step in IEEE binary32, round-to-nearest-even, no fused multiply-add):
 *   1. mn = min x_i, mx = max x_i over the group; then mn = mn + 0.0f and
 *      mx = mx + 0.0f (a zero extreme is +0 whatever the order of reduction,
 *      so the stored binary16 patterns are unique).
 *   2. range = mx - mn;  scale = range / (2^b - 1);  inv = 1 / scale.
 *   3. If scale == 0, or scale or inv is not finite, every code is 0
 *      (degenerate group).  Otherwise
 *      code_i = clamp(rint((x_i - mn) * inv), 0, 2^b - 1).
 *   4. Stored parameters: scale16 = binary16(scale), zero16 = binary16(mn),
 *      both rounded to nearest even.  Codes use the binary32 scale/mn.
 *   Dequantised value: x^ = code * scale16 + zero16.
 *   Inputs must be finite with |x| <= 65504 (binary16 range of the stored
 *   parameters); NaN or Inf inputs give unspecified codes.
 *
 * Decode attention (per batch row b and query head hq, kv head
 * h = hq / (Hq / Hkv)):
 *   s_t = sm_scale * sum_d q_d * k^_{t,d},   t in [0, seq_lens[b])
 *   o_d = sum_t softmax(s)_t * v^_{t,d}
 * computed in binary32 with exact integer codes (see kvq_decode_attention).
 * A sequence of length 0 yields o = 0.
 *
 * Cache format
 * ------------
 * The cache of one layer is B x Hkv "slots"; each slot holds `capacity`
 * token positions.  Four arrays, each slot-major ([B][Hkv][...]), all owned
 * by the caller:
 *
 *   k_codes : capacity * (D * b_k / 8) bytes per slot  (K rows)
 *   v_codes : capacity * (D * b_v / 8) bytes per slot  (V tiles)
 *   k_params: capacity * (D / Gk) * 4  bytes per slot  (K scale/zero)
 *   v_params: capacity * (D / Gv) * 4  bytes per slot  (V scale/zero)
 *
 * Gk = group, Gv = group_v (or group).  Params: for token position p and
 * group g of an array with group size G, the 4 bytes at offset
 * (p * (D/G) + g) * 4 hold binary16 scale (lower address) then binary16 zero.
 *
 * K rows (token-major; row p at byte offset p * D*b/8 of the slot).  With
 * E = 16 / b codes per 16-bit half-word, the code of element d goes to
 *     slice  c = (d mod 8) / 2         (slice c = bytes [c*D*b/32, (c+1)*D*b/32))
 *     word   w = (d / 8) / E           (little-endian 32-bit word w of the slice)
 *     bits   16*(d mod 2) + b*((d / 8) mod E)   .. + b - 1   of that word.
 *
 * V tiles (16 consecutive positions form a tile; tile j at byte offset
 * j * 2*D*b of the slot).  Inside a tile the bytes belong to 32 "lanes" of
 * N = D*b/16 bytes each, stored in pieces of P = min(16, N) bytes:
 * lane L's byte n lives at offset (n / P) * 32*P + L*P + (n mod P).
 * For position p (k = p mod 16) and element d, with E = 16/b and
 * W = D*b/128 words per half-lane:
 *     lane  L = 4*(d mod 8) + (k mod 8)/2
 *     word  q = (k / 8) * W + (d / 8) / E      (little-endian, bytes 4q..4q+3 of the lane)
 *     bits  16*(k mod 2) + b*((d / 8) mod E)   .. + b - 1   of that word.
 *
 * Both layouts put every code at the place where one m16n8k16 tensor-core
 * fragment of the decode kernel wants it, so that the kernel loads each
 * fragment with one wide shared-memory read and unpacks two codes with one
 * logic operation.  Every byte belongs to one token position, except that a
 * V word is shared by two positions (each owns one 16-bit half); appends of
 * any length and alignment are supported.
 *
 * Conventions
 * -----------
 * All data pointers are device pointers owned by the caller; the library
 * never allocates.  Calls are asynchronous on `stream` (NULL = legacy default
 * stream).  Host-side argument errors are returned before anything is
 * launched.  Conditions only the device can see (an append past `capacity`,
 * a length above `max_seq_len` or `capacity`, a bounded wait that ran out)
 * set bits in a per-device error word that kvq_device_error_flags() reads and
 * clears; the offending rows are skipped or clamped, never written out of
 * bounds.  A paged cache's block-table entries are device data too: an entry
 * outside the pool is flagged and never followed.  Layouts of K, V, Q and out are row-major with head_dim innermost.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, without requiring the CUDA headers. */
typedef struct CUstream_st* kvq_stream_t;

/* Element types of K, V, Q and the attention output. */
enum kvq_dtype {
  KVQ_F32 = 0,  /* IEEE binary32 */
  KVQ_BF16 = 1, /* bfloat16 */
  KVQ_F16 = 2   /* IEEE binary16 */
};

/* Status codes returned by every entry point. */
enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1, /* a size, pointer, alignment or enum is invalid */
  KVQ_ERR_UNSUPPORTED = 2, /* valid but not supported (e.g. bits = 3)       */
  KVQ_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required    */
  KVQ_ERR_CUDA = 4         /* a CUDA runtime call or kernel launch failed   */
};

/* Bits of the per-device error word (kvq_device_error_flags). */
enum kvq_device_error {
  KVQ_DEVERR_CAPACITY = 1u,    /* append with pos + n_new > capacity (rows skipped)   */
  KVQ_DEVERR_SEQ_LEN = 2u,     /* seq_lens[b] > max_seq_len or capacity (clamped)     */
  KVQ_DEVERR_TIMEOUT = 4u,     /* a bounded shared-memory pipeline wait gave up       */
  KVQ_DEVERR_BAD_POS = 8u,     /* pos[b] < 0 (rows skipped)                            */
  KVQ_DEVERR_BAD_PAGE = 16u    /* block_table entry outside [0, num_pages) (see below) */
};

/* Bits of kvq_cache_desc.flags. */
enum kvq_cache_flags {
  /* Key-only rotation (summary page "Quantize What Counts", "Results",
   * "Integration with rotation": rotating only the keys of a K4V2 cache comes
   * close to K4V4).  Each key row is stored as H k, H the unnormalised
   * Walsh-Hadamard matrix of size D (Sylvester order, H[i][j] =
   * (-1)^popcount(i & j)), computed before quantization by the butterfly
   * for h = 1, 2, ..., D/2: (x[i], x[i+h]) <- (x[i] + x[i+h], x[i] - x[i+h])
   * for i & h == 0, each step a binary32 operation rounded to nearest even;
   * the groups, scales and zeros then apply to H k.  Decode multiplies the
   * query by H / D, so scores are unchanged in exact arithmetic
   * ((H q / D) . (H k) = q . k).  Values are never rotated. */
  KVQ_FLAG_ROTATE_KEYS = 1,
  /* Paged layout (block tables): the cache is a pool of `num_pages` pages of
   * `page_size` positions, and each batch row maps its logical positions to
   * pages through `block_table`, so that ragged batches need no per-row
   * capacity padding and rows can share pages (prefixes).  This is a
   * serving-system variant of the cache format, not something the summary
   * page describes; the codes, parameters and their placement inside a page
   * are exactly those of the slot format above.  See kvq_cache_desc. */
  KVQ_FLAG_PAGED = 2
};

/* Which array kvq_cache_bytes() sizes. */
enum kvq_cache_array {
  KVQ_K_CODES = 0,
  KVQ_V_CODES = 1,
  KVQ_K_PARAMS = 2,
  KVQ_V_PARAMS = 3
};

/*
 * One layer's packed cache.  Sizes:
 *   batch (B) >= 1, kv_heads (Hkv) >= 1, head_dim (D) in {64, 128},
 *   capacity >= 16 and a multiple of 16 token positions per slot,
 *   bits_k, bits_v in {2, 4, 8} (the page's key-priority rule is b_k > b_v;
 *   other orders are accepted so that they can be compared),
 *   group (G) in {32, 64, 128} with G <= D: the keys' group size;
 *   group_v: the values' group size, 0 (= group) or in {32, 64, 128} with
 *   group <= group_v <= D ("Results", "Group-size sensitivity": finer
 *   groups help the keys, coarser ones are enough for the values).
 * Pointers: device memory, 16-byte aligned, sized by kvq_cache_bytes().
 *
 * Paged layout (flags & KVQ_FLAG_PAGED):
 *   page_size (P): positions per page, a power of two >= 32 that divides
 *     capacity; capacity is the logical length limit of every batch row.
 *   num_pages: pages in the pool, >= 1.  A page holds P positions of all
 *     kv_heads: the four arrays are page-major, [num_pages][Hkv][...], and
 *     (page, h) is laid out exactly like a slot of capacity P above.  Size
 *     them with kvq_cache_bytes(num_pages, kv_heads, head_dim, page_size,
 *     ...).
 *   block_table: device int32 [batch][capacity / P], 4-byte aligned:
 *     positions [j*P, (j+1)*P) of batch row b live at local positions
 *     0 .. P-1 of page block_table[b * (capacity / P) + j].  Entries that a
 *     call never reaches are not read.  Rows may share pages for reading;
 *     the pages one kvq_quantize_append() call writes must not be shared
 *     between its batch rows (their writes would race).  An entry outside
 *     [0, num_pages) that a call reaches flags KVQ_DEVERR_BAD_PAGE: an
 *     append skips the 16-position tiles that map to it; decode attention
 *     reads nothing from it and that row's output is unspecified.
 * Without the flag, page_size and num_pages must be 0 and block_table NULL.
 */
typedef struct kvq_cache_desc {
  int32_t batch;
  int32_t kv_heads;
  int32_t head_dim;
  int32_t capacity;
  int32_t bits_k;
  int32_t bits_v;
  int32_t group;
  int32_t flags;    /* kvq_cache_flags; other bits must be 0 */
  int32_t group_v;  /* values' group size; 0: same as group */
  int32_t reserved; /* must be 0 */
  uint8_t* k_codes;
  uint8_t* v_codes;
  void* k_params; /* binary16 (scale, zero) pairs */
  void* v_params; /* binary16 (scale, zero) pairs */
  int32_t page_size;            /* KVQ_FLAG_PAGED: positions per page; else 0 */
  int32_t num_pages;            /* KVQ_FLAG_PAGED: pages in the pool; else 0 */
  const int32_t* block_table;   /* KVQ_FLAG_PAGED: [batch][capacity / page_size] */
} kvq_cache_desc;

/*
 * Bytes of one cache array for the given shape (all slots), or 0 if the
 * shape is invalid.  `group` is the group size of the array asked for: the
 * keys' for KVQ_K_PARAMS, the values' for KVQ_V_PARAMS.  For a paged cache
 * pass batch = num_pages and capacity = page_size.  Pure host function.
 */
size_t kvq_cache_bytes(int32_t batch, int32_t kv_heads, int32_t head_dim,
                       int32_t capacity, int32_t bits_k, int32_t bits_v,
                       int32_t group, int32_t which);

/*
 * Checks a descriptor on the host (shape, alignment, non-null pointers).
 * Returns KVQ_OK, KVQ_ERR_INVALID_ARG or KVQ_ERR_UNSUPPORTED.  No CUDA call.
 */
int kvq_validate_cache(const kvq_cache_desc* cache);

/*
 * Quantize-and-append: the cache write of "Quantize What Counts" (summary
 * page, "Problem statement": the BF16 cache is stored at 4 bits or fewer;
 * "Key contributions": keys at b_k, values at b_v bits).
 *
 *   k, v   : device, [B][Hkv][n_new][D] row-major, element type in_dtype
 *            (KVQ_F32, KVQ_BF16 or KVQ_F16), 16-byte aligned.
 *   pos    : device int32[B]; batch row b writes positions
 *            [pos[b], pos[b] + n_new) of each of its Hkv slots.
 *   n_new  : >= 1 new tokens per batch row (n_new = 0 is a no-op).
 *
 * Writes codes and binary16 (scale, zero) for keys with bits_k and values
 * with bits_v, in the format above.  Positions outside the new range are not
 * touched (the other half of a shared V word is preserved).  Rows whose
 * range would pass `capacity` (or with pos[b] < 0) are skipped and flag
 * KVQ_DEVERR_CAPACITY (KVQ_DEVERR_BAD_POS).  Paged layout: each 16-position
 * tile is written to the page its block-table entry names; tiles whose entry
 * is outside [0, num_pages) are skipped and flag KVQ_DEVERR_BAD_PAGE.  Does not advance any length:
 * the caller owns seq_lens.  One kernel launch.
 */
int kvq_quantize_append(const kvq_cache_desc* cache, const void* k,
                        const void* v, int32_t in_dtype, const int32_t* pos,
                        int32_t n_new, kvq_stream_t stream);

/*
 * Workspace bytes kvq_decode_attention() needs for this cache, number of
 * query heads and maximum length, on the current device (the split-K plan
 * depends on its SM count).  0 if the arguments are invalid, and 0 when
 * every row fits in one split (no workspace is needed then).
 */
size_t kvq_decode_workspace_bytes(const kvq_cache_desc* cache,
                                  int32_t num_q_heads, int32_t max_seq_len);

/*
 * Decode attention over the packed cache (one query token per batch row).
 *
 *   q           : device, [B][Hq][D] row-major, q_dtype in {F32, BF16, F16}.
 *   num_q_heads : Hq, a multiple of Hkv (grouped-query attention; query
 *                 head hq reads kv head hq / (Hq / Hkv)).
 *   seq_lens    : device int32[B]; batch row b attends to positions
 *                 [0, seq_lens[b]).  Values above max_seq_len or capacity
 *                 are clamped and flag KVQ_DEVERR_SEQ_LEN.  Paged layout:
 *                 positions are read through the block table; a row that
 *                 reaches an entry outside the pool flags
 *                 KVQ_DEVERR_BAD_PAGE and its output is unspecified.
 *   max_seq_len : host upper bound of seq_lens (sizes the split-K grid).
 *   sm_scale    : softmax scale; <= 0 selects 1/sqrt(D).
 *   out         : device, [B][Hq][D], out_dtype in {F32, BF16, F16}.
 *   workspace   : device scratch of at least kvq_decode_workspace_bytes(),
 *                 16-byte aligned (may be NULL when that is 0); holds the
 *                 per-split partial outputs and log-sum-exps.
 *
 * Kernel launches on `stream`: split-K flash-decoding over the packed cache,
 * then a log-sum-exp combine of the splits; when every row fits in one
 * split, the decode kernel writes the output itself (one launch).
 * Arithmetic: codes are exact in binary16, products and sums in binary32
 * (tensor cores), softmax in binary32.
 */
int kvq_decode_attention(const kvq_cache_desc* cache, const void* q,
                         int32_t q_dtype, int32_t num_q_heads,
                         const int32_t* seq_lens, int32_t max_seq_len,
                         float sm_scale, void* out, int32_t out_dtype,
                         void* workspace, size_t workspace_bytes,
                         kvq_stream_t stream);

/*
 * Decode attention with the step's append fused in (one launch, plus the
 * combine when rows are split): the same result as
 *   kvq_quantize_append(cache, k_new, v_new, in_dtype, pos, n_new, stream)
 *   kvq_decode_attention(cache, q, ..., seq_lens, ...)
 * with pos[b] = seq_lens[b] - n_new, i.e. the n_new new tokens of every batch
 * row are the last ones it attends to (a decode step that appends its own
 * key and value rows).  The split-K CTA that owns a new position quantizes
 * and writes it before reading it ("Quantize What Counts", summary page,
 * "Problem statement": the cache is written once per token and read by
 * every later step).
 *
 *   k_new, v_new : device, [B][Hkv][n_new][D] row-major, in_dtype (F32, BF16
 *                  or F16), 16-byte aligned.  n_new = 0: plain decode.
 *   other arguments as for kvq_decode_attention(); the workspace size is the
 *   same (kvq_decode_workspace_bytes()).
 *
 * Rows with seq_lens[b] < n_new append nothing and flag KVQ_DEVERR_BAD_POS;
 * rows whose length is clamped (KVQ_DEVERR_SEQ_LEN) append nothing.  The
 * written bytes equal those of kvq_quantize_append() (same quantizer, same
 * format; positions outside the new range keep their bytes).
 * When one kv head serves more query heads than one CTA takes (more than 8),
 * every CTA of that kv head writes the new rows itself, without waiting for
 * the others: the stores are whole 32-bit words (K codes, parameters) or
 * 16-bit halves (V codes) carrying identical bits, so a copy that reads a
 * row while another CTA stores it sees the same value either way.  Nothing
 * else about the result depends on that ordering.
 */
int kvq_append_decode_attention(const kvq_cache_desc* cache, const void* k_new,
                                const void* v_new, int32_t in_dtype, int32_t n_new,
                                const void* q, int32_t q_dtype, int32_t num_q_heads,
                                const int32_t* seq_lens, int32_t max_seq_len,
                                float sm_scale, void* out, int32_t out_dtype,
                                void* workspace, size_t workspace_bytes,
                                kvq_stream_t stream);

/*
 * Size of the fixed device scratch array used by
 * kvq_decode_attention_static(): 4 MiB, held on every device that loads the
 * library until the process exits.
 */
#define KVQ_STATIC_SCRATCH_BYTES (4u << 20)

/*
 * kvq_decode_attention() for callers that cannot allocate device memory.
 * The summary page has no counterpart to this call; it exists for engines
 * that must not call cudaMalloc on the request path (it can synchronize the
 * device and fail under fragmentation) and for plain-C hosts without a
 * device allocator.  Arguments as for kvq_decode_attention(), minus the
 * workspace: the split-K partial results go to a fixed array of
 * KVQ_STATIC_SCRATCH_BYTES inside the library's device image.
 *   - Returns KVQ_ERR_WORKSPACE, launching nothing, when this shape needs
 *     more scratch than that (kvq_decode_workspace_bytes() tells how much).
 *   - Allocates nothing.  The first call on each device looks up the array's
 *     device address (cudaGetSymbolAddress) with that device current; make
 *     that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; nothing in it needs to start at zero.  Calls whose kernels
 *     may overlap on the GPU (different streams without ordering between
 *     them) race on the array: serialize them.
 */
int kvq_decode_attention_static(const kvq_cache_desc* cache, const void* q,
                                int32_t q_dtype, int32_t num_q_heads,
                                const int32_t* seq_lens, int32_t max_seq_len,
                                float sm_scale, void* out, int32_t out_dtype,
                                kvq_stream_t stream);

/*
 * Tokens per split that kvq_decode_attention() will use for these
 * arguments on the current device (0 if invalid).  Informational.
 *
 * Environment read when a decode plan is made (plans are cached per shape
 * and per these settings; results stay within the attention tolerance
 * under every setting):
 *   KVQ_SPLIT_TOKENS=n       split size override, a multiple of 64 (tests);
 *   KVQ_DECODE_SCHEDULE=balanced  one wave of CTAs sharing all rows' stages
 *                            equally (stream-K); slower than the default
 *                            per-row splits on B200, kept for comparison;
 *   KVQ_DECODE_KERNEL=tcgen05     the tensor-memory (tcgen05) decode kernel
 *                            for head_dim 128; slower than the default,
 *                            kept for comparison.
 */
int32_t kvq_decode_split_tokens(const kvq_cache_desc* cache,
                                int32_t num_q_heads, int32_t max_seq_len);

/*
 * Failure-detection test knob; not for production use.  The summary page has
 * no counterpart: it exists so that a test can make a bounded device wait run
 * out without faulting or hanging the GPU.  With drop_stage 0 or 1, the next
 * decode-attention launch in this process (only that one) makes stage
 * `drop_stage` of the first warp's copy pipeline in its first CTA expect 16
 * bytes more than its copies bring, and every bounded wait of that launch
 * gives up after wait_limit_ns (1000 .. 1e9 ns) instead of one second.  The
 * wait on that stage then runs out: the kernel flags KVQ_DEVERR_TIMEOUT,
 * waits (bounded) for its copies in flight, and returns; that call's output
 * is unspecified, and the cache is untouched.  drop_stage < 0 disarms the
 * knob.  Returns KVQ_OK, or KVQ_ERR_INVALID_ARG for a stage above 1 or a
 * limit out of range.
 */
int kvq_debug_inject_wait_timeout(int32_t drop_stage, int64_t wait_limit_ns);

/*
 * Reads and clears the current device's error word (bits of
 * kvq_device_error) after synchronizing `stream`.  Returns KVQ_OK or
 * KVQ_ERR_CUDA.
 */
int kvq_device_error_flags(kvq_stream_t stream, uint32_t* flags);

/*
 * The same read-and-clear in one return value: the error word's bits
 * (kvq_device_error, >= 0) after synchronizing `stream`, or -KVQ_ERR_CUDA
 * if the copy or the synchronization failed.
 */
int kvq_last_device_error(kvq_stream_t stream);

/* Static text for a kvq_status value. */
const char* kvq_strerror(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
