// Host side of the C ABI declared in kvq.h: argument validation, the
// split-K plan, kernel selection and launches.  No allocation anywhere.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <tuple>
#include <utility>

#include "internal.h"

namespace kvq {
bool get_decode_kernel_k2v2(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k2v4(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k2v8(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k4v2(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k4v4(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k4v8(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k8v2(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k8v4(int, int, int, int, DecodeKernel*);
bool get_decode_kernel_k8v8(int, int, int, int, DecodeKernel*);

bool get_decode_tc_kernel_k2v2(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k2v4(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k2v8(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k4v2(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k4v4(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k4v8(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k8v2(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k8v4(int, int, int, DecodeKernel*);
bool get_decode_tc_kernel_k8v8(int, int, int, DecodeKernel*);

bool get_decode_tc_kernel(int bits_k, int bits_v, int groups_k, int groups_v, int heads_per_cta,
                          DecodeKernel* out) {
  using Fn = bool (*)(int, int, int, DecodeKernel*);
  static const Fn table[3][3] = {
      {get_decode_tc_kernel_k2v2, get_decode_tc_kernel_k2v4, get_decode_tc_kernel_k2v8},
      {get_decode_tc_kernel_k4v2, get_decode_tc_kernel_k4v4, get_decode_tc_kernel_k4v8},
      {get_decode_tc_kernel_k8v2, get_decode_tc_kernel_k8v4, get_decode_tc_kernel_k8v8}};
  auto idx = [](int b) { return b == 2 ? 0 : b == 4 ? 1 : b == 8 ? 2 : -1; };
  const int i = idx(bits_k), j = idx(bits_v);
  if (i < 0 || j < 0) return false;
  return table[i][j](groups_k, groups_v, heads_per_cta, out);
}

bool get_decode_kernel(int head_dim, int bits_k, int bits_v, int groups_k, int groups_v,
                       int variant, DecodeKernel* out) {
  using Fn = bool (*)(int, int, int, int, DecodeKernel*);
  static const Fn table[3][3] = {
      {get_decode_kernel_k2v2, get_decode_kernel_k2v4, get_decode_kernel_k2v8},
      {get_decode_kernel_k4v2, get_decode_kernel_k4v4, get_decode_kernel_k4v8},
      {get_decode_kernel_k8v2, get_decode_kernel_k8v4, get_decode_kernel_k8v8}};
  auto idx = [](int b) { return b == 2 ? 0 : b == 4 ? 1 : b == 8 ? 2 : -1; };
  const int i = idx(bits_k), j = idx(bits_v);
  if (i < 0 || j < 0) return false;
  return table[i][j](head_dim, groups_k, groups_v, variant, out);
}
}  // namespace kvq

// Per-device error word (one copy on every device that loads the library).
static __device__ uint32_t g_kvq_device_error;

// Armed failure-detection test knob (kvq_debug_inject_wait_timeout): the
// stage to drop in the next decode launch (-1: none) and its wait limit.
static std::atomic<long long> g_fault_stage{-1};
static std::atomic<long long> g_fault_limit_ns{0};

namespace {

using kvq::DecodeKernel;

constexpr int kMaxDevices = 64;

int to_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_bits(int b) { return b == 2 || b == 4 || b == 8; }

int check_shape(int B, int Hkv, int D, int cap, int bk, int bv, int G) {
  if (B < 1 || Hkv < 1 || cap < 16 || cap % 16 != 0) return KVQ_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return KVQ_ERR_UNSUPPORTED;
  if (!valid_bits(bk) || !valid_bits(bv)) return KVQ_ERR_UNSUPPORTED;
  if (G != 32 && G != 64 && G != 128) return KVQ_ERR_UNSUPPORTED;
  if (G > D) return KVQ_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535) return KVQ_ERR_UNSUPPORTED;  // grid limits
  return KVQ_OK;
}

// Values' group size (group_v = 0 means the keys' group).
int group_v_of(const kvq_cache_desc* c) { return c->group_v != 0 ? c->group_v : c->group; }

int check_cache(const kvq_cache_desc* c) {
  if (!c || (c->flags & ~(KVQ_FLAG_ROTATE_KEYS | KVQ_FLAG_PAGED)) != 0 || c->reserved != 0)
    return KVQ_ERR_INVALID_ARG;
  int st = check_shape(c->batch, c->kv_heads, c->head_dim, c->capacity, c->bits_k, c->bits_v,
                       c->group);
  if (st != KVQ_OK) return st;
  const int gv = group_v_of(c);
  st = check_shape(c->batch, c->kv_heads, c->head_dim, c->capacity, c->bits_k, c->bits_v, gv);
  if (st != KVQ_OK) return st;
  // instances exist for equal groups and for coarser value groups
  if (gv < c->group) return KVQ_ERR_UNSUPPORTED;
  const void* ptrs[4] = {c->k_codes, c->v_codes, c->k_params, c->v_params};
  for (const void* p : ptrs)
    if (!p || !aligned(p, 16)) return KVQ_ERR_INVALID_ARG;
  if (c->flags & KVQ_FLAG_PAGED) {
    // pages of a power-of-two number of positions, at least one decode
    // stage (32 positions) so that no copy crosses a page
    const int P = c->page_size;
    if (P < 32 || (P & (P - 1)) != 0 || c->capacity % P != 0 || c->num_pages < 1 ||
        !c->block_table || !aligned(c->block_table, 4))
      return KVQ_ERR_INVALID_ARG;
  } else if (c->page_size != 0 || c->num_pages != 0 || c->block_table) {
    return KVQ_ERR_INVALID_ARG;
  }
  return KVQ_OK;
}

// Page mapping of a cache (block_table NULL: slot layout).
void page_args(const kvq_cache_desc* c, const int32_t** table, int* shift, int* per_seq,
               int* num_pages) {
  const bool paged = (c->flags & KVQ_FLAG_PAGED) != 0;
  *table = paged ? c->block_table : nullptr;
  int sh = 0;
  while (paged && (1 << sh) < c->page_size) ++sh;
  *shift = sh;
  *per_seq = paged ? c->capacity >> sh : 0;
  *num_pages = paged ? c->num_pages : 0;
}

bool valid_dtype(int t) { return t == KVQ_F32 || t == KVQ_BF16 || t == KVQ_F16; }

// Device address of the error word on the current device (looked up once per
// device; the symbol's host-side name is not a device address).
// Only a successful lookup is kept: a failed one is retried on the next call.
int error_word(uint32_t** out) {
  static std::mutex mu;
  static uint32_t* ptrs[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kvq_device_error) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // reset the runtime's last-error state; the next call retries
      return KVQ_ERR_CUDA;
    }
    ptrs[dev] = static_cast<uint32_t*>(p);
  }
  *out = ptrs[dev];
  return KVQ_OK;
}

int variant_of(int heads_per_cta, int q_dtype);

// Which decode kernel runs.  The register-fragment kernel (mma.sync, codes
// unpacked straight into tensor-core fragments) serves every shape.  The
// tensor-memory kernel (tcgen05, head_dim 128, no fused append) is selected
// with KVQ_DECODE_KERNEL=tcgen05; it computes the same result but measured
// slower on B200 (its small-N products are bound by the tensor core reading
// the unpacked binary16 operands, about 75 cycles per 128x16x16 product).
bool use_tc_kernel(const kvq_cache_desc* c, bool fused) {
  if (c->head_dim != 128 || fused) return false;
  const char* env = std::getenv("KVQ_DECODE_KERNEL");
  return env && std::string(env) == "tcgen05";
}

bool select_decode_kernel(const kvq_cache_desc* c, int heads_per_cta, int q_dtype, bool fused,
                          DecodeKernel* k) {
  const int gk = c->head_dim / c->group, gv = c->head_dim / group_v_of(c);
  if (use_tc_kernel(c, fused))
    return kvq::get_decode_tc_kernel(c->bits_k, c->bits_v, gk, gv, heads_per_cta, k);
  // variant bit 2 selects the paged layout's instances
  const int paged = (c->flags & KVQ_FLAG_PAGED) != 0 ? 4 : 0;
  return kvq::get_decode_kernel(c->head_dim, c->bits_k, c->bits_v, gk, gv,
                                variant_of(heads_per_cta, q_dtype) | paged, k);
}

// Opt a kernel in to more than 48 KB of dynamic shared memory, once per
// (device, kernel).
cudaError_t prepare_kernel(const DecodeKernel& k) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({dev, k.fn})) return cudaSuccess;
  e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem_bytes);
  // the largest shared-memory carveout, so that the occupancy the plan is
  // sized for (several CTAs per SM) is the one the hardware gives
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k.fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && k.fn_fused != nullptr)
    e = cudaFuncSetAttribute(k.fn_fused, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && k.fn_fused != nullptr)
    e = cudaFuncSetAttribute(k.fn_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             k.smem_bytes);
  if (e == cudaSuccess) done.insert({dev, k.fn});
  return e;
}

struct Plan {
  int heads_per_cta, head_groups, split_tokens, num_splits;
  bool direct;         // one split per row: the decode writes the output itself
  size_t ws_o_floats;  // partial outputs [B][Hq][splits][D]
  size_t ws_bytes;     // partials + log-sum-exps (enough for either schedule)
  // Balanced (stream-K) schedule of a plain decode (stream_q > 0): a one-wave
  // grid of stream_grid CTAs, each taking at least stream_q stages;
  // stream_parts partial slots per row.
  int stream_q, stream_grid, stream_parts, stage_tokens;
  size_t stream_o_floats;
};

// Smallest share of stages of a CTA in the balanced schedule (it bounds the
// partial results a unit can leave, hence the workspace).
constexpr int kStreamMinStages = 4;

int variant_of(int heads_per_cta, int q_dtype) {
  return (heads_per_cta <= 4 ? 0 : 2) + (q_dtype == KVQ_F32 ? 1 : 0);
}

// Split-K plan.  Tokens per split are a multiple of 64, at least 256 (per-CTA
// set-up and partial-result traffic).  When one wave of resident CTAs gives
// every (batch row, kv head, head group) at least four splits, use exactly
// one wave: splits are rounded up, so the grid never spills into a second
// wave, and equal lengths finish together.  Otherwise aim at about three
// waves, so that the block scheduler can balance ragged lengths (measured on
// B200 with cold caches: three waves beat four on the ragged batch).  The
// plan depends only on the shape, Hq, max_seq_len and the device.
int make_plan_uncached(const kvq_cache_desc* c, int Hq, int max_seq_len, Plan* p) {
  const int gq = Hq / c->kv_heads;
  p->heads_per_cta = gq < 8 ? gq : 8;
  p->head_groups = (gq + p->heads_per_cta - 1) / p->heads_per_cta;
  if (static_cast<long long>(c->kv_heads) * p->head_groups > 65535) return KVQ_ERR_UNSUPPORTED;
  if (max_seq_len <= 0) {
    p->split_tokens = 64;
    p->num_splits = 0;
    p->direct = false;
    p->ws_o_floats = 0;
    p->ws_bytes = 0;
    return KVQ_OK;
  }
  // the plan is that of the kernel a plain decode runs (the fused append
  // follows the same plan, so that the workspace size does not depend on it)
  DecodeKernel k;
  if (!select_decode_kernel(c, p->heads_per_cta, KVQ_BF16, false, &k)) return KVQ_ERR_UNSUPPORTED;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return KVQ_ERR_CUDA;
  if (prepare_kernel(k) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k.fn, k.threads, k.smem_bytes) !=
          cudaSuccess)
    return KVQ_ERR_CUDA;
  if (k.max_per_sm > 0 && per_sm > k.max_per_sm) per_sm = k.max_per_sm;
  if (per_sm < 1) per_sm = 1;
  const long long units = static_cast<long long>(c->batch) * c->kv_heads * p->head_groups;
  const long long slots = static_cast<long long>(sms) * per_sm;
  const long long T = k.tile;  // splits are whole tiles of the kernel
  const long long max_t = (max_seq_len + T - 1) / T * T;
  long long split;
  if (slots >= 4 * units) {
    const long long per_unit = slots / units;
    split = ((max_seq_len + per_unit - 1) / per_unit + T - 1) / T * T;
  } else {
    const long long work = units * max_seq_len;
    split = ((work + 3 * slots - 1) / (3 * slots) + T - 1) / T * T;
  }
  if (split < 256) split = 256;
  if (split > max_t) split = max_t;
  if (const char* env = std::getenv("KVQ_SPLIT_TOKENS")) {
    const long long v = std::atoll(env);
    if (v >= 64 && v % 64 == 0) split = v;
  }
  p->split_tokens = static_cast<int>(split);
  p->num_splits = static_cast<int>((max_seq_len + split - 1) / split);
  if (p->num_splits > 65535) return KVQ_ERR_UNSUPPORTED;
  p->direct = p->num_splits == 1;
  p->ws_o_floats = static_cast<size_t>(c->batch) * Hq * p->num_splits * c->head_dim;
  if (p->direct) {
    p->ws_bytes = 0;  // every CTA writes its rows' final output
  } else {
    p->ws_bytes = static_cast<size_t>(c->batch) * Hq * p->num_splits * (c->head_dim + 1) * 4;
    p->ws_bytes = (p->ws_bytes + 15) / 16 * 16;
  }
  // Balanced schedule (KVQ_DECODE_SCHEDULE=balanced), when rows need
  // splitting anyway and the batch fits the kernel's row table: one wave of
  // CTAs with equal shares of stages.  Not the default: measured on B200, a
  // span costs about as much as four stages of fixed work, and SMs of
  // different GPCs stream at speeds up to ~15% apart, so a static partition
  // ends later than the block scheduler's dynamic one on the ragged batch.
  p->stream_q = 0;
  p->stream_grid = 0;
  p->stream_parts = 0;
  p->stage_tokens = k.stage_tokens;
  p->stream_o_floats = 0;
  const char* sched = std::getenv("KVQ_DECODE_SCHEDULE");
  const bool stream_ok = sched && std::string(sched) == "balanced" &&
                         std::getenv("KVQ_SPLIT_TOKENS") == nullptr;
  if (stream_ok && !p->direct && k.stage_tokens > 0 && c->batch <= kvq::kStreamRows) {
    const long long ns_max = (max_seq_len + k.stage_tokens - 1) / k.stage_tokens;
    p->stream_q = kStreamMinStages;
    p->stream_grid = static_cast<int>(slots);
    p->stream_parts = static_cast<int>((ns_max + kStreamMinStages - 1) / kStreamMinStages + 1);
    p->stream_o_floats = static_cast<size_t>(c->batch) * Hq * p->stream_parts * c->head_dim;
    size_t sb = static_cast<size_t>(c->batch) * Hq * p->stream_parts * (c->head_dim + 1) * 4;
    sb = (sb + 15) / 16 * 16;
    if (sb > p->ws_bytes) p->ws_bytes = sb;
  }
  return KVQ_OK;
}

// Plans are cached per (device, shape incl. both group sizes and the flags,
// Hq, max_seq_len, split override): the occupancy query behind a plan costs
// microseconds of host time.  The plan never depends on the query type (the
// workspace size is queried without it), so the occupancy of the 16-bit
// query instance stands for every query type.
int make_plan(const kvq_cache_desc* c, int Hq, int max_seq_len, Plan* p) {
  using Key = std::tuple<int, int, int, int, int, int, int, int, int, int, int, int, long long>;
  static std::mutex mu;
  static std::map<Key, Plan> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  long long override_split = 0;
  if (const char* env = std::getenv("KVQ_SPLIT_TOKENS")) override_split = std::atoll(env);
  if (const char* env = std::getenv("KVQ_DECODE_SCHEDULE"))
    if (std::string(env) == "balanced") override_split = -1 - override_split;
  const Key key{dev, c->batch, c->kv_heads, c->head_dim, c->bits_k, c->bits_v, c->group,
                group_v_of(c), (c->flags << 1) | (use_tc_kernel(c, false) ? 1 : 0), Hq,
                max_seq_len, c->capacity, override_split};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *p = it->second;
      return KVQ_OK;
    }
  }
  const int st = make_plan_uncached(c, Hq, max_seq_len, p);
  if (st == KVQ_OK) {
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() > 4096) cache.clear();
    cache.emplace(key, *p);
  }
  return st;
}

int check_decode_args(const kvq_cache_desc* c, int Hq, int max_seq_len) {
  const int st = check_cache(c);
  if (st != KVQ_OK) return st;
  if (Hq < 1 || Hq % c->kv_heads != 0 || max_seq_len < 0) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

}  // namespace

extern "C" {

size_t kvq_cache_bytes(int32_t batch, int32_t kv_heads, int32_t head_dim, int32_t capacity,
                       int32_t bits_k, int32_t bits_v, int32_t group, int32_t which) {
  if (check_shape(batch, kv_heads, head_dim, capacity, bits_k, bits_v, group) != KVQ_OK) return 0;
  const size_t slots = static_cast<size_t>(batch) * kv_heads;
  switch (which) {
    case KVQ_K_CODES: return slots * capacity * head_dim * bits_k / 8;
    case KVQ_V_CODES: return slots * capacity * head_dim * bits_v / 8;
    case KVQ_K_PARAMS:
    case KVQ_V_PARAMS: return slots * capacity * (head_dim / group) * 4;
    default: return 0;
  }
}

int kvq_validate_cache(const kvq_cache_desc* cache) { return check_cache(cache); }

int kvq_quantize_append(const kvq_cache_desc* cache, const void* k, const void* v,
                        int32_t in_dtype, const int32_t* pos, int32_t n_new,
                        kvq_stream_t stream) {
  int st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (!valid_dtype(in_dtype) || n_new < 0 || n_new > cache->capacity) return KVQ_ERR_INVALID_ARG;
  if (!k || !v || !pos || !aligned(k, 16) || !aligned(v, 16) || !aligned(pos, 4))
    return KVQ_ERR_INVALID_ARG;
  if (n_new == 0) return KVQ_OK;
  kvq::QuantizeArgs a;
  a.k = k;
  a.v = v;
  a.in_dtype = in_dtype;
  a.k_codes = cache->k_codes;
  a.v_codes = cache->v_codes;
  a.k_params = static_cast<uint32_t*>(cache->k_params);
  a.v_params = static_cast<uint32_t*>(cache->v_params);
  a.pos = pos;
  a.n_new = n_new;
  a.batch = cache->batch;
  a.kv_heads = cache->kv_heads;
  a.head_dim = cache->head_dim;
  a.capacity = cache->capacity;
  a.bits_k = cache->bits_k;
  a.bits_v = cache->bits_v;
  a.group = cache->group;
  a.group_v = group_v_of(cache);
  a.rotate_keys = (cache->flags & KVQ_FLAG_ROTATE_KEYS) != 0;
  page_args(cache, &a.block_table, &a.page_shift, &a.pages_per_seq, &a.num_pages);
  st = error_word(&a.err);
  if (st != KVQ_OK) return st;
  return to_status(kvq::launch_quantize_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t kvq_decode_workspace_bytes(const kvq_cache_desc* cache, int32_t num_q_heads,
                                  int32_t max_seq_len) {
  if (check_decode_args(cache, num_q_heads, max_seq_len) != KVQ_OK) return 0;
  Plan p;
  if (make_plan(cache, num_q_heads, max_seq_len, &p) != KVQ_OK) return 0;
  return p.ws_bytes;
}

int32_t kvq_decode_split_tokens(const kvq_cache_desc* cache, int32_t num_q_heads,
                                int32_t max_seq_len) {
  if (check_decode_args(cache, num_q_heads, max_seq_len) != KVQ_OK) return 0;
  Plan p;
  if (make_plan(cache, num_q_heads, max_seq_len, &p) != KVQ_OK) return 0;
  return p.split_tokens;
}

}  // extern "C"

namespace {
// Decode attention, with the step's append fused in when k_new != NULL.
int decode_impl(const kvq_cache_desc* cache, const void* k_new, const void* v_new,
                int32_t in_dtype, int32_t n_new, const void* q, int32_t q_dtype,
                int32_t num_q_heads, const int32_t* seq_lens, int32_t max_seq_len,
                float sm_scale, void* out, int32_t out_dtype, void* workspace,
                size_t workspace_bytes, kvq_stream_t stream) {
  int st = check_decode_args(cache, num_q_heads, max_seq_len);
  if (st != KVQ_OK) return st;
  if (!valid_dtype(q_dtype) || !valid_dtype(out_dtype)) return KVQ_ERR_INVALID_ARG;
  if (!q || !seq_lens || !out || !aligned(q, 16) || !aligned(seq_lens, 4) || !aligned(out, 16))
    return KVQ_ERR_INVALID_ARG;
  if (!(sm_scale == sm_scale)) return KVQ_ERR_INVALID_ARG;  // NaN
  Plan p;
  st = make_plan(cache, num_q_heads, max_seq_len, &p);
  if (st != KVQ_OK) return st;
  if (p.ws_bytes > 0 && (!workspace || !aligned(workspace, 16) || workspace_bytes < p.ws_bytes))
    return KVQ_ERR_WORKSPACE;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int D = cache->head_dim;
  const float scale = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf(static_cast<float>(D));
  float* ws_o = p.ws_bytes > 0 ? static_cast<float*>(workspace) : nullptr;
  float* ws_lse = nullptr;
  bool balanced = false;  // the balanced (stream-K) schedule runs
  if (p.num_splits > 0) {
    DecodeKernel k;
    if (!select_decode_kernel(cache, p.heads_per_cta, q_dtype, k_new != nullptr, &k))
      return KVQ_ERR_UNSUPPORTED;
    // the balanced schedule serves the kernel it was planned for (both the
    // plain and the fused decode, so that they take the same splits)
    balanced = p.stream_q > 0 && k.stage_tokens == p.stage_tokens;
    if (prepare_kernel(k) != cudaSuccess) return KVQ_ERR_CUDA;
    kvq::DecodeArgs a;
    a.k_codes = cache->k_codes;
    a.v_codes = cache->v_codes;
    a.k_params = static_cast<const uint32_t*>(cache->k_params);
    a.v_params = static_cast<const uint32_t*>(cache->v_params);
    a.q = q;
    a.q_dtype = q_dtype;
    a.seq_lens = seq_lens;
    a.batch = cache->batch;
    a.kv_heads = cache->kv_heads;
    a.q_heads = num_q_heads;
    a.gq = num_q_heads / cache->kv_heads;
    a.capacity = cache->capacity;
    a.max_seq_len = max_seq_len;
    a.heads_per_cta = p.heads_per_cta;
    a.head_groups = p.head_groups;
    a.split_tokens = p.split_tokens;
    a.num_splits = balanced ? p.stream_parts : p.num_splits;
    a.stream_q = balanced ? p.stream_q : 0;
    ws_lse = ws_o ? ws_o + (balanced ? p.stream_o_floats : p.ws_o_floats) : nullptr;
    a.sm_scale_log2 = scale * 1.4426950408889634f;
    a.rotate_q = (cache->flags & KVQ_FLAG_ROTATE_KEYS) != 0;
    page_args(cache, &a.block_table, &a.page_shift, &a.pages_per_seq, &a.num_pages);
    a.k_new = k_new;
    a.v_new = v_new;
    a.in_dtype = in_dtype;
    a.n_new = n_new;
    // one-shot test knob: only the next launch after arming it carries it
    const long long fault = g_fault_stage.exchange(-1);
    a.fault_stage = fault >= 0 ? static_cast<int>(fault) : -1;
    a.wait_limit_ns = fault >= 0 ? static_cast<unsigned long long>(g_fault_limit_ns.load())
                                 : 1000000000ull;
    a.ws_o = ws_o;
    a.ws_lse = ws_lse;
    a.direct = p.direct && !balanced;
    a.out = out;
    a.out_dtype = out_dtype;
    st = error_word(&a.err);
    if (st != KVQ_OK) return st;
    // (the fused instance takes the split grid as (units, rows, splits),
    // each row's last split first: see the decode kernel)
    const int units = cache->kv_heads * p.head_groups;
    const dim3 grid = balanced         ? dim3(p.stream_grid, 1, 1)
                      : k_new != nullptr ? dim3(units, cache->batch, p.num_splits)
                                         : dim3(p.num_splits, units, cache->batch);
    if ((k_new != nullptr ? k.launch_fused : k.launch)(a, grid, s) != cudaSuccess)
      return KVQ_ERR_CUDA;
    if (a.direct) return KVQ_OK;
  }
  kvq::CombineArgs ca;
  ca.ws_o = ws_o;
  ca.ws_lse = ws_lse;
  ca.seq_lens = seq_lens;
  ca.out = out;
  ca.out_dtype = out_dtype;
  ca.batch = cache->batch;
  ca.q_heads = num_q_heads;
  ca.head_dim = D;
  ca.capacity = cache->capacity;
  ca.max_seq_len = max_seq_len;
  ca.split_tokens = p.split_tokens;
  ca.num_splits = balanced ? p.stream_parts : p.num_splits;
  ca.stream_q = balanced ? p.stream_q : 0;
  ca.stream_grid = p.stream_grid;
  ca.stage_tokens = p.stage_tokens;
  ca.kv_heads = cache->kv_heads;
  ca.head_groups = p.head_groups;
  ca.gq = num_q_heads / cache->kv_heads;
  ca.heads_per_cta = p.heads_per_cta;
  return to_status(kvq::launch_combine(ca, s));
}
}  // namespace

extern "C" {

int kvq_decode_attention(const kvq_cache_desc* cache, const void* q, int32_t q_dtype,
                         int32_t num_q_heads, const int32_t* seq_lens, int32_t max_seq_len,
                         float sm_scale, void* out, int32_t out_dtype, void* workspace,
                         size_t workspace_bytes, kvq_stream_t stream) {
  return decode_impl(cache, nullptr, nullptr, 0, 0, q, q_dtype, num_q_heads, seq_lens,
                     max_seq_len, sm_scale, out, out_dtype, workspace, workspace_bytes, stream);
}

int kvq_append_decode_attention(const kvq_cache_desc* cache, const void* k_new,
                                const void* v_new, int32_t in_dtype, int32_t n_new,
                                const void* q, int32_t q_dtype, int32_t num_q_heads,
                                const int32_t* seq_lens, int32_t max_seq_len, float sm_scale,
                                void* out, int32_t out_dtype, void* workspace,
                                size_t workspace_bytes, kvq_stream_t stream) {
  if (n_new < 0 || (n_new > 0 && (!valid_dtype(in_dtype) || !k_new || !v_new ||
                                  !aligned(k_new, 16) || !aligned(v_new, 16))))
    return KVQ_ERR_INVALID_ARG;
  return decode_impl(cache, n_new > 0 ? k_new : nullptr, n_new > 0 ? v_new : nullptr, in_dtype,
                     n_new, q, q_dtype, num_q_heads, seq_lens, max_seq_len, sm_scale, out,
                     out_dtype, workspace, workspace_bytes, stream);
}

int kvq_debug_inject_wait_timeout(int32_t drop_stage, int64_t wait_limit_ns) {
  if (drop_stage < 0) {
    g_fault_stage.store(-1);
    return KVQ_OK;
  }
  if (drop_stage > 1) return KVQ_ERR_INVALID_ARG;  // only the first two stages are armed
  if (wait_limit_ns < 1000 || wait_limit_ns > 1000000000LL) return KVQ_ERR_INVALID_ARG;
  g_fault_limit_ns.store(wait_limit_ns);
  g_fault_stage.store(drop_stage);
  return KVQ_OK;
}

int kvq_device_error_flags(kvq_stream_t stream, uint32_t* flags) {
  if (!flags) return KVQ_ERR_INVALID_ARG;
  uint32_t* word = nullptr;
  int st = error_word(&word);
  if (st != KVQ_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, word, sizeof host, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, sizeof host, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  *flags = host;
  return KVQ_OK;
}

int kvq_last_device_error(kvq_stream_t stream) {
  uint32_t flags = 0;
  const int st = kvq_device_error_flags(stream, &flags);
  return st == KVQ_OK ? static_cast<int>(flags & 0x7fffffffu) : -st;
}

const char* kvq_strerror(int32_t status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported shape or option";
    case KVQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
  }
}

}  // extern "C"
