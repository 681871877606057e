// Declarations shared by the host entry points and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// Rows a balanced (stream-K) decode schedules at most (their prefix sums
// live in shared memory).
constexpr int kStreamRows = 256;

// Launches `kernel` with programmatic stream serialization: its blocks may
// start while the previous kernel in the stream finishes, and wait for it in
// pdl_wait() before touching global memory.  Captured into CUDA graphs as a
// programmatic edge.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

struct QuantizeArgs {
  const void* k;
  const void* v;
  int in_dtype;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint32_t* k_params;  // binary16 (scale, zero) pairs
  uint32_t* v_params;
  const int32_t* pos;
  int n_new;
  int batch, kv_heads, head_dim, capacity, bits_k, bits_v, group;
  int group_v;       // values' group size
  uint32_t* err;
  bool rotate_keys;  // store keys as H k (Walsh-Hadamard along head_dim)
  // Paged layout (block_table != NULL): position p of batch row b is local
  // position p mod 2^page_shift of page block_table[b * pages_per_seq +
  // (p >> page_shift)]; (page, kv head) is laid out like a slot of
  // 2^page_shift positions.
  const int32_t* block_table;
  int page_shift, pages_per_seq, num_pages;
};

cudaError_t launch_quantize_append(const QuantizeArgs& a, cudaStream_t stream);

// Split-K decode.  One CTA = one (split, kv head x head group, batch row).
struct DecodeArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint32_t* k_params;
  const uint32_t* v_params;
  const void* q;
  int q_dtype;
  const int32_t* seq_lens;
  int batch, kv_heads, q_heads, gq, capacity, max_seq_len;
  int heads_per_cta;  // <= 8
  int head_groups;    // ceil(gq / heads_per_cta)
  int split_tokens;   // multiple of 64
  int num_splits;     // splits per row (grid.x; grid.z of the fused instance); balanced schedule: partial slots per row
  // Balanced (stream-K) schedule when > 0: grid.x CTAs share the rows' stages
  // evenly, at least stream_q stages each (plain decode only).
  int stream_q;
  float sm_scale_log2;  // softmax scale times log2(e)
  bool rotate_q;        // keys are stored rotated: use H q / D
  const int32_t* block_table;  // paged layout, as in QuantizeArgs (NULL: slots)
  int page_shift, pages_per_seq, num_pages;
  // Fused append (NULL k_new: none): before attending, each CTA quantizes
  // the new rows k_new / v_new ([B][Hkv][n_new][D], element type in_dtype)
  // of positions [seq_lens[b] - n_new, seq_lens[b]) that fall in its split.
  const void* k_new;
  const void* v_new;
  int in_dtype, n_new;
  // Failure-detection test knob (kvq_debug_inject_wait_timeout): when
  // fault_stage is 0 or 1, that stage of the first CTA's first warp expects
  // 16 bytes more than its copies bring, so that the wait on it runs out;
  // every bounded wait of the launch gives up after wait_limit_ns.
  int fault_stage;
  unsigned long long wait_limit_ns;
  float* ws_o;        // [B][Hq][num_splits][D] partial outputs
  float* ws_lse;      // [B][Hq][num_splits] log2-domain log-sum-exp
  uint32_t* err;
  // One split per row (num_splits == 1): each CTA writes its rows' final
  // output to `out` (no partials, no combine launch).
  bool direct;
  void* out;
  int out_dtype;
};

// Kernel variant, from the query type and the number of heads per CTA:
//   0: 16-bit Q, <= 4 heads    1: fp32 Q, <= 4 heads
//   2: 16-bit Q, 5..8 heads    3: fp32 Q, 5..8 heads
struct DecodeKernel {
  const void* fn;        // __global__ function
  const void* fn_fused;  // the same with the fused append (k_new != NULL)
  int threads;
  int smem_bytes;
  int tile;              // split lengths are rounded to a multiple of this
  int max_per_sm;        // CTAs per SM the kernel allows itself (0: no limit of its own)
  int stage_tokens;      // positions per stage of the balanced schedule (0: not supported)
  cudaError_t (*launch)(const DecodeArgs&, dim3 grid, cudaStream_t stream);
  cudaError_t (*launch_fused)(const DecodeArgs&, dim3 grid, cudaStream_t stream);
};

// Returns false if (D, bits, key groups, value groups, variant) has no instance
// (variant bits 0-1: query-head variant; bit 2: the paged layout's instances).
bool get_decode_kernel(int head_dim, int bits_k, int bits_v, int groups_k, int groups_v,
                       int variant, DecodeKernel* out);

// The tensor-memory decode kernel (head_dim 128, no fused append): false if
// (bits, key groups, value groups) has no instance.
bool get_decode_tc_kernel(int bits_k, int bits_v, int groups_k, int groups_v, int heads_per_cta,
                          DecodeKernel* out);

struct CombineArgs {
  const float* ws_o;
  const float* ws_lse;
  const int32_t* seq_lens;
  void* out;
  int out_dtype;
  int batch, q_heads, head_dim, capacity, max_seq_len, split_tokens, num_splits;
  // balanced schedule of the decode (stream_q > 0): its grid size, stage
  // length and unit layout, from which each row's count of partials follows
  int stream_q, stream_grid, stage_tokens, kv_heads, head_groups, gq, heads_per_cta;
};

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);

}  // namespace kvq
