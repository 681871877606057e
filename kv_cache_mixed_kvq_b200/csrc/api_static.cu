// Decode attention for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: engines that plan every byte of
// device memory at start-up and forbid allocation on the request path
// (cudaMalloc can synchronize the device and can fail when memory is
// fragmented), and plain-C hosts that have no device allocator of their own.
// For them, kvq_decode_attention_static() takes its split-K scratch from a
// fixed array that lives in this library's device image (allocated by the
// CUDA runtime when the library's module is loaded on a device, held until
// the process exits) instead of a caller-provided workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "kvq.h"

// The scratch array.  In host code this name is only a host-side stand-in for
// the symbol, not a device address: host code must obtain the address with
// cudaGetSymbolAddress (below) and pass that to the kernels.
static __device__ __align__(256) unsigned char g_kvq_static_scratch[KVQ_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// Device address of the scratch array on the current device, looked up with
// that device current.  A successful lookup is kept for the rest of the
// process; a failed one returns KVQ_ERR_CUDA and is retried on the next call.
int static_scratch(void** out) {
  static std::mutex mu;
  static void* ptrs[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kvq_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attention_static(const kvq_cache_desc* cache, const void* q,
                                           int32_t q_dtype, int32_t num_q_heads,
                                           const int32_t* seq_lens, int32_t max_seq_len,
                                           float sm_scale, void* out, int32_t out_dtype,
                                           kvq_stream_t stream) {
  // Split-K partials for this shape; 0 also for invalid arguments, which the
  // regular entry point below reports with its own status.
  const size_t need = kvq_decode_workspace_bytes(cache, num_q_heads, max_seq_len);
  if (need > KVQ_STATIC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = static_scratch(&scratch);
  if (st != KVQ_OK) return st;
  // Every partial result that the combine step reads is written first by the
  // decode kernel of the same call, so the scratch needs no clearing.
  return kvq_decode_attention(cache, q, q_dtype, num_q_heads, seq_lens, max_seq_len, sm_scale,
                              out, out_dtype, scratch, KVQ_STATIC_SCRATCH_BYTES, stream);
}
