// Log-sum-exp combine of split-K partial results.
//
// Each split s of batch row b, query head hq holds a normalised partial
// output O_s and its log2-domain log-sum-exp lse_s; the full softmax output is
//   o = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L),   L = max_s lse_s.
// One warp per (batch row, query head); each lane owns D/32 elements.
#include "common.cuh"
#include "internal.h"

namespace kvq {
namespace {

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const CombineArgs a) {
  constexpr int PER = D / 32;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.batch * a.q_heads) return;
  const int b = row / a.q_heads;
  int len = a.seq_lens[b];
  len = max(0, min(len, min(a.max_seq_len, a.capacity)));
  const int ns = (len + a.split_tokens - 1) / a.split_tokens;
  const size_t base = static_cast<size_t>(row) * a.num_splits;

  // weights 2^(lse_s - L): lanes load the log-sum-exps of 32 splits at a
  // time in parallel; the partial outputs are then read with the loads of
  // several splits in flight.
  float L = -INFINITY;
  for (int s = lane; s < ns; s += 32) L = fmaxf(L, a.ws_lse[base + s]);
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) L = fmaxf(L, __shfl_xor_sync(0xffffffffu, L, m));

  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.0f;
  float den = 0.0f;
  for (int s0 = 0; s0 < ns; s0 += 32) {
    const int cnt = min(32, ns - s0);
    const float wl = lane < cnt ? exp2_approx(a.ws_lse[base + s0 + lane] - L) : 0.0f;
    constexpr int U = 4;
    for (int s = 0; s < cnt; s += U) {
      float w[U];
      float v[U][PER];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        w[u] = __shfl_sync(0xffffffffu, wl, (s + u) & 31);
        const int si = s0 + min(s + u, cnt - 1);
        const float* o = a.ws_o + (base + si) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 t = *reinterpret_cast<const float4*>(o);
          v[u][0] = t.x; v[u][1] = t.y; v[u][2] = t.z; v[u][3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(o);
          v[u][0] = t.x; v[u][1] = t.y;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (s + u >= cnt) break;
        den += w[u];
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] = fmaf(w[u], v[u][i], acc[i]);
      }
    }
  }
  const float inv = ns > 0 ? 1.0f / den : 0.0f;
  const size_t out = static_cast<size_t>(row) * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const float v = ns > 0 ? acc[i] * inv : 0.0f;
    if (a.out_dtype == KVQ_F32)
      reinterpret_cast<float*>(a.out)[out + i] = v;
    else if (a.out_dtype == KVQ_BF16)
      reinterpret_cast<__nv_bfloat16*>(a.out)[out + i] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<__half*>(a.out)[out + i] = __float2half_rn(v);
  }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  const int rows = a.batch * a.q_heads;
  const dim3 grid((rows + 3) / 4);
  if (a.head_dim == 64)
    combine_kernel<64><<<grid, 128, 0, stream>>>(a);
  else
    combine_kernel<128><<<grid, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
