// Log-sum-exp combine of split-K partial results.
//
// Each split s of batch row b, query head hq holds a normalised partial
// output O_s and its log2-domain log-sum-exp lse_s; the full softmax output is
//   o = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L),   L = max_s lse_s.
// One CTA of four warps per (batch row, query head); the warps take every
// fourth split, each lane owns D/32 elements, and the warps' results are
// merged through shared memory.  With the decode's balanced schedule the
// partials of a row are those of the CTAs that covered its unit.
#include "common.cuh"
#include "internal.h"

namespace kvq {
namespace {

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const CombineArgs a) {
  constexpr int PER = D / 32;  // output elements per lane
  constexpr int U = 8;         // partial outputs in flight per lane
  __shared__ float s_acc[4][D];
  __shared__ float s_m[4], s_den[4];
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = row / a.q_heads;
  const int lim = min(a.max_seq_len, a.capacity);
  int ns;  // partial results of this row
  if (a.stream_q > 0) {
    // balanced schedule: the CTAs that covered this row's unit, from the same
    // prefix sums as the decode kernel (built from the lengths alone, before
    // the wait for the decode grid); a unit one CTA covered whole was written
    // by it directly
    __shared__ int s_off[kStreamRows + 1];
    __shared__ int s_w[4];
    const int units = a.kv_heads * a.head_groups;  // per row
    stream_row_offsets(a.seq_lens, a.batch, lim, units, a.stage_tokens, s_off, nullptr, s_w);
    pdl_wait();
    pdl_trigger();
    const int S = s_off[kStreamRows];
    const int Q = max(a.stream_q, (S + a.stream_grid - 1) / a.stream_grid);
    const int hq = row % a.q_heads;
    const int u = (hq / a.gq) * a.head_groups + (hq % a.gq) / a.heads_per_cta;
    const int nsu = (s_off[b + 1] - s_off[b]) / units;
    ns = 0;
    if (nsu > 0) {
      const int ubase = s_off[b] + u * nsu;
      ns = (ubase + nsu - 1) / Q - ubase / Q + 1;
      if (ns == 1) return;
    }
  } else {
    // (the lengths are read before the wait: no kernel of this library
    // writes them)
    const int len = max(0, min(a.seq_lens[b], lim));
    ns = (len + a.split_tokens - 1) / a.split_tokens;
    pdl_wait();
    pdl_trigger();
  }
  const size_t base = static_cast<size_t>(row) * a.num_splits;

  // Warp w merges splits w, w+4, w+8, ... with its own running maximum M;
  // lanes load 32 of its log-sum-exps at a time; the partial outputs of U
  // splits at a time are all requested before any is used (the first U
  // together with the log-sum-exps).
  float M = -INFINITY, den = 0.0f;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.0f;
  const int mine = ns > warp ? (ns - warp + 3) / 4 : 0;  // splits of this warp
  for (int c0 = 0; c0 < mine; c0 += 32) {
    const int cnt = min(32, mine - c0);
    float v[U][PER];
    auto load = [&](int s) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int si = warp + 4 * (c0 + min(s + u, cnt - 1));
        const float* o = a.ws_o + (base + si) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 t = *reinterpret_cast<const float4*>(o);
          v[u][0] = t.x; v[u][1] = t.y; v[u][2] = t.z; v[u][3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(o);
          v[u][0] = t.x; v[u][1] = t.y;
        }
      }
    };
    load(0);
    const float lse = lane < cnt ? a.ws_lse[base + warp + 4 * (c0 + lane)] : -INFINITY;
    float cm = lse;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, m));
    const float Mn = fmaxf(M, cm);
    const float r = exp2_approx(M - Mn);  // M = -inf on the first chunk: r = 0
    den *= r;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] *= r;
    M = Mn;
    const float wl = lane < cnt ? exp2_approx(lse - M) : 0.0f;
    for (int s = 0; s < cnt; s += U) {
      if (s > 0) load(s);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float w = __shfl_sync(0xffffffffu, wl, (s + u) & 31);
        if (s + u < cnt) {
          den += w;
#pragma unroll
          for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, v[u][i], acc[i]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) s_acc[warp][lane * PER + i] = acc[i];
  if (lane == 0) {
    s_m[warp] = M;
    s_den[warp] = den;
  }
  __syncthreads();

  // Merge the four warps' results: weights 2^(M_w - max M).
  if (threadIdx.x >= D) return;
  const int d = threadIdx.x;
  const float Mx = fmaxf(fmaxf(s_m[0], s_m[1]), fmaxf(s_m[2], s_m[3]));
  float num = 0.0f, dd = 0.0f;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float f = s_den[w] > 0.0f ? exp2_approx(s_m[w] - Mx) : 0.0f;
    num = fmaf(f, s_acc[w][d], num);
    dd = fmaf(f, s_den[w], dd);
  }
  const float val = ns > 0 ? num / dd : 0.0f;
  const size_t out = static_cast<size_t>(row) * D + d;
  if (a.out_dtype == KVQ_F32)
    reinterpret_cast<float*>(a.out)[out] = val;
  else if (a.out_dtype == KVQ_BF16)
    reinterpret_cast<__nv_bfloat16*>(a.out)[out] = __float2bfloat16_rn(val);
  else
    reinterpret_cast<__half*>(a.out)[out] = __float2half_rn(val);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  const dim3 grid(a.batch * a.q_heads);
  if (a.head_dim == 64) return launch_pdl(combine_kernel<64>, grid, dim3(128), 0, stream, a);
  return launch_pdl(combine_kernel<128>, grid, dim3(128), 0, stream, a);
}

}  // namespace kvq
