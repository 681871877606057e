// Quantize-and-append kernel: group-wise asymmetric min-max quantization of
// new K/V rows into the packed cache ("Quantize What Counts: More for Keys,
// Less for Values", summary page, "Problem statement" / "Key contributions":
// keys at b_k bits, values at b_v bits; "Results", "Group-size sensitivity":
// one scale/zero per group of head_dim elements).
//
// One CTA handles one 16-position tile of one (batch row, kv head) slot:
// 16 tokens x D/8 threads, each thread owning 8 consecutive elements of one
// token.  Loads are 16-byte vectors; the group min/max is a butterfly of warp
// shuffles over the D/8-thread token; codes are merged into the packed words
// with shuffles as well.  A V tile that the append covers completely is
// assembled in shared memory and written with 16-byte stores; a tile at the
// edge of the appended range is written half-word by half-word so that the
// other positions' bits stay untouched.
#include "common.cuh"
#include "internal.h"

namespace kvq {
namespace {

// Group quantizer on 8 elements of this thread; the group spans G/8
// consecutive threads.  Every step is IEEE binary32 with explicit rounding
// intrinsics (no contraction), so the codes equal those of a sequential
// evaluation of the same formula.
__device__ __forceinline__ uint32_t quantize8(const float x[8], int bits, int group,
                                              uint32_t codes[8]) {
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
  }
  for (int m = 1; m < group / 8; m <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  }
  // a zero extreme is stored as +0 whatever its sign
  mn = (mn == 0.0f) ? 0.0f : mn;
  mx = (mx == 0.0f) ? 0.0f : mx;
  const float levels = static_cast<float>((1 << bits) - 1);
  const float range = __fsub_rn(mx, mn);
  const float scale = __fdiv_rn(range, levels);
  const float inv = __fdiv_rn(1.0f, scale);
  const bool degenerate = (scale == 0.0f) || !isfinite(scale) || !isfinite(inv);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float t = __fmul_rn(__fsub_rn(x[i], mn), inv);
    const float r = fminf(fmaxf(rintf(t), 0.0f), levels);
    codes[i] = degenerate ? 0u : static_cast<uint32_t>(r);
  }
  return pack_half2(__float2half_rn(scale), __float2half_rn(mn));
}

__device__ __forceinline__ uint32_t or_over_lanes(uint32_t v, int width) {
  for (int m = 1; m < width; m <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

template <int D, typename TIn>
__global__ void __launch_bounds__(2 * D) quantize_append_kernel(QuantizeArgs a) {
  constexpr int LPT = D / 8;  // threads per token
  __shared__ __align__(16) uint8_t vtile[2 * D * 8];

  const int tid = threadIdx.x;
  const int k = tid / LPT;  // position within the tile
  const int l = tid % LPT;  // elements 8l .. 8l+7
  const int b = blockIdx.z;
  const int h = blockIdx.y;
  const int pos = a.pos[b];
  if (pos < 0 || static_cast<long long>(pos) + a.n_new > a.capacity) {
    if (blockIdx.x == 0 && h == 0 && tid == 0)
      flag_error(a.err, pos < 0 ? KVQ_DEVERR_BAD_POS : KVQ_DEVERR_CAPACITY);
    return;
  }
  const int tile = pos / 16 + static_cast<int>(blockIdx.x);
  const int end = pos + a.n_new;
  if (tile * 16 >= end) return;
  const int p = tile * 16 + k;
  const bool valid = p >= pos && p < end;
  const bool full_tile = tile * 16 >= pos && tile * 16 + 16 <= end;

  const size_t slot = static_cast<size_t>(b) * a.kv_heads + h;
  const size_t src = (slot * a.n_new + (valid ? p - pos : 0)) * D + 8 * l;
  float x[2][8];
  if (valid) {
    Load8<TIn>::run(reinterpret_cast<const TIn*>(a.k) + src, x[0]);
    Load8<TIn>::run(reinterpret_cast<const TIn*>(a.v) + src, x[1]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[0][i] = x[1][i] = 0.0f;
  }

  const int ng = D / a.group;
  const int lanes_per_group = a.group / 8;

  // ---------------------------------------------------------------- keys
  {
    const int bits = a.bits_k;
    uint32_t codes[8];
    const uint32_t param = quantize8(x[0], bits, a.group, codes);
    const int E = 16 / bits;
    const int e = l % E, w = l / E;
    uint32_t part[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      part[c] = or_over_lanes((codes[2 * c] << (e * bits)) | (codes[2 * c + 1] << (16 + e * bits)),
                              E);
    if (valid) {
      const int slice = D * bits / 32;
      uint8_t* row = a.k_codes + (slot * a.capacity + p) * (D * bits / 8);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if ((c & (E - 1)) == e) *reinterpret_cast<uint32_t*>(row + c * slice + 4 * w) = part[c];
      if (l % lanes_per_group == 0)
        a.k_params[(slot * a.capacity + p) * ng + l / lanes_per_group] = param;
    }
  }

  // -------------------------------------------------------------- values
  {
    const int bits = a.bits_v;
    uint32_t codes[8];
    const uint32_t param = quantize8(x[1], bits, a.group, codes);
    const int E = 16 / bits;
    const int e = l % E, w = l / E;
    const int W = D * bits / 128;
    const int N = D * bits / 16;
    const int P = N < 16 ? N : 16;
    const int q = (k / 8) * W + w;
    const int n = 4 * q + 2 * (k % 2);  // byte of this position's half-word in the lane
    uint32_t half[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) half[r] = or_over_lanes(codes[r] << (e * bits), E);
    const size_t tile_bytes = 2 * D * bits;
    uint8_t* gtile = a.v_codes + slot * (a.capacity / 16) * tile_bytes + tile * tile_bytes;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if ((r & (E - 1)) != e) continue;
      const int lane = 4 * r + (k % 8) / 2;
      const int off = (n / P) * 32 * P + lane * P + (n % P);
      const uint16_t val = static_cast<uint16_t>(half[r]);
      if (full_tile)
        *reinterpret_cast<uint16_t*>(vtile + off) = val;
      else if (valid)
        *reinterpret_cast<uint16_t*>(gtile + off) = val;
    }
    if (valid && l % lanes_per_group == 0)
      a.v_params[(slot * a.capacity + p) * ng + l / lanes_per_group] = param;
    if (full_tile) {
      __syncthreads();
      for (int i = tid; i < static_cast<int>(tile_bytes / 16); i += blockDim.x)
        reinterpret_cast<uint4*>(gtile)[i] = reinterpret_cast<const uint4*>(vtile)[i];
    }
  }
}

template <int D, typename TIn>
cudaError_t launch_typed(const QuantizeArgs& a, cudaStream_t stream) {
  const dim3 grid((a.n_new + 30) / 16, a.kv_heads, a.batch);
  quantize_append_kernel<D, TIn><<<grid, 2 * D, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dim(const QuantizeArgs& a, cudaStream_t stream) {
  switch (a.in_dtype) {
    case KVQ_F32: return launch_typed<D, float>(a, stream);
    case KVQ_BF16: return launch_typed<D, __nv_bfloat16>(a, stream);
    default: return launch_typed<D, __half>(a, stream);
  }
}

}  // namespace

cudaError_t launch_quantize_append(const QuantizeArgs& a, cudaStream_t stream) {
  return a.head_dim == 64 ? launch_dim<64>(a, stream) : launch_dim<128>(a, stream);
}

}  // namespace kvq
