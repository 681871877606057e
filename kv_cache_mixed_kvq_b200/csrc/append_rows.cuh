// Quantize-and-append of the step's new rows inside the decode kernel
// (kvq_append_decode_attention): the cache write of "Quantize What Counts:
// More for Keys, Less for Values" (summary page, "Problem statement" / "Key
// contributions": keys at b_k bits, values at b_v bits, group-wise scale and
// zero) done by the decode CTAs whose split holds the new positions, so that
// a decode step with an append is one launch.
//
// The path is cold (a few rows per CTA), so it favours few registers over
// speed: one warp per (position, K or V) row, lane l holding elements l,
// l + 32, ... of the row, a few rows' inputs loaded before any is quantized;
// shared memory holds one row's binary32 values (rotation) and D one-byte
// codes.  Per group of G elements, in binary32 with explicit
// round-to-nearest operations:
//   mn, mx = group min and max (a zero extreme stored as +0);
//   scale = (mx - mn) / (2^b - 1);  inv = 1 / scale;
//   code = clamp(rint((x - mn) * inv), 0, 2^b - 1), or 0 for a degenerate
//   group (scale 0, or scale or inv not finite);
//   stored (scale, zero) = (binary16(scale), binary16(mn)).
// Keys of a rotated cache are first replaced by H k, the unnormalised
// Walsh-Hadamard transform by the butterfly h = 1, 2, ..., D/2 (each step a
// binary32 add or subtract).  The codes are then placed by the format's
// formulas (K: slice (d mod 8)/2, word (d/8)/E, bit 16 (d mod 2) + b ((d/8)
// mod E); V: lane 4 (d mod 8) + (k mod 8)/2, word (k/8) W + (d/8)/E, bit
// 16 (k mod 2) + b ((d/8) mod E)), one 32-bit K word or one 16-bit V
// half-word per store, so positions outside the append keep their bytes.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace kvq {

__device__ __forceinline__ float load_input(const void* p, int dtype, size_t i) {
  if (dtype == KVQ_F32) return static_cast<const float*>(p)[i];
  const uint16_t h = static_cast<const uint16_t*>(p)[i];
  if (dtype == KVQ_BF16) return __uint_as_float(static_cast<uint32_t>(h) << 16);
  return __half2float(__ushort_as_half(h));
}

// Codes and parameters of one row (lane-strided elements x[i] = element
// lane + 32 i) into codes[] (shared, D bytes) and params[] (global, D/G
// words).
template <int D, int B, int G>
__device__ __forceinline__ void quantize_row_warp(const float (&x)[D / 32], uint8_t* codes,
                                                  uint32_t* params, int lane) {
  static_assert(G % 32 == 0 && D % G == 0, "groups of whole lane strides");
  constexpr int PER_G = G / 32;  // elements of a group per lane
  const float levels = static_cast<float>((1 << B) - 1);
#pragma unroll
  for (int g = 0; g < D / G; ++g) {
    float mn = x[g * PER_G], mx = x[g * PER_G];
#pragma unroll
    for (int i = 1; i < PER_G; ++i) {
      mn = fminf(mn, x[g * PER_G + i]);
      mx = fmaxf(mx, x[g * PER_G + i]);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    }
    mn = (mn == 0.0f) ? 0.0f : mn;
    mx = (mx == 0.0f) ? 0.0f : mx;
    const float scale = __fdiv_rn(__fsub_rn(mx, mn), levels);
    const float inv = __fdiv_rn(1.0f, scale);
    const bool degenerate = (scale == 0.0f) || !isfinite(scale) || !isfinite(inv);
#pragma unroll
    for (int i = 0; i < PER_G; ++i) {
      int c = 0;
      if (!degenerate) {
        c = static_cast<int>(rintf(__fmul_rn(__fsub_rn(x[g * PER_G + i], mn), inv)));
        c = min(max(c, 0), (1 << B) - 1);
      }
      codes[lane + 32 * (g * PER_G + i)] = static_cast<uint8_t>(c);
    }
    if (lane == 0) params[g] = pack_half2(__float2half_rn(scale), __float2half_rn(mn));
  }
  __syncwarp();
}

// Writes the new positions [p0, p1) of slot (b, hk) (input rows p - pos of
// k_new / v_new) into the cache.  Warp w takes rows r = w, w + kWarps, ...
// (row r: position p0 + r/2, keys for even r, values for odd r), loading
// APPEND_BATCH rows' inputs before quantizing any of them.  `stage`: this
// warp's 5 D bytes of shared memory.  `row_of(p)`: the position's row in the
// per-position arrays, or -1 when the block table names no page (the row is
// skipped and flagged).
template <class C, class RowOf>
__device__ __forceinline__ void append_rows(const DecodeArgs& a, int b, int hk, int pos, int p0,
                                         int p1, uint8_t* stage, RowOf row_of) {
  constexpr int D = C::D, PER = D / 32, NB = C::APPEND_BATCH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* f = reinterpret_cast<float*>(stage);
  uint8_t* codes = stage + 4 * D;
  // the cache arrays are the caller's writable memory (read-only elsewhere
  // in the decode kernel)
  uint8_t* k_codes = const_cast<uint8_t*>(a.k_codes);
  uint8_t* v_codes = const_cast<uint8_t*>(a.v_codes);
  uint32_t* k_params = const_cast<uint32_t*>(a.k_params);
  uint32_t* v_params = const_cast<uint32_t*>(a.v_params);
  const int n_rows = 2 * (p1 - p0);
  for (int r0 = warp; r0 < n_rows; r0 += C::kWarps * NB) {
    float x[NB][PER];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int r = r0 + C::kWarps * j;
      if (r >= n_rows) break;
      const int p = p0 + r / 2;
      const size_t in_row = (static_cast<size_t>(b) * a.kv_heads + hk) * a.n_new + (p - pos);
#pragma unroll
      for (int i = 0; i < PER; ++i)
        x[j][i] = load_input((r & 1) ? a.v_new : a.k_new, a.in_dtype, in_row * D + lane + 32 * i);
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int r = r0 + C::kWarps * j;
      if (r >= n_rows) break;
      const int p = p0 + r / 2;
      const bool is_v = (r & 1) != 0;
      const long long row = row_of(p);
      if (row < 0) {
        if (lane == 0) flag_error(a.err, KVQ_DEVERR_BAD_PAGE);
        continue;
      }
      if (!is_v && a.rotate_q) {
        // keys of a rotated cache: H k by the butterfly, in shared memory
#pragma unroll
        for (int i = 0; i < PER; ++i) f[lane + 32 * i] = x[j][i];
        __syncwarp();
        for (int h = 1; h < D; h <<= 1) {
          for (int t = lane; t < D / 2; t += 32) {
            const int i0 = (t / h) * 2 * h + (t % h);
            const float u = f[i0], w = f[i0 + h];
            f[i0] = __fadd_rn(u, w);
            f[i0 + h] = __fsub_rn(u, w);
          }
          __syncwarp();
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) x[j][i] = f[lane + 32 * i];
        __syncwarp();
      }
      const size_t rw = static_cast<size_t>(row);
      if (!is_v) {
        constexpr int B = C::BK, E = 16 / B, WPS = C::KSLICE / 4;
        quantize_row_warp<D, B, C::GK>(x[j], codes, k_params + rw * C::NGK, lane);
        for (int q = lane; q < C::KROW / 4; q += 32) {
          const int c = q / WPS, w = q % WPS;
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < E; ++e)
#pragma unroll
            for (int lo = 0; lo < 2; ++lo)
              word |= static_cast<uint32_t>(codes[8 * (w * E + e) + 2 * c + lo])
                      << (16 * lo + B * e);
          *reinterpret_cast<uint32_t*>(k_codes + rw * C::KROW + 4 * q) = word;
        }
      } else {
        constexpr int B = C::BV, E = 16 / B, W = C::WV, PC = C::VP;
        quantize_row_warp<D, B, C::GV>(x[j], codes, v_params + rw * C::NGV, lane);
        const int k = static_cast<int>(rw % 16);  // position inside its 16-position tile
        uint8_t* tile = v_codes + (rw / 16) * C::VTILE;
        for (int hw = lane; hw < 8 * W; hw += 32) {
          const int m = hw % 8, wq = hw / 8;
          uint32_t half = 0;
#pragma unroll
          for (int e = 0; e < E; ++e)
            half |= static_cast<uint32_t>(codes[8 * (wq * E + e) + m]) << (B * e);
          const int L = 4 * m + (k % 8) / 2;
          const int n = 4 * ((k / 8) * W + wq) + 2 * (k % 2);
          *reinterpret_cast<uint16_t*>(tile + (n / PC) * 32 * PC + L * PC + (n % PC)) =
              static_cast<uint16_t>(half);
        }
      }
      __syncwarp();  // the stage is reused by this warp's next row
    }
  }
}

}  // namespace kvq
