// Split-K flash-decoding over the packed mixed-precision cache.
//
// One decode step of attention ("Quantize What Counts: More for Keys, Less
// for Values", summary page, "Problem statement": the quantized KV cache is
// what inference reads) for one (split of the tokens, kv head, batch row):
//
//   s_t = sm_scale * q . k^_t,  k^ = code * scale + zero   (per group)
//   o   = sum_t softmax(s)_t v^_t
//
// Design (B200, sm_100a):
//  * a producer warp streams 64-token stages of the four cache arrays into
//    shared memory with 1-D bulk copies (cp.async.bulk, no multicast) on an
//    mbarrier ring; four consumer warps each take one 16-token tile;
//  * codes stay integers: every code becomes an exact binary16 subnormal
//    (code * 2^(pos-24)) with one AND, so tensor cores (mma.sync m16n8k16,
//    fp32 accumulate) multiply raw codes; the per-group scale and zero are
//    applied afterwards:  q.k^ = sum_g scale_g (q . c_g) + zero_g sum_{d in g} q_d
//    and  o = sum_t (p_t scale_t) c_t + sum_t p_t zero_t;
//  * the query (B operand of the score product) is scaled by a power of two
//    and, for binary32 queries, split into binary16 high and low parts in two
//    columns; the weights p_t * scale_t (B operand of the output product) are
//    always split into high and low parts, so products keep ~22 bits;
//  * online softmax in binary32 (exp2 domain), partial results per split are
//    merged by a separate log-sum-exp combine kernel.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace kvq {

template <int D_, int BK_, int BV_, int NG_, int QS_, int NQ_, int NP_>
struct DecodeCfg {
  static constexpr int D = D_, BK = BK_, BV = BV_, NG = NG_, QS = QS_, NQ = NQ_, NP = NP_;
  static constexpr int kWarps = 4;  // consumer warps
  static constexpr int kThreads = 32 * (kWarps + 1);
  static constexpr int kStageTokens = 16 * kWarps;
  static constexpr int kStages = 4;
  static constexpr int G = D / NG;
  static constexpr int KSTEPS = D / 16;  // k-steps (scores) == m-tiles (output)
  static constexpr int KROW = D * BK / 8;
  static constexpr int KSLICE = D * BK / 32;  // bytes of one lane's K slice
  static constexpr int KW = KSLICE / 4;
  static constexpr int VTILE = 2 * D * BV;
  static constexpr int VN = D * BV / 16;  // bytes per lane per V tile
  static constexpr int VP = VN < 16 ? VN : 16;
  static constexpr int VW = VN / 4;
  static constexpr int WV = D * BV / 128;  // V words per half-lane
  static constexpr int PROW = NG * 4;
  static constexpr int STAGE_K = kStageTokens * KROW;
  static constexpr int STAGE_V = kWarps * VTILE;
  static constexpr int STAGE_P = kStageTokens * PROW;
  static constexpr int STAGE_BYTES = STAGE_K + STAGE_V + 2 * STAGE_P;
  static constexpr int RING_BYTES = kStages * STAGE_BYTES;
  static constexpr int PEX_FLOATS = kWarps * 16 * 8;
  static constexpr int ALPHA_FLOATS = kWarps * 8;
  static constexpr int SMEM_BYTES = RING_BYTES + 4 * (PEX_FLOATS + ALPHA_FLOATS) + 16 * kStages;
  static constexpr int HT = QS == 1 ? 2 * NQ : NQ;  // score head slots per thread
  static_assert(RING_BYTES >= kWarps * 8 * D * 4, "merge buffer must fit in the ring");
  static_assert(STAGE_BYTES % 16 == 0 && STAGE_K % 16 == 0 && STAGE_V % 16 == 0, "alignment");
  static_assert(G >= 16 && G % 16 == 0, "group must cover whole 16-element steps");
};

// Bit position and pre-shift of extraction e for b-bit fields: fields that
// would reach the binary16 exponent are shifted down by 8 first.
template <int B>
__device__ __forceinline__ constexpr int field_shift(int e) { return (e * B >= 8) ? 8 : 0; }
template <int B>
__device__ __forceinline__ constexpr int field_pos(int e) { return e * B - field_shift<B>(e); }

// Register i of a lane's packed words: two codes (low and high half-word) as
// binary16 subnormals code * 2^(field_pos - 24).
template <int B, int NW>
__device__ __forceinline__ uint32_t extract_codes(const uint32_t (&w)[NW], int base_word, int i) {
  constexpr int E = 16 / B;
  const int word = base_word + i / E;
  const int e = i % E;
  const uint32_t m = ((1u << B) - 1u) << field_pos<B>(e);
  return (w[word] >> field_shift<B>(e)) & (m | (m << 16));
}

template <int BYTES, int NW>
__device__ __forceinline__ void lds_words(const uint8_t* p, uint32_t (&w)[NW], int first) {
  if constexpr (BYTES % 16 == 0) {
#pragma unroll
    for (int i = 0; i < BYTES / 16; ++i) {
      const uint4 u = *reinterpret_cast<const uint4*>(p + 16 * i);
      w[first + 4 * i] = u.x;
      w[first + 4 * i + 1] = u.y;
      w[first + 4 * i + 2] = u.z;
      w[first + 4 * i + 3] = u.w;
    }
  } else if constexpr (BYTES == 8) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    w[first] = u.x;
    w[first + 1] = u.y;
  } else {
    static_assert(BYTES == 4, "slice size");
    w[first] = *reinterpret_cast<const uint32_t*>(p);
  }
}

__device__ __forceinline__ float warp_max_xor(float v, int lo_mask) {
  for (int m = lo_mask; m < 32; m <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

template <class C>
__global__ void __launch_bounds__(C::kThreads) decode_kernel(const DecodeArgs a) {
  constexpr int D = C::D, NG = C::NG, NQ = C::NQ, NP = C::NP, QS = C::QS, HT = C::HT;
  constexpr int KSTEPS = C::KSTEPS, G = C::G;
  extern __shared__ __align__(128) uint8_t smem[];
  float* pex = reinterpret_cast<float*>(smem + C::RING_BYTES);  // [warp][16 tokens][8 heads]
  float* alph = pex + C::PEX_FLOATS;                            // [warp][8 heads]
  uint64_t* full = reinterpret_cast<uint64_t*>(alph + C::ALPHA_FLOATS);
  uint64_t* empty = full + C::kStages;

  const int split = blockIdx.x;
  const int hk = blockIdx.y / a.head_groups;
  const int hg = blockIdx.y % a.head_groups;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int len = a.seq_lens[b];
  const int lim = min(a.max_seq_len, a.capacity);
  if (len < 0 || len > lim) {
    if (split == 0 && blockIdx.y == 0 && threadIdx.x == 0) flag_error(a.err, KVQ_DEVERR_SEQ_LEN);
    len = max(0, min(len, lim));
  }
  const int t0 = split * a.split_tokens;
  if (t0 >= len) return;
  const int t1 = min(t0 + a.split_tokens, len);
  const int n_iters = (t1 - t0 + C::kStageTokens - 1) / C::kStageTokens;
  const int head0 = hk * a.gq + hg * a.heads_per_cta;
  const int nh = min(a.heads_per_cta, a.gq - hg * a.heads_per_cta);
  const size_t slot = static_cast<size_t>(b) * a.kv_heads + hk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == C::kWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint8_t* kb = a.k_codes + slot * a.capacity * C::KROW;
      const uint8_t* vb = a.v_codes + slot * (a.capacity / 16) * C::VTILE;
      const uint8_t* kpb = reinterpret_cast<const uint8_t*>(a.k_params) + slot * a.capacity * C::PROW;
      const uint8_t* vpb = reinterpret_cast<const uint8_t*>(a.v_params) + slot * a.capacity * C::PROW;
      int issued = 0;
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % C::kStages;
        if (it >= C::kStages && !mbar_wait_bounded(&empty[s], ((it / C::kStages) + 1) & 1, a.err))
          break;
        const int tb = t0 + it * C::kStageTokens;
        const int n16 = (min(C::kStageTokens, t1 - tb) + 15) & ~15;
        uint8_t* st = smem + s * C::STAGE_BYTES;
        const uint32_t kbytes = n16 * C::KROW, vbytes = (n16 / 16) * C::VTILE,
                       pbytes = n16 * C::PROW;
        mbar_arrive_expect_tx(&full[s], kbytes + vbytes + 2 * pbytes);
        bulk_copy_g2s(st, kb + static_cast<size_t>(tb) * C::KROW, kbytes, &full[s]);
        bulk_copy_g2s(st + C::STAGE_K, vb + static_cast<size_t>(tb / 16) * C::VTILE, vbytes,
                      &full[s]);
        bulk_copy_g2s(st + C::STAGE_K + C::STAGE_V, kpb + static_cast<size_t>(tb) * C::PROW,
                      pbytes, &full[s]);
        bulk_copy_g2s(st + C::STAGE_K + C::STAGE_V + C::STAGE_P,
                      vpb + static_cast<size_t>(tb) * C::PROW, pbytes, &full[s]);
        ++issued;
      }
      // Drain: every copy issued must have landed before shared memory is
      // reused below (normally already true; bounded in any case).
      for (int it = max(0, issued - C::kStages); it < issued; ++it)
        mbar_wait_bounded(&full[it % C::kStages], (it / C::kStages) & 1, a.err);
    }
  }

  // ------------------------------------------------------------ consumers
  const int g = lane >> 2, c = lane & 3;
  float m_run[HT], l_run[HT];
  float oacc[KSTEPS][NP][4];
  float zacc[NP][NG];
  // Power-of-two exponent applied to the output weights p * scale_v so that
  // their binary16 parts stay normal; only ever decreases (see below).
  int u_run = 100;
#pragma unroll
  for (int hs = 0; hs < HT; ++hs) {
    m_run[hs] = -INFINITY;
    l_run[hs] = 0.0f;
  }
#pragma unroll
  for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
    for (int pt = 0; pt < NP; ++pt)
#pragma unroll
      for (int r = 0; r < 4; ++r) oacc[j][pt][r] = 0.0f;
#pragma unroll
  for (int pt = 0; pt < NP; ++pt)
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) zacc[pt][gr] = 0.0f;

  if (warp < C::kWarps) {
    // -------- query fragments (B operand of the score product), once per CTA
    float qraw[NQ][KSTEPS][4];
    float amax = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NQ; ++nt) {
      const int n = 8 * nt + g;
      const int head = QS == 2 ? n / 2 : n;
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int d = 16 * j + 2 * c + (r & 1) + 8 * (r >> 1);
          float v = 0.0f;
          if (head < nh)
            v = load_elem(a.q, a.q_dtype,
                          (static_cast<size_t>(b) * a.q_heads + head0 + head) * D + d);
          qraw[nt][j][r] = v;
          amax = fmaxf(amax, fabsf(v));
        }
    }
    amax = warp_max_xor(amax, 1);
    const int eq = amax > 0.0f ? max(-100, min(100, 14 - ilogbf(amax))) : 0;
    uint32_t bq[NQ][KSTEPS][2];
#pragma unroll
    for (int nt = 0; nt < NQ; ++nt) {
      const int part = QS == 2 ? (g & 1) : 0;
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int e = (2 * j + r) % (16 / C::BK);
          __half hv[2];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const float v = ldexpf(qraw[nt][j][2 * r + h2], eq - field_pos<C::BK>(e));
            const __half hi = __float2half_rn(v);
            hv[h2] = part ? __float2half_rn(v - __half2float(hi)) : hi;
          }
          bq[nt][j][r] = pack_half2(hv[0], hv[1]);
        }
    }
    // sum of q over each group, in the same units as the code products:
    // the score product of an all-ones code matrix.
    float qsum[NG][NQ][4];
#pragma unroll
    for (int gr = 0; gr < NG; ++gr)
#pragma unroll
      for (int nt = 0; nt < NQ; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) qsum[gr][nt][r] = 0.0f;
#pragma unroll
    for (int j = 0; j < KSTEPS; ++j) {
      const int gr = 16 * j / G;
      const uint32_t one0 = 0x00010001u << field_pos<C::BK>((2 * j) % (16 / C::BK));
      const uint32_t one1 = 0x00010001u << field_pos<C::BK>((2 * j + 1) % (16 / C::BK));
#pragma unroll
      for (int nt = 0; nt < NQ; ++nt)
        mma_f16_16816(qsum[gr][nt], one0, one0, one1, one1, bq[nt][j][0], bq[nt][j][1]);
    }
    const float F = ldexpf(a.sm_scale_log2, 24 - eq);

    // ------------------------------------------------------ main loop
    float* wpex = pex + warp * 128;
    float* walph = alph + warp * 8;
    for (int it = 0; it < n_iters; ++it) {
      const int s = it % C::kStages;
      if (!mbar_wait_bounded(&full[s], (it / C::kStages) & 1, a.err)) break;
      const int tb = t0 + it * C::kStageTokens + 16 * warp;
      if (tb < t1) {
        const int nvalid = t1 - tb;
        const uint8_t* st = smem + s * C::STAGE_BYTES;
        const uint8_t* kt = st + warp * 16 * C::KROW;
        const uint8_t* vt = st + C::STAGE_K + warp * C::VTILE;
        const uint32_t* kp =
            reinterpret_cast<const uint32_t*>(st + C::STAGE_K + C::STAGE_V) + warp * 16 * NG;
        const uint32_t* vp =
            reinterpret_cast<const uint32_t*>(st + C::STAGE_K + C::STAGE_V + C::STAGE_P) +
            warp * 16 * NG;

        // ---- scores: S^T[token][head] = codes . q'
        uint32_t kw[2 * C::KW];
        lds_words<C::KSLICE>(kt + g * C::KROW + c * C::KSLICE, kw, 0);
        lds_words<C::KSLICE>(kt + (g + 8) * C::KROW + c * C::KSLICE, kw, C::KW);
        float acc[NG][NQ][4];
#pragma unroll
        for (int gr = 0; gr < NG; ++gr)
#pragma unroll
          for (int nt = 0; nt < NQ; ++nt)
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[gr][nt][r] = 0.0f;
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j) {
          const int gr = 16 * j / G;
          const uint32_t a0 = extract_codes<C::BK>(kw, 0, 2 * j);
          const uint32_t a1 = extract_codes<C::BK>(kw, C::KW, 2 * j);
          const uint32_t a2 = extract_codes<C::BK>(kw, 0, 2 * j + 1);
          const uint32_t a3 = extract_codes<C::BK>(kw, C::KW, 2 * j + 1);
#pragma unroll
          for (int nt = 0; nt < NQ; ++nt)
            mma_f16_16816(acc[gr][nt], a0, a1, a2, a3, bq[nt][j][0], bq[nt][j][1]);
        }
        float sc[HT][2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int row = g + 8 * rr;
          float ks[NG], kz[NG];
#pragma unroll
          for (int gr = 0; gr < NG; ++gr) {
            const float2 f = unpack_half2(kp[row * NG + gr]);
            ks[gr] = f.x;
            kz[gr] = f.y;
          }
#pragma unroll
          for (int nt = 0; nt < NQ; ++nt) {
            float v[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float t = 0.0f;
#pragma unroll
              for (int gr = 0; gr < NG; ++gr)
                t = fmaf(ks[gr], acc[gr][nt][2 * rr + e], fmaf(kz[gr], qsum[gr][nt][2 * rr + e], t));
              v[e] = t;
            }
            const bool ok = row < nvalid;
            if (QS == 2) {
              sc[nt][rr] = ok ? (v[0] + v[1]) * F : -INFINITY;
            } else {
              sc[2 * nt][rr] = ok ? v[0] * F : -INFINITY;
              sc[2 * nt + 1][rr] = ok ? v[1] * F : -INFINITY;
            }
          }
        }

        // ---- online softmax (exp2 domain)
        bool changed = false;
#pragma unroll
        for (int hs = 0; hs < HT; ++hs) {
          const int head = QS == 2 ? 4 * hs + c : 8 * (hs / 2) + 2 * c + (hs & 1);
          const float mt = warp_max_xor(fmaxf(sc[hs][0], sc[hs][1]), 4);
          const float mnew = fmaxf(m_run[hs], mt);
          changed |= mnew > m_run[hs];
          const float alpha = mnew == -INFINITY ? 1.0f : exp2f(m_run[hs] - mnew);
          const float mref = mnew == -INFINITY ? 0.0f : mnew;
          const float p0 = exp2f(sc[hs][0] - mref);
          const float p1 = exp2f(sc[hs][1] - mref);
          l_run[hs] = fmaf(l_run[hs], alpha, p0 + p1);
          m_run[hs] = mnew;
          wpex[g * 8 + head] = p0;
          wpex[(g + 8) * 8 + head] = p1;
          if (g == 0) walph[head] = alpha;
        }
        __syncwarp();
        changed = __any_sync(0xffffffffu, changed);

        // ---- weights p * scale_v as binary16 high/low parts (B operand).
        // They are scaled by 2^u_run with u_run chosen from the largest value
        // scale in the tile (p <= 1), so that the largest weight stays below
        // 2^15 and the low part of every weight that matters stays a normal
        // binary16.  When a tile needs a smaller exponent, the output
        // accumulators are rescaled by the (exact) power of two.
        const int kk[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
        float2 svz[4][NG];
        float smax = 0.0f;
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int gr = 0; gr < NG; ++gr) {
            svz[x][gr] = unpack_half2(vp[kk[x] * NG + gr]);
            if (kk[x] < nvalid) smax = fmaxf(smax, svz[x][gr].x);
          }
        smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 1));
        smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 2));
        const int u_need = smax > 0.0f ? min(100, 14 - ilogbf(smax)) : 100;
        const bool u_changed = u_need < u_run;
        const float u_shift = u_changed ? __int_as_float((127 + u_need - u_run) << 23) : 1.0f;
        if (u_changed) u_run = u_need;
        const float f_u = __int_as_float((127 + u_run) << 23);
        uint32_t bp[NP][NG][2];
#pragma unroll
        for (int pt = 0; pt < NP; ++pt) {
          const int hd = 4 * pt + (g >> 1);
          const int part = g & 1;
          float pv[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) pv[x] = wpex[kk[x] * 8 + hd];
          const float az = changed ? walph[hd] : 1.0f;
#pragma unroll
          for (int gr = 0; gr < NG; ++gr) {
            __half hv[4];
            float z = 0.0f;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const float P = pv[x] == 0.0f ? 0.0f : (pv[x] * f_u) * svz[x][gr].x;
              const __half hi = __float2half_rn(P);
              hv[x] = part ? __float2half_rn(P - __half2float(hi)) : hi;
              z += pv[x] == 0.0f ? 0.0f : pv[x] * svz[x][gr].y;
            }
            bp[pt][gr][0] = pack_half2(hv[0], hv[1]);
            bp[pt][gr][1] = pack_half2(hv[2], hv[3]);
            if (part == 0) zacc[pt][gr] = fmaf(zacc[pt][gr], az, z);
          }
        }
        if (changed || u_changed) {
#pragma unroll
          for (int pt = 0; pt < NP; ++pt) {
            const float ao = (changed ? walph[4 * pt + c] : 1.0f) * u_shift;
#pragma unroll
            for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
              for (int r = 0; r < 4; ++r) oacc[j][pt][r] *= ao;
          }
        }

        // ---- output: O^T[dim][head] += codes^T . (p * scale_v)
        uint32_t vw[C::VW];
#pragma unroll
        for (int pc = 0; pc < C::VN / C::VP; ++pc)
          lds_words<C::VP>(vt + pc * 32 * C::VP + lane * C::VP, vw, pc * (C::VP / 4));
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j) {
          const int gr = 16 * j / G;
          const uint32_t a0 = extract_codes<C::BV>(vw, 0, 2 * j);
          const uint32_t a1 = extract_codes<C::BV>(vw, 0, 2 * j + 1);
          const uint32_t a2 = extract_codes<C::BV>(vw, C::WV, 2 * j);
          const uint32_t a3 = extract_codes<C::BV>(vw, C::WV, 2 * j + 1);
#pragma unroll
          for (int pt = 0; pt < NP; ++pt)
            mma_f16_16816(oacc[j][pt], a0, a1, a2, a3, bp[pt][gr][0], bp[pt][gr][1]);
        }
        __syncwarp();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  // ------------------------------------------------------------ epilogue
  __syncthreads();  // all stages consumed; the ring becomes the merge buffer
  float* ob = reinterpret_cast<float*>(smem);  // [warp][8][D]
  float* mb = pex;                             // [warp][8]
  float* lb = pex + 32;                        // [warp][8]
  float* zb = pex + 64;                        // [warp][8][NG]
  if (warp < C::kWarps) {
#pragma unroll
    for (int hs = 0; hs < HT; ++hs) {
      float l = l_run[hs];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      const int head = QS == 2 ? 4 * hs + c : 8 * (hs / 2) + 2 * c + (hs & 1);
      if (g == 0) {
        mb[warp * 8 + head] = m_run[hs];
        lb[warp * 8 + head] = l;
      }
    }
#pragma unroll
    for (int pt = 0; pt < NP; ++pt)
#pragma unroll
      for (int gr = 0; gr < NG; ++gr) {
        float z = zacc[pt][gr];
        z += __shfl_xor_sync(0xffffffffu, z, 1);
        z += __shfl_xor_sync(0xffffffffu, z, 2);
        if ((g & 1) == 0 && c == 0) zb[(warp * 8 + 4 * pt + (g >> 1)) * NG + gr] = z;
      }
#pragma unroll
    for (int pt = 0; pt < NP; ++pt) {
      const int head = 4 * pt + c;
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j) {
        const float s0 = ldexpf(1.0f, 24 - u_run - field_pos<C::BV>((2 * j) % (16 / C::BV)));
        const float s1 = ldexpf(1.0f, 24 - u_run - field_pos<C::BV>((2 * j + 1) % (16 / C::BV)));
        ob[(warp * 8 + head) * D + 16 * j + g] = (oacc[j][pt][0] + oacc[j][pt][1]) * s0;
        ob[(warp * 8 + head) * D + 16 * j + 8 + g] = (oacc[j][pt][2] + oacc[j][pt][3]) * s1;
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nh * D; idx += C::kThreads) {
    const int head = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, mb[w * 8 + head]);
    float num = 0.0f, den = 0.0f;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) {
      const float mw = mb[w * 8 + head];
      if (mw == -INFINITY) continue;
      const float wt = exp2f(mw - M);
      num = fmaf(wt, ob[(w * 8 + head) * D + d] + zb[(w * 8 + head) * NG + d / G], num);
      den = fmaf(wt, lb[w * 8 + head], den);
    }
    const size_t row = (static_cast<size_t>(b) * a.q_heads + head0 + head) * a.num_splits + split;
    a.ws_o[row * D + d] = num / den;
    if (d == 0) a.ws_lse[row] = M + log2f(den);
  }
}

template <class C>
cudaError_t launch_decode(const DecodeArgs& a, dim3 grid, cudaStream_t stream) {
  decode_kernel<C><<<grid, C::kThreads, C::SMEM_BYTES, stream>>>(a);
  return cudaGetLastError();
}

template <class C>
DecodeKernel make_decode_kernel() {
  DecodeKernel k;
  k.fn = reinterpret_cast<const void*>(&decode_kernel<C>);
  k.threads = C::kThreads;
  k.smem_bytes = C::SMEM_BYTES;
  k.launch = &launch_decode<C>;
  return k;
}

// Instances for one (bits_k, bits_v) pair: D in {64, 128}, groups per row,
// and the four query variants.
template <int BK, int BV>
bool get_decode_kernel_bits(int head_dim, int num_groups, int variant, DecodeKernel* out) {
#define KVQ_VARIANTS(D, NG)                                                        \
  switch (variant) {                                                               \
    case 0: *out = make_decode_kernel<DecodeCfg<D, BK, BV, NG, 1, 1, 1>>(); return true; \
    case 1: *out = make_decode_kernel<DecodeCfg<D, BK, BV, NG, 2, 1, 1>>(); return true; \
    case 2: *out = make_decode_kernel<DecodeCfg<D, BK, BV, NG, 1, 1, 2>>(); return true; \
    case 3: *out = make_decode_kernel<DecodeCfg<D, BK, BV, NG, 2, 2, 2>>(); return true; \
    default: return false;                                                         \
  }
  if (head_dim == 128) {
    if (num_groups == 1) { KVQ_VARIANTS(128, 1) }
    if (num_groups == 2) { KVQ_VARIANTS(128, 2) }
    if (num_groups == 4) { KVQ_VARIANTS(128, 4) }
  } else if (head_dim == 64) {
    if (num_groups == 1) { KVQ_VARIANTS(64, 1) }
    if (num_groups == 2) { KVQ_VARIANTS(64, 2) }
  }
#undef KVQ_VARIANTS
  return false;
}

}  // namespace kvq
