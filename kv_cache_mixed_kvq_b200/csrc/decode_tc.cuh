// Split-K flash-decoding over the packed mixed-precision cache on the
// Blackwell tensor cores (tcgen05, operands and accumulators in tensor
// memory), head_dim 128.
//
// One decode step of attention ("Quantize What Counts: More for Keys, Less
// for Values", summary page, "Problem statement": the quantized KV cache is
// what inference reads) for one (split of the tokens, kv head, batch row):
//
//   s_t = sm_scale * q . k^_t,  k^ = code * scale + zero   (per group)
//   o   = sum_t softmax(s)_t v^_t
//
// Design (B200, sm_100a): one CTA per SM, tiles of 128 positions, three
// warp roles that hand tiles to each other through mbarriers (every wait
// bounded), so that unpacking, the tensor-core products and the softmax of
// different tiles overlap:
//  * control warp (one thread): streams whole tiles (K rows, V tiles and both
//    parameter arrays of 128 positions) into a ring of shared-memory stages
//    with 1-D bulk copies (cp.async.bulk, no multicast), and issues the two
//    tensor-core products of every tile (tcgen05.mma, D in tensor memory);
//  * four unpack warps: codes become exact binary16 operands with one AND
//    per two codes (code * 2^(pos-24), a subnormal or first-binade value) and
//    go from registers to tensor memory (tcgen05.st), the keys as
//    A[position][dim] of the score product and the values as A[dim][position]
//    of the output product; two tensor-memory buffers, so that tile i+1 is
//    unpacked while tile i is multiplied;
//  * four softmax warps, one position and one dimension per thread: read the
//    scores (tcgen05.ld), apply the per-group scale and zero
//      q.k^ = sum_g scale_g (q . c_g) + zero_g sum_{d in g} q_d,
//    run the online softmax in binary32 (exp2 domain, a running maximum
//    shared by the four warps and updated lazily, only when a score exceeds
//    it by more than 2^3), write the output product's B operand (weights
//    p_t * scale_t, split into binary16 high and low parts and scaled by a
//    power of two that only decreases), sum the zero term
//    sum_t p_t zero_t, and fold each tile's output product (read back one
//    dimension per thread) into binary32 accumulators in registers.
// The score product's B operand is the query, split into binary16 high and
// low parts, scaled per head by a power of two and per dimension by the
// code's 2^-pos, laid out block-diagonally by key group so that each group's
// partial dot products land in their own columns.  Partial results per split
// are merged by the log-sum-exp combine kernel, or written directly when a
// row has a single split.
#pragma once

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace kvq {

// HP: query heads per CTA, padded (4 or 8).  NGK / NGV: groups per row of
// the keys / values.
template <int BK_, int BV_, int NGK_, int NGV_, int HP_>
struct TcCfg {
  static constexpr int D = 128, BK = BK_, BV = BV_, NGK = NGK_, NGV = NGV_, HP = HP_;
  static constexpr int kUnpackWarps = 4, kSoftmaxWarps = 4;
  static constexpr int kWarps = kUnpackWarps + kSoftmaxWarps + 1;  // + the control warp
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kCtrlWarp = kUnpackWarps + kSoftmaxWarps;
  static constexpr int TILE = 128;  // positions per tile (M of the score product)
  static constexpr int GK = D / NGK, GV = D / NGV;
  static constexpr int C = 2 * HP;  // columns per group: (high, low) per head
  static constexpr int NS = NGK * C < 16 ? 16 : NGK * C;  // N of the score product
  static constexpr int NO = NGV * C < 16 ? 16 : NGV * C;  // N of the output product
  static constexpr int NBS = NS / 8, NBO = NO / 8;        // 8-column blocks
  static constexpr int KROW = D * BK / 8;      // bytes per K row
  static constexpr int KSLICE = D * BK / 32;   // bytes of one lane's slice of a row
  static constexpr int KW = KSLICE / 4;        // words per slice
  static constexpr int EK = 16 / BK, EV = 16 / BV;  // fields per 16-bit half
  static constexpr int VTILE = 2 * D * BV;     // bytes per 16-position V tile
  static constexpr int VN = D * BV / 16;       // bytes per lane of a V tile
  static constexpr int VP = VN < 16 ? VN : 16; // piece size of the lane bytes
  static constexpr int WV = D * BV / 128;      // V words per half-lane
  static constexpr int PROWK = NGK * 4, PROWV = NGV * 4;  // parameter bytes per position
  // one stage = one tile: K rows, V tiles, K parameters, V parameters
  static constexpr int ST_K = TILE * KROW, ST_V = (TILE / 16) * VTILE;
  static constexpr int ST_PK = TILE * PROWK, ST_PV = TILE * PROWV;
  static constexpr int STAGE = ST_K + ST_V + ST_PK + ST_PV;
  static constexpr int BQ_BYTES = D * NS * 2;     // score B operand: 128 dims x NS
  static constexpr int BW_BYTES = TILE * NO * 2;  // output B operand (x2): 128 positions x NO
  static constexpr int RED_FLOATS = kSoftmaxWarps * (HP + 1 + NGV * HP);
  // stages: as many as fit in about 200 KB next to the operands (at most 12)
  static constexpr int FIXED = BQ_BYTES + 2 * BW_BYTES + 4 * RED_FLOATS + 256;
  static constexpr int NST_FIT = (200 * 1024 - FIXED) / STAGE;
  static constexpr int NSTAGES = NST_FIT > 12 ? 12 : NST_FIT;
  static constexpr int RING = NSTAGES * STAGE;
  static constexpr int BQ_OFF = RING, BW_OFF = RING + BQ_BYTES;
  static constexpr int RED_OFF = BW_OFF + 2 * BW_BYTES;
  static constexpr int BAR_OFF = RED_OFF + 4 * RED_FLOATS;
  static constexpr int NBARS = NSTAGES + 8;  // full[NSTAGES], unpacked[2], s_done[2], w_ready[2], o_done[2]
  static constexpr int SMEM_BYTES = BAR_OFF + 8 * NBARS + 32;
  // tensor memory columns (512: the whole SM; one CTA per SM)
  static constexpr int TM_AK = 0;                // key codes [2]: 128 positions x 64 columns
  static constexpr int TM_AV = 128;              // value codes [2]: 128 dims x 64 columns
  static constexpr int TM_DS = 256;              // scores [2]: 128 positions x NS
  static constexpr int TM_DO = 256 + 2 * NS;     // output [2]: 128 dims x NO
  static constexpr int TM_COLS = 512;
  static_assert(TM_DO + 2 * NO <= TM_COLS, "tensor memory columns");
  static_assert(NSTAGES >= 2, "stages");
  static_assert(SMEM_BYTES > 114 * 1024 && SMEM_BYTES <= 227 * 1024,
                "one CTA per SM (it holds all of the SM's tensor memory)");
  static_assert(STAGE % 16 == 0 && ST_K % 16 == 0 && ST_V % 16 == 0 && ST_PK % 16 == 0,
                "stage alignment");
  static_assert(BQ_OFF % 128 == 0 && BW_OFF % 128 == 0 && BW_BYTES % 128 == 0, "operand alignment");
  static_assert(GK >= 32 && GV >= 32, "a group must cover whole warps of dimensions");
  static_assert(2 * BW_BYTES >= HP * D * 4, "query rows must fit in the output operand buffers");
};

// Position of the tile held by tensor-memory lane r of a 16-lane block: the
// middle quads are swapped so that the eight lanes of a quarter warp write
// the output operand's rows without bank conflicts.
__device__ __forceinline__ int tc_lane_pos(int r) {
  return (r >= 4 && r < 12) ? (r ^ 12) : r;
}

// Field e of b-bit codes in a 16-bit half: pre-shift and bit position.
template <int B>
__host__ __device__ constexpr int tc_fshift(int e) { return (e * B >= 8) ? 8 : 0; }
template <int B>
__host__ __device__ constexpr int tc_fpos(int e) { return e * B - tc_fshift<B>(e); }

// Two codes (low and high half) of field e of a word as binary16 values
// code * 2^(tc_fpos(e) - 24).
template <int B>
__device__ __forceinline__ uint32_t tc_extract(uint32_t w, int e) {
  const uint32_t m = ((1u << B) - 1u) << tc_fpos<B>(e);
  return (w >> tc_fshift<B>(e)) & (m | (m << 16));
}

// Keys of warp q's 32 positions (two 16-position blocks) -> tensor memory
// at column `col` (lanes = positions, columns = dimension pairs).  For the
// 16x256b store, thread (g, c) owns the rows tc_lane_pos(g) and
// tc_lane_pos(g + 8) of a block; repetition j, half x holds the dims
// 8(2j + x) + 2c + {0, 1}.
template <class C>
__device__ __forceinline__ void tc_unpack_keys(const uint8_t* st, int q, int lane, uint32_t tbase,
                                               int col) {
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    const int r0 = 32 * q + 16 * blk;
    uint32_t wa[C::KW], wb[C::KW];
    const uint8_t* pa = st + (r0 + tc_lane_pos(g)) * C::KROW + c * C::KSLICE;
    const uint8_t* pb = st + (r0 + tc_lane_pos(g + 8)) * C::KROW + c * C::KSLICE;
    if constexpr (C::KSLICE % 16 == 0) {
#pragma unroll
      for (int i = 0; i < C::KSLICE / 16; ++i) {
        const uint4 u = *reinterpret_cast<const uint4*>(pa + 16 * i);
        const uint4 v = *reinterpret_cast<const uint4*>(pb + 16 * i);
        wa[4 * i] = u.x; wa[4 * i + 1] = u.y; wa[4 * i + 2] = u.z; wa[4 * i + 3] = u.w;
        wb[4 * i] = v.x; wb[4 * i + 1] = v.y; wb[4 * i + 2] = v.z; wb[4 * i + 3] = v.w;
      }
    } else {
      static_assert(C::KSLICE == 8, "slice size");
      const uint2 u = *reinterpret_cast<const uint2*>(pa);
      const uint2 v = *reinterpret_cast<const uint2*>(pb);
      wa[0] = u.x; wa[1] = u.y;
      wb[0] = v.x; wb[1] = v.y;
    }
    uint32_t r[32];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int m = 2 * j + x;  // 8-dim block index
        r[4 * j + x] = tc_extract<C::BK>(wa[m / C::EK], m % C::EK);
        r[4 * j + 2 + x] = tc_extract<C::BK>(wb[m / C::EK], m % C::EK);
      }
    tc::st_16x256b_x8(tc::addr(tbase, r0, col), r);
  }
}

// Values of warp q's 32 dimensions over the tile's 128 positions -> tensor
// memory at column `col` (lanes = dimensions, columns = position pairs).
// Lane block blk covers dims 32q + 16blk + [0, 16), i.e. the 8-dim blocks
// me = 4q + 2blk (rows g) and me + 1 (rows g + 8); for the 16-position V
// tile s, column 8s + 2c + kh holds positions 16s + 2c + 8kh + {0, 1}.
// The field of block me within its half-word is the same for every warp
// once the word is shifted right by 16 * (me / EV) bits of the lane's data
// (whole words) and by kWarpShift bits.
template <class C>
__device__ __forceinline__ void tc_unpack_values(const uint8_t* sv, int q, int lane,
                                                 uint32_t tbase, int col) {
  constexpr int EV = C::EV;
  uint32_t ra[32], rb[32];
  // fields of me = 4q + 2blk + x: e = me % EV; for 2-bit codes the warps
  // with q odd use fields 4..7 (one shift by 8 per word, then 0..3)
  const int wshift = (EV == 8 && (q & 1)) ? 8 : 0;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint8_t* vt = sv + s * C::VTILE + lane * C::VP;
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      const int me = 4 * q + 2 * blk;
      const int q0 = me / EV, q1 = C::WV + me / EV;  // words of positions kh = 0, 1
      const int n0 = 4 * q0, n1 = 4 * q1;
      uint32_t w0 = *reinterpret_cast<const uint32_t*>(vt + (n0 / C::VP) * 32 * C::VP + n0 % C::VP);
      uint32_t w1 = *reinterpret_cast<const uint32_t*>(vt + (n1 / C::VP) * 32 * C::VP + n1 % C::VP);
      constexpr int ex = EV == 8 ? 4 : EV;  // fields reached after the warp's shift
      const int e0 = (2 * blk) % ex, e1 = (2 * blk + 1) % ex;
      if constexpr (EV == 8) {
        w0 >>= wshift;
        w1 >>= wshift;
      }
      uint32_t* r = blk ? rb : ra;
      r[4 * s + 0] = tc_extract<C::BV>(w0, e0);
      r[4 * s + 1] = tc_extract<C::BV>(w1, e0);
      r[4 * s + 2] = tc_extract<C::BV>(w0, e1);
      r[4 * s + 3] = tc_extract<C::BV>(w1, e1);
    }
  }
  tc::st_16x256b_x8(tc::addr(tbase, 32 * q, col), ra);
  tc::st_16x256b_x8(tc::addr(tbase, 32 * q + 16, col), rb);
}

// Field position of the value codes of dimension d (its output row's scale).
template <class C>
__device__ __forceinline__ int tc_vpos(int d) {
  const int e = (d >> 3) % C::EV;
  return e * C::BV - ((e * C::BV >= 8) ? 8 : 0);
}

__device__ __forceinline__ float warp_max_all(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}
__device__ __forceinline__ float warp_sum_all(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// Two binary32 values as (high, low) binary16 parts packed per value:
// returns the words (hi(a) | lo(a) << 16) and (hi(b) | lo(b) << 16).
__device__ __forceinline__ void tc_split_pair(float a, float b, uint32_t& wa, uint32_t& wb) {
  const uint32_t hi = f2_to_h2(a, b);
  const float2 hf = unpack_half2(hi);
  const uint32_t lo = f2_to_h2(a - hf.x, b - hf.y);
  wa = __byte_perm(hi, lo, 0x5410);
  wb = __byte_perm(hi, lo, 0x7632);
}

// Barrier of the four softmax warps only (named barrier 1).
__device__ __forceinline__ void softmax_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// The same barrier, returning whether any of the 128 threads passed true.
__device__ __forceinline__ bool softmax_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u)
      : "memory");
  return r != 0;
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1) decode_tc_kernel(const DecodeArgs a) {
  constexpr int D = C::D, HP = C::HP, NGK = C::NGK, NGV = C::NGV, CC = C::C, TILE = C::TILE;
  constexpr int NST = C::NSTAGES;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint8_t* bq = smem + C::BQ_OFF;
  uint8_t* bw = smem + C::BW_OFF;  // two buffers of BW_BYTES
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* unpacked = full + NST;
  uint64_t* s_done = unpacked + 2;
  uint64_t* w_ready = s_done + 2;
  uint64_t* o_done = w_ready + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(full + C::NBARS);
  int* votes = reinterpret_cast<int*>(tslot + 2);  // [4]

  const int split = blockIdx.x;
  const int hk = blockIdx.y / a.head_groups;
  const int hg = blockIdx.y % a.head_groups;
  const int b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  pdl_wait();
  pdl_trigger();
  int len = a.seq_lens[b];
  const int lim = min(a.max_seq_len, a.capacity);
  if (len < 0 || len > lim) {
    if (split == 0 && blockIdx.y == 0 && tid == 0) flag_error(a.err, KVQ_DEVERR_SEQ_LEN);
    len = max(0, min(len, lim));
  }
  const int t0 = split * a.split_tokens;
  const int head0 = hk * a.gq + hg * a.heads_per_cta;
  const int nh = min(a.heads_per_cta, a.gq - hg * a.heads_per_cta);
  if (t0 >= len) {
    if (a.direct && len == 0 && split == 0)
      for (int i = tid; i < nh * D; i += C::kThreads)
        store_out(a.out, a.out_dtype,
                  (static_cast<size_t>(b) * a.q_heads + head0 + i / D) * D + i % D, 0.0f);
    return;
  }
  const int n_tok = min(t0 + a.split_tokens, len) - t0;
  const int n_tiles = (n_tok + TILE - 1) / TILE;
  const size_t slot = static_cast<size_t>(b) * a.kv_heads + hk;
  uint32_t* const err = a.err;
  const uint64_t wlim = a.wait_limit_ns;

  if (warp == 0) {
    tc::alloc(tslot, C::TM_COLS);
    tc::relinquish();
  }
  if (tid == 32 * C::kCtrlWarp) {
    for (int i = 0; i < NST; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&unpacked[i], C::kUnpackWarps);
      mbar_init(&s_done[i], 1);
      mbar_init(&w_ready[i], C::kSoftmaxWarps);
      mbar_init(&o_done[i], 1);
    }
    fence_barrier_init();
  }

  // ------------------------------------------------------------- copies
  // Tile j: positions t0 + TILE*j .. + n16 (n16: the valid count rounded up
  // to 16); a paged cache maps them page by page (pages hold >= 32).
  auto issue = [&](int j, int st) {
    const int base = j * TILE;
    const int n16 = (min(TILE, n_tok - base) + 15) & ~15;
    uint8_t* dst = ring + st * C::STAGE;
    if (j == a.fault_stage && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
      // test knob: bytes announced, no copy issued (the wait runs out)
      mbar_arrive_expect_tx(&full[st],
                            n16 * (C::KROW + C::PROWK + C::PROWV) + (n16 / 16) * C::VTILE);
      return;
    }
    // two passes over the page chunks: bytes first (one expect_tx), then copies
    uint32_t bytes = 0;
    for (int pass = 0; pass < 2; ++pass) {
      if (pass == 1) mbar_arrive_expect_tx(&full[st], bytes);
      int p0 = 0;
      while (p0 < n16) {
        const int tb = t0 + base + p0;
        int chunk = n16 - p0;
        size_t r = slot * a.capacity + tb;
        bool ok = true;
        if (a.block_table != nullptr) {
          const int P = 1 << a.page_shift;
          chunk = min(chunk, P - (tb & (P - 1)));
          const int page =
              a.block_table[static_cast<size_t>(b) * a.pages_per_seq + (tb >> a.page_shift)];
          ok = page >= 0 && page < a.num_pages;
          if (!ok && pass == 0) flag_error(err, KVQ_DEVERR_BAD_PAGE);  // never read
          if (ok) r = ((static_cast<size_t>(page) * a.kv_heads + hk) << a.page_shift) + (tb & (P - 1));
        }
        if (ok && pass == 0) bytes += chunk * (C::KROW + C::PROWK + C::PROWV) + (chunk / 16) * C::VTILE;
        if (ok && pass == 1) {
          bulk_copy_g2s(dst + p0 * C::KROW, a.k_codes + r * C::KROW, chunk * C::KROW, &full[st]);
          bulk_copy_g2s(dst + C::ST_K + (p0 / 16) * C::VTILE, a.v_codes + (r / 16) * C::VTILE,
                        (chunk / 16) * C::VTILE, &full[st]);
          bulk_copy_g2s(dst + C::ST_K + C::ST_V + p0 * C::PROWK,
                        reinterpret_cast<const uint8_t*>(a.k_params) + r * C::PROWK,
                        chunk * C::PROWK, &full[st]);
          bulk_copy_g2s(dst + C::ST_K + C::ST_V + C::ST_PK + p0 * C::PROWV,
                        reinterpret_cast<const uint8_t*>(a.v_params) + r * C::PROWV,
                        chunk * C::PROWV, &full[st]);
        }
        p0 += chunk;
      }
    }
  };
  __syncthreads();  // barriers initialised before any copy completes on them
  if (tid == 32 * C::kCtrlWarp)
    for (int j = 0; j < min(NST, n_tiles); ++j) issue(j, j);

  // ------------------------------------------ query operand, once per CTA
  // The softmax warps (threads s = 0..127) stage the query rows (binary32) in
  // the output operand buffers, unused until the first weights; with
  // rotated keys the rows become H q / D.
  const bool is_sm = warp >= C::kUnpackWarps && warp < C::kCtrlWarp;
  const int s_tid = tid - 32 * C::kUnpackWarps;  // softmax thread index (0..127)
  const int sq = warp - C::kUnpackWarps;          // softmax warp = tensor-memory quadrant
  float* qs = reinterpret_cast<float*>(bw);       // [HP][D]
  float F[HP];        // log2-domain score per unit of the code product
  float qz[NGK][HP];  // sm_scale * log2(e) * sum of q over key group g
  if (is_sm) {
    for (int i = s_tid; i < HP * D; i += 128) {
      const int hh = i / D;
      qs[i] = hh < nh ? load_elem(a.q, a.q_dtype,
                                  (static_cast<size_t>(b) * a.q_heads + head0 + hh) * D + i % D)
                      : 0.0f;
    }
    softmax_sync();
    if (a.rotate_q) {
#pragma unroll 1
      for (int h = 1; h < D; h *= 2) {
        for (int i = s_tid; i < nh * D / 2; i += 128) {
          const int r = i % (D / 2);
          float* x = qs + (i / (D / 2)) * D + (r / h) * 2 * h + (r % h);
          const float x0 = x[0], x1 = x[h];
          x[0] = x0 + x1;
          x[h] = x0 - x1;
        }
        softmax_sync();
      }
      for (int i = s_tid; i < nh * D; i += 128) qs[i] *= 1.0f / D;  // exact: D = 2^7
      softmax_sync();
    }
    // per head: largest |q| (for the split's power of two) and the sum over
    // each key group; thread s_tid = dim
    float* qmax = red;       // [warp][HP]
    float* qsum = red + 4 * HP;  // [warp][HP]
#pragma unroll
    for (int hh = 0; hh < HP; ++hh) {
      const float v = qs[hh * D + s_tid];
      const float mx = warp_max_all(fabsf(v));
      const float sm = warp_sum_all(v);
      if (lane == 0) {
        qmax[sq * HP + hh] = mx;
        qsum[sq * HP + hh] = sm;
      }
    }
    softmax_sync();
    int eqh[HP];
#pragma unroll
    for (int hh = 0; hh < HP; ++hh) {
      float mx = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) mx = fmaxf(mx, qmax[w * HP + hh]);
      eqh[hh] = mx > 0.0f ? max(-100, min(100, 14 - ilogbf(mx))) : 0;
      F[hh] = a.sm_scale_log2 * pow2i(24 - eqh[hh]);
#pragma unroll
      for (int g = 0; g < NGK; ++g) {
        float s = 0.0f;
        constexpr int WPG = C::GK / 32;  // warps per key group
#pragma unroll
        for (int w = 0; w < WPG; ++w) s += qsum[(g * WPG + w) * HP + hh];
        qz[g][hh] = a.sm_scale_log2 * s;
      }
    }
    // score B operand, MN-major: row kappa (this thread) = dim
    // 16j + 8x + 2c + h for kappa = 16j + 4c + 2x + h; columns g*CC + 2hh +
    // {high, low} of the dim's key group, zero elsewhere
    {
      const int kap = s_tid;
      const int j = kap >> 4, c = (kap >> 2) & 3, x = (kap >> 1) & 1, h = kap & 1;
      const int d = 16 * j + 8 * x + 2 * c + h;
      const int gk = d / C::GK;
      const int e = (d >> 3) % C::EK;
      const int pos = e * C::BK - ((e * C::BK >= 8) ? 8 : 0);
      uint32_t row[C::NS / 2];
#pragma unroll
      for (int i = 0; i < C::NS / 2; ++i) row[i] = 0u;
#pragma unroll
      for (int hh = 0; hh < HP; ++hh) {
        const float v = qs[hh * D + d] * pow2i(eqh[hh] - pos);
        const __half hi = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(hi));
#pragma unroll
        for (int g = 0; g < NGK; ++g)
          if (g == gk) row[g * HP + hh] = pack_half2(hi, lo);
      }
#pragma unroll
      for (int nb = 0; nb < C::NBS; ++nb)
        *reinterpret_cast<uint4*>(bq + ((kap >> 3) * C::NBS + nb) * 128 + (kap & 7) * 16) =
            make_uint4(row[4 * nb], row[4 * nb + 1], row[4 * nb + 2], row[4 * nb + 3]);
    }
    softmax_sync();  // every read of qs done before the buffers take weights
    // zero the padding columns of both output operand buffers once
    if constexpr (C::NO > NGV * CC) {
      for (int i = s_tid; i < 2 * TILE * C::NBO; i += 128) {
        const int buf = i / (TILE * C::NBO), k = i % (TILE * C::NBO);
        const int kap = k / C::NBO, nb = k % C::NBO;
        if (nb * 8 >= NGV * CC)
          *reinterpret_cast<uint4*>(bw + buf * C::BW_BYTES +
                                    ((kap >> 3) * C::NBO + nb) * 128 + (kap & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
    }
    fence_proxy_async_shared();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tslot;

  if (warp < C::kUnpackWarps) {
    // ========================================================= unpack warps
    const int q = warp;
    for (int i = 0; i < n_tiles; ++i) {
      const int bi = i & 1;
      bool to = !mbar_wait_bounded(&full[i % NST], (i / NST) & 1, err, wlim);
      // the buffers of tile i - 2 are free once its output product is done
      if (!to && i >= 2) to = !mbar_wait_bounded(&o_done[bi], ((i - 2) >> 1) & 1, err, wlim);
      if (__any_sync(0xffffffffu, to)) break;  // (tcgen05.st is warp-collective)
      tc::fence_after_sync();
      const uint8_t* sp = ring + (i % NST) * C::STAGE;
      tc_unpack_keys<C>(sp, q, lane, tbase, C::TM_AK + 64 * bi);
      tc_unpack_values<C>(sp + C::ST_K, q, lane, tbase, C::TM_AV + 64 * bi);
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&unpacked[bi]);
    }
  } else if (warp == C::kCtrlWarp) {
    // ======================================================== control warp
    if (lane == 0) {
      const uint32_t idesc_s = tc::idesc_f16(128, C::NS);
      const uint32_t idesc_o = tc::idesc_f16(128, C::NO);
      const uint32_t bq_addr = smem_addr(bq), bw_addr = smem_addr(bw);
      int issued = min(NST, n_tiles);
      int s_committed = 0, o_committed = 0;
      bool ok = true;
      for (int j = 0; j <= n_tiles && ok; ++j) {
        if (j < n_tiles) {
          ok = mbar_wait_bounded(&unpacked[j & 1], (j >> 1) & 1, err, wlim);
          if (!ok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_f16_ts(tc::addr(tbase, 0, C::TM_DS + C::NS * (j & 1)),
                           tc::addr(tbase, 0, C::TM_AK + 64 * (j & 1) + 8 * ks),
                           tc::smem_desc(bq_addr + ks * 2 * (C::NBS * 128), C::NBS * 128, 128),
                           idesc_s, ks > 0);
          tc::commit(&s_done[j & 1]);
          s_committed = j + 1;
        }
        if (j >= 1) {
          const int pj = j - 1;
          ok = mbar_wait_bounded(&w_ready[pj & 1], (pj >> 1) & 1, err, wlim);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t bwa = bw_addr + (pj & 1) * C::BW_BYTES;
#pragma unroll
          for (int s = 0; s < 8; ++s)
            tc::mma_f16_ts(tc::addr(tbase, 0, C::TM_DO + C::NO * (pj & 1)),
                           tc::addr(tbase, 0, C::TM_AV + 64 * (pj & 1) + 8 * s),
                           tc::smem_desc(bwa + s * 2 * (C::NBO * 128), C::NBO * 128, 128),
                           idesc_o, s > 0);
          tc::commit(&o_done[pj & 1]);
          o_committed = j;
          // tile pj is consumed (codes unpacked, parameters read): refill its stage
          if (pj + NST < n_tiles) {
            fence_proxy_async_shared();
            issue(pj + NST, pj % NST);
            issued = pj + NST + 1;
          }
        }
      }
      if (!ok) {
        // drain: every copy issued and every product committed must finish
        // before the CTA exits (bounded)
        for (int k = max(0, issued - NST); k < issued; ++k)
          mbar_wait_bounded(&full[k % NST], (k / NST) & 1, err, wlim);
        if (s_committed > 0)
          mbar_wait_bounded(&s_done[(s_committed - 1) & 1], ((s_committed - 1) >> 1) & 1, err, wlim);
        if (o_committed > 0)
          mbar_wait_bounded(&o_done[(o_committed - 1) & 1], ((o_committed - 1) >> 1) & 1, err, wlim);
      }
    }
    __syncwarp();
  } else {
    // ======================================================== softmax warps
    // shared by the four warps: running maximum per head (lazily updated),
    // weight exponent u (only decreases); per thread: partial sums
    constexpr float kLazy = 8.0f;
    float m_run[HP], l_part[HP], z_part[NGV][HP], o_acc[HP];
    float alpha_prev[HP], alpha_cur[HP];  // rescales due at the next two read-backs
    int u_run = 100, u_prev = 100;
    float u_bound = pow2i(7 - 100);
#pragma unroll
    for (int hh = 0; hh < HP; ++hh) {
      m_run[hh] = -INFINITY;
      l_part[hh] = 0.0f;
      o_acc[hh] = 0.0f;
      alpha_prev[hh] = alpha_cur[hh] = 1.0f;
#pragma unroll
      for (int g = 0; g < NGV; ++g) z_part[g][hh] = 0.0f;
    }
    // this thread's dimension (output side) and position (score side)
    const int d_me = s_tid;
    const int gv_me = d_me / C::GV;
    const float vscale_me = pow2i(24 - tc_vpos<C>(d_me));
    const int tok_me = 16 * (s_tid >> 4) + tc_lane_pos(s_tid & 15);
    const int rr = tok_me & 15;
    const int kap_me = 16 * (tok_me >> 4) + 4 * ((rr & 7) >> 1) + 2 * (rr >> 3) + (rr & 1);
    const int bw_row_off = (kap_me >> 3) * C::NBO * 128 + (kap_me & 7) * 16;

    // Folds the output product of tile j (made with exponent uj, after the
    // rescale alpha of its own update) into o_acc; false if its wait ran out.
    auto read_back = [&](int j, int uj, const float (&alpha)[HP]) -> bool {
      if (__any_sync(0xffffffffu, !mbar_wait_bounded(&o_done[j & 1], (j >> 1) & 1, err, wlim)))
        return false;
      tc::fence_after_sync();
      uint32_t r[CC];
      tc::ld_32x32b<CC>(tc::addr(tbase, 32 * sq, C::TM_DO + C::NO * (j & 1) + gv_me * CC), r);
      tc::wait_ld();
      const float s = vscale_me * pow2i(-uj);
#pragma unroll
      for (int hh = 0; hh < HP; ++hh)
        o_acc[hh] = fmaf(o_acc[hh], alpha[hh],
                         (__uint_as_float(r[2 * hh]) + __uint_as_float(r[2 * hh + 1])) * s);
      return true;
    };

    // A wait that runs out ends the loop of all four warps together, at the
    // next barrier of the group (their named barriers must all be reached).
    bool ok = true;
    bool to = false;  // a wait of this group ran out
    for (int i = 0; i < n_tiles; ++i) {
      const int bi = i & 1;
      to = to || __any_sync(0xffffffffu, !mbar_wait_bounded(&s_done[bi], (i >> 1) & 1, err, wlim));
      tc::fence_after_sync();
      const uint8_t* sp = ring + (i % NST) * C::STAGE;
      const int n_valid = min(TILE, n_tok - i * TILE);
      const bool valid = tok_me < n_valid;
      float lg[HP], sv[NGV], zv[NGV];
      float smax = 0.0f;
      {
        uint32_t sr[C::NS];
        if (!to) tc::ld_32x32b<C::NS>(tc::addr(tbase, 32 * sq, C::TM_DS + C::NS * bi), sr);
        const uint8_t* pk = sp + C::ST_K + C::ST_V + tok_me * C::PROWK;
        const uint8_t* pv = sp + C::ST_K + C::ST_V + C::ST_PK + tok_me * C::PROWV;
        float sk[NGK], zk[NGK];
#pragma unroll
        for (int g = 0; g < NGK; ++g) {
          const float2 p2 = unpack_half2(*reinterpret_cast<const uint32_t*>(pk + 4 * g));
          sk[g] = p2.x;
          zk[g] = p2.y;
        }
#pragma unroll
        for (int g = 0; g < NGV; ++g) {
          const float2 p2 = unpack_half2(*reinterpret_cast<const uint32_t*>(pv + 4 * g));
          sv[g] = valid ? p2.x : 0.0f;
          zv[g] = valid ? p2.y : 0.0f;
          smax = fmaxf(smax, sv[g]);
        }
        tc::wait_ld();
#pragma unroll
        for (int hh = 0; hh < HP; ++hh) {
          float t = 0.0f, z = 0.0f;
#pragma unroll
          for (int g = 0; g < NGK; ++g) {
            const float s2 =
                __uint_as_float(sr[g * CC + 2 * hh]) + __uint_as_float(sr[g * CC + 2 * hh + 1]);
            t = fmaf(sk[g], s2, t);
            z = fmaf(zk[g], qz[g][hh], z);
          }
          lg[hh] = (valid && hh < nh) ? fmaf(t, F[hh], z) : -INFINITY;
        }
      }
      // ---- weights with the current maximum and exponent (optimistic)
      bool need = smax >= u_bound;
#pragma unroll
      for (int hh = 0; hh < HP; ++hh) need |= lg[hh] > m_run[hh] + kLazy;
      float p[HP];
      uint8_t* bw_row = bw + bi * C::BW_BYTES + bw_row_off;
      auto weights = [&]() {
        const float fu = pow2i(u_run);
#pragma unroll
        for (int hh = 0; hh < HP; ++hh) {
          const float mref = m_run[hh] == -INFINITY ? 0.0f : m_run[hh];
          p[hh] = exp2_approx(lg[hh] - mref);
        }
#pragma unroll
        for (int g = 0; g < NGV; ++g) {
          const float f = fu * sv[g];
          uint32_t wd[HP];  // (high, low) of each head: columns 2hh, 2hh + 1
#pragma unroll
          for (int hh = 0; hh < HP; hh += 2)
            tc_split_pair(p[hh] * f, p[hh + 1] * f, wd[hh], wd[hh + 1]);
          // columns g*CC + 2hh + {high, low}: 8 columns per 16-byte chunk
#pragma unroll
          for (int k = 0; k < CC / 8; ++k)
            *reinterpret_cast<uint4*>(bw_row + ((g * CC) / 8 + k) * 128) =
                make_uint4(wd[4 * k], wd[4 * k + 1], wd[4 * k + 2], wd[4 * k + 3]);
        }
      };
      weights();
      const bool wneed = __any_sync(0xffffffffu, need);
      if (lane == 0) votes[sq] = wneed ? 1 : 0;
      if (softmax_sync_or(to)) {
        ok = false;
        break;
      }
      if (votes[0] | votes[1] | votes[2] | votes[3]) {
        // ---- exchange: tile maxima of the scores and of the value scales
        float* rm = red;  // [warp][HP + 1]
#pragma unroll
        for (int hh = 0; hh < HP; ++hh) {
          const float mx = warp_max_all(lg[hh]);
          if (lane == 0) rm[sq * (HP + 1) + hh] = mx;
        }
        {
          const float sx = warp_max_all(smax);
          if (lane == 0) rm[sq * (HP + 1) + HP] = sx;
        }
        softmax_sync();
        float sx = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) sx = fmaxf(sx, rm[w * (HP + 1) + HP]);
#pragma unroll
        for (int hh = 0; hh < HP; ++hh) {
          float mt = -INFINITY;
#pragma unroll
          for (int w = 0; w < 4; ++w) mt = fmaxf(mt, rm[w * (HP + 1) + hh]);
          if (mt > m_run[hh] + kLazy) {
            const float alpha = m_run[hh] == -INFINITY ? 1.0f : exp2_approx(m_run[hh] - mt);
            m_run[hh] = mt;
            l_part[hh] *= alpha;
#pragma unroll
            for (int g = 0; g < NGV; ++g) z_part[g][hh] *= alpha;
            alpha_cur[hh] *= alpha;
          }
        }
        if (sx >= u_bound) {
          u_run = min(u_run, 6 - ilogbf(sx));
          u_bound = pow2i(7 - u_run);
        }
        weights();
        softmax_sync();  // everyone has read rm before it is written again
      }
#pragma unroll
      for (int hh = 0; hh < HP; ++hh) {
        l_part[hh] += p[hh];
#pragma unroll
        for (int g = 0; g < NGV; ++g) z_part[g][hh] = fmaf(p[hh], zv[g], z_part[g][hh]);
      }
      // weights in shared memory for the tensor core, scores read: hand over
      fence_proxy_async_shared();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&w_ready[bi]);
      // ---- previous tile's output product (a wait that runs out is acted
      // on at the group's next barrier)
      if (i >= 1) to = !read_back(i - 1, u_prev, alpha_prev);
#pragma unroll
      for (int hh = 0; hh < HP; ++hh) {
        alpha_prev[hh] = alpha_cur[hh];
        alpha_cur[hh] = 1.0f;
      }
      u_prev = u_run;
    }
    if (ok && !to) ok = read_back(n_tiles - 1, u_prev, alpha_prev);

    // ------------------------------------------------------------ epilogue
    // sums of the weights and of the zero terms over all positions
    float* rl = red;             // [warp][HP]
    float* rz = red + 4 * HP;    // [warp][NGV][HP]
    softmax_sync();
#pragma unroll
    for (int hh = 0; hh < HP; ++hh) {
      const float ls = warp_sum_all(l_part[hh]);
      if (lane == 0) rl[sq * HP + hh] = ls;
#pragma unroll
      for (int g = 0; g < NGV; ++g) {
        const float zs = warp_sum_all(z_part[g][hh]);
        if (lane == 0) rz[(sq * NGV + g) * HP + hh] = zs;
      }
    }
    softmax_sync();
#pragma unroll
    for (int hh = 0; hh < HP; ++hh) {
      if (hh >= nh) break;
      float L = 0.0f, Z = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        L += rl[w * HP + hh];
        Z += rz[(w * NGV + gv_me) * HP + hh];
      }
      const float o = (o_acc[hh] + Z) * __frcp_rn(L);
      const size_t row = static_cast<size_t>(b) * a.q_heads + head0 + hh;
      if (a.direct) {
        store_out(a.out, a.out_dtype, row * D + d_me, o);
      } else {
        a.ws_o[(row * a.num_splits + split) * D + d_me] = o;
        if (s_tid == 0) a.ws_lse[row * a.num_splits + split] = m_run[hh] + __log2f(L);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::dealloc(tbase, C::TM_COLS);
}

template <class C>
cudaError_t launch_decode_tc(const DecodeArgs& a, dim3 grid, cudaStream_t stream) {
  return launch_pdl(decode_tc_kernel<C>, grid, dim3(C::kThreads), C::SMEM_BYTES, stream, a);
}

template <class C>
DecodeKernel make_decode_tc_kernel() {
  DecodeKernel k;
  k.fn = reinterpret_cast<const void*>(&decode_tc_kernel<C>);
  k.fn_fused = nullptr;
  k.threads = C::kThreads;
  k.smem_bytes = C::SMEM_BYTES;
  k.launch = &launch_decode_tc<C>;
  k.launch_fused = nullptr;
  k.tile = C::TILE;
  k.max_per_sm = 1;  // all 512 tensor-memory columns of the SM
  k.stage_tokens = 0;
  return k;
}

// Instances for one (bits_k, bits_v) pair at head_dim 128: the key/value
// group pairs of the cache format and 4 or 8 heads per CTA.
template <int BK, int BV>
bool get_decode_tc_kernel_bits(int groups_k, int groups_v, int heads_per_cta, DecodeKernel* out) {
#define KVQ_TC(NGK, NGV)                                                             \
  if (groups_k == NGK && groups_v == NGV) {                                          \
    *out = heads_per_cta <= 4 ? make_decode_tc_kernel<TcCfg<BK, BV, NGK, NGV, 4>>()  \
                              : make_decode_tc_kernel<TcCfg<BK, BV, NGK, NGV, 8>>(); \
    return true;                                                                     \
  }
  KVQ_TC(1, 1)
  KVQ_TC(2, 2)
  KVQ_TC(4, 4)
  KVQ_TC(2, 1)
  KVQ_TC(4, 2)
  KVQ_TC(4, 1)
#undef KVQ_TC
  return false;
}

}  // namespace kvq
