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
//  * each of the CTA's four warps runs its own copy pipeline: lane 0 streams
//    the warp's next 32 positions of the four cache arrays into a ring of
//    two shared-memory slots with 1-D bulk copies (cp.async.bulk, no
//    multicast) counted on the warp's own mbarriers (bounded waits), and the
//    warp processes its two 16-token tiles phase by phase;
//  * keys and values may have different group sizes (NGK, NGV groups per
//    row): the score side uses the key groups, the output side the value
//    groups;
//  * codes stay integers: every code becomes an exact binary16 subnormal
//    (code * 2^(pos-24)) with one AND, so tensor cores (mma.sync m16n8k16,
//    fp32 accumulate) multiply raw codes; the per-group scale and zero are
//    applied afterwards:  q.k^ = sum_g scale_g (q . c_g) + zero_g sum_{d in g} q_d
//    and  o = sum_t (p_t scale_t) c_t + sum_t p_t zero_t;
//  * the query rows of each span are bulk-copied into one of two shared
//    buffers (the next span's while the current one runs);
//  * the query (B operand of the score product) is scaled by a power of two
//    and split into binary16 high and low parts in two columns (the low part
//    is zero for 16-bit queries); the weights p_t * scale_t (B operand of the
//    output product) are split the same way and scaled per warp by a power of
//    two, so products keep ~22 bits;
//  * online softmax in binary32 (exp2 domain) with a lazily updated maximum;
//    partial results per split are merged by a separate log-sum-exp combine,
//    except when a row has a single split: its CTA then writes the output;
//  * the default grid is one CTA per split; the opt-in balanced schedule
//    (one wave, several spans per CTA) keeps each warp's copy ring running
//    across spans (see decode_kernel);
//  * with rotated keys (KVQ_FLAG_ROTATE_KEYS) the prologue turns the query
//    into H q / D in shared memory;
//  * paged layout (KVQ_FLAG_PAGED): a stage's 32 positions lie in one page;
//    lane 0 looks the page up in the block table one stage ahead;
//  * the FUSED instances (kvq_append_decode_attention) first quantize and
//    write the step's new positions that fall in the CTA's split (see
//    append_rows.cuh), then stream as above.
#pragma once

#include <type_traits>

#include "append_rows.cuh"
#include "common.cuh"
#include "internal.h"

namespace kvq {

// QS == 2: each lane's two score columns are the high and low parts of one
// head (up to 4 heads per n-tile); QS == 1: two heads (up to 8 per n-tile).
// NGK / NGV: groups per row of the keys / values (separate group sizes).
template <int D_, int BK_, int BV_, int NGK_, int NGV_, int QS_, int NQ_, int NP_>
struct DecodeCfg {
  static constexpr int D = D_, BK = BK_, BV = BV_, QS = QS_, NQ = NQ_, NP = NP_;
  static constexpr int NGK = NGK_, NGV = NGV_;
  static constexpr int kWarps = 4;  // warps per CTA; each runs its own copy pipeline
  // CTAs per SM the registers must allow: four for up to four heads per CTA,
  // three for 5..8 heads with 16-bit queries (two with 32-element key
  // groups), two with binary32 queries
  static constexpr int kMinBlocks = NP_ == 1 ? 4 : (QS_ == 1 && NGK_ < 4) ? 3 : 2;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int TPW = 2;     // 16-token tiles per warp per stage
  static constexpr int kStageTokens = 16 * TPW * kWarps;
  static constexpr int GK = D / NGK, GV = D / NGV;
  static constexpr int KSTEPS = D / 16;  // k-steps (scores) == m-tiles (output)
  static constexpr int KROW = D * BK / 8;
  static constexpr int KSLICE = D * BK / 32;  // bytes of one lane's K slice
  static constexpr int KW = KSLICE / 4;
  static constexpr int VTILE = 2 * D * BV;
  static constexpr int VN = D * BV / 16;  // bytes per lane per V tile
  static constexpr int VP = VN < 16 ? VN : 16;
  static constexpr int VW = VN / 4;
  static constexpr int WV = D * BV / 128;  // V words per half-lane
  static constexpr int PROWK = NGK * 4, PROWV = NGV * 4;  // parameter bytes per position
  // one slot = one warp's 16*TPW positions of a stage: K rows, V tiles, K params, V params
  static constexpr int SLOT_K = 16 * TPW * KROW;
  static constexpr int SLOT_V = TPW * VTILE;
  static constexpr int SLOT_PK = 16 * TPW * PROWK, SLOT_PV = 16 * TPW * PROWV;
  static constexpr int SLOT_BYTES = SLOT_K + SLOT_V + SLOT_PK + SLOT_PV;
  // Copies in flight per warp.  Two slots measured as fast as three or four
  // on every workload shape (graph replay on B200), with a third less
  // shared memory.
  static constexpr int kSlots = 2;
  static constexpr int RING_BYTES = kWarps * kSlots * SLOT_BYTES;
  // staged output weights: per warp and tile [group][head][part][WB_RS halves]
  static constexpr int WB_RS = 24;  // halves per row: 16 positions + pad (conflict-free)
  static constexpr int WB_HALVES = NGV * 8 * 2 * WB_RS;
  static constexpr int WB_BYTES = TPW * kWarps * WB_HALVES * 2;
  // the warps' partial outputs at the end of a span, [warp][head][D] binary32,
  // share the staging buffer's region (the ring keeps receiving the next
  // span's copies meanwhile)
  static constexpr int OB_HEADS = 4 * NP;
  static constexpr int OB_BYTES = kWarps * OB_HEADS * D * 4;
  static constexpr int STAGE_BYTES = WB_BYTES > OB_BYTES ? WB_BYTES : OB_BYTES;
  // query rows of a span ([head][D] in the query type, binary32 at most),
  // two buffers: the next span's rows arrive while this span runs
  static constexpr int QBUF_BYTES = OB_HEADS * D * 4;
  static constexpr int ALPHA_FLOATS = kWarps * 8;
  static constexpr int MERGE_FLOATS = kWarps * 8 * (2 + NGV) + 2 * 8 * (kWarps + 1);
  static constexpr int QBUF_OFF = RING_BYTES + STAGE_BYTES;
  static constexpr int ALPHA_OFF = QBUF_OFF + 2 * QBUF_BYTES;
  // mbarriers: [warp][slot] copy slots, then the two query buffers; then
  // the CTA's span counter and query flag (4 ints) and each warp's view of
  // the next span (4 ints per warp)
  static constexpr int BAR_OFF = ALPHA_OFF + 4 * (ALPHA_FLOATS + MERGE_FLOATS);
  static constexpr int CTL_OFF = BAR_OFF + 8 * (kWarps * kSlots + 2);
  // + the balanced schedule's row table: lengths (kStreamRows ints) and the
  // prefix sums of the rows' stages (kStreamRows + 1 ints)
  static constexpr int SMEM_BYTES = CTL_OFF + 16 + 16 * kWarps + 4 * (2 * kStreamRows + 1);
  static constexpr int HT = QS == 1 ? 2 * NQ : NQ;  // score head slots per lane
  static_assert(kThreads == 128, "the stream schedule's scan runs on 128 threads");
  static_assert(WB_BYTES >= 8 * D * 4, "rotated queries must fit in the staging buffer");
  // fused append: rows whose inputs one warp loads before quantizing them,
  // and its shared scratch (one binary32 row and one row of codes)
  static constexpr int APPEND_BATCH = 4;
  static constexpr int APPEND_SCRATCH = 5 * D;
  static_assert(WB_BYTES >= kWarps * APPEND_SCRATCH, "append scratch must fit in the staging buffer");
  static_assert(SLOT_BYTES % 16 == 0 && SLOT_K % 16 == 0 && SLOT_V % 16 == 0, "alignment");
  static_assert(QBUF_OFF % 16 == 0 && QBUF_BYTES % 16 == 0 && BAR_OFF % 8 == 0, "alignment");
  static_assert(GK >= 16 && GK % 16 == 0 && GV >= 16 && GV % 16 == 0,
                "groups must cover whole 16-element steps");
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

// (scale_a, scale_b) and (zero_a, zero_b) of two (scale, zero) binary16 pairs.
__device__ __forceinline__ float2 scales_of(uint32_t a, uint32_t b) {
  return unpack_half2(__byte_perm(a, b, 0x5410));
}
__device__ __forceinline__ float2 zeros_of(uint32_t a, uint32_t b) {
  return unpack_half2(__byte_perm(a, b, 0x7632));
}

// D = A * B (C = 0), m16n8k16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816_zc(float d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                 uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// Shared-memory 8x8 b16 matrix stores and transposed loads (N = 2 or 4
// matrices; each lane addresses one 16-byte row: matrix lane/8, row lane%8).
template <int N>
__device__ __forceinline__ void stmatrix_b16(void* p, const uint32_t* r) {
  if constexpr (N == 4)
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(p)),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
  else
    asm volatile("stmatrix.sync.aligned.m8n8.x2.shared.b16 [%0], {%1, %2};" ::"r"(smem_addr(p)), "r"(r[0]),
                 "r"(r[1])
                 : "memory");
}
template <int N>
__device__ __forceinline__ void ldmatrix_trans_b16(const void* p, uint32_t* d) {
  if constexpr (N == 4)
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(smem_addr(p))
                 : "memory");
  else
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(d[0]), "=r"(d[1])
                 : "r"(smem_addr(p))
                 : "memory");
}

// (scale, zero) words of two consecutive positions (N groups each).
template <int N>
__device__ __forceinline__ void lds_param_pair(const uint32_t* p, uint32_t (&w0)[N], uint32_t (&w1)[N]) {
  if constexpr (N == 1) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    w0[0] = u.x;
    w1[0] = u.y;
  } else if constexpr (N == 2) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    w0[0] = u.x; w0[1] = u.y;
    w1[0] = u.z; w1[1] = u.w;
  } else {
    static_assert(N == 4, "groups per row");
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint4 v = *reinterpret_cast<const uint4*>(p + 4);
    w0[0] = u.x; w0[1] = u.y; w0[2] = u.z; w0[3] = u.w;
    w1[0] = v.x; w1[1] = v.y; w1[2] = v.z; w1[3] = v.w;
  }
}

// Paged layout or slot layout: fixed at compile time in the plain instances;
// tested at run time in the fused ones, whose append prologue keeps its
// registers and schedule best that way (measured: the Qwen-shaped fused step
// took 77 us with the layout fixed at compile time against 65 us).
template <bool FUSED, bool PAGED>
__device__ __forceinline__ bool paged_layout(const DecodeArgs& a) {
  if constexpr (FUSED)
    return a.block_table != nullptr;
  else
    return PAGED;
}

// One span of a CTA's work: positions [t0, t1) of (batch row b, kv head hk,
// head group hg); app_pos: first position the fused append writes (-1:
// none); the result is the rows' final output (direct) or the partial result
// at index ws_index of the rows' partial slots.
struct Span {
  int b, hk, hg, t0, t1, app_pos, ws_index;
  bool direct;
};

// Bulk copy of span s's query rows (heads head0 .. head0 + nh - 1 of row
// b, [head][D] in the query type) into a query buffer; thread 0 only.  The
// rows are contiguous, start on a multiple of 128 bytes from the query base
// (16-byte aligned, as the API requires) and are whole 16-byte units.
template <class C>
__device__ __forceinline__ void issue_q_rows(const DecodeArgs& a, const Span& s, uint8_t* dst,
                                             uint64_t* bar) {
  const int head0 = s.hk * a.gq + s.hg * a.heads_per_cta;
  const int nh = min(a.heads_per_cta, a.gq - s.hg * a.heads_per_cta);
  const int es = a.q_dtype == KVQ_F32 ? 4 : 2;
  const uint32_t bytes = static_cast<uint32_t>(nh * C::D * es);
  mbar_arrive_expect_tx(bar, bytes);
  bulk_copy_g2s(dst,
                static_cast<const uint8_t*>(a.q) +
                    (static_cast<size_t>(s.b) * a.q_heads + head0) * C::D * es,
                bytes, bar);
}

// FUSED: the instance used by the fused append + decode call (the append
// prologue is compiled only there, so the plain decode keeps its registers
// and schedule).  PAGED: the instance for the paged layout (block-table
// lookups); the slot layout's instances are compiled without them (their
// per-stage checks cost 3 % of the steady-state decode).
// One span cur: the copy pipeline, the online softmax and the four warps'
// merge.  Each warp's copies form one stream over the CTA's spans: stage g of
// the stream lands in slot g mod kSlots with phase parity (g / kSlots) mod 2.
// g0: stages of this warp's stream before cur (advanced by cur's stages);
// pre: cur's stages already issued by the previous span (replaced by the
// next span's; meaningful in lane 0, which issues).  peek(s) gives the CTA's
// next span (false: none) and next(s) moves on to it.  The next span's
// query rows go out at cur's start (query buffer (qspan + 1) mod 2; cur's
// are in buffer qspan mod 2; qspan: the CTA's spans so far, kept in shared
// memory), and the slots that cur's last stages free are
// refilled with its first stages (not in the fused instance, whose append
// comes first, nor with the paged layout, whose page lookups would stall
// the warp), so that the next span starts without waiting (rotated keys
// transform their own copy of the rows instead).
// Returns true when a wait ran out (the CTA then stops; the rows are
// flagged).
template <class C, bool FUSED, bool PAGED, class PeekFn, class NextFn>
__device__ __forceinline__ bool decode_span(const DecodeArgs& a, uint8_t* smem, const Span& cur,
                                            PeekFn&& peek, NextFn&& next, Span& nxt,
                                            bool& has_next, int ws_stride, int& g0, int& pre) {
  constexpr int D = C::D, NGK = C::NGK, NGV = C::NGV, NQ = C::NQ, NP = C::NP, QS = C::QS;
  constexpr int HT = C::HT, KSTEPS = C::KSTEPS, GK = C::GK, GV = C::GV;
  uint16_t* wbuf = reinterpret_cast<uint16_t*>(smem + C::RING_BYTES);  // staged weights
  float* alph = reinterpret_cast<float*>(smem + C::ALPHA_OFF);          // [warp][8]
  float* mrg = alph + C::ALPHA_FLOATS;                                  // merge area
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);      // [warp][slot]
  uint64_t* qfull = full + C::kWarps * C::kSlots;                       // [query buffer]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* wfull = full + warp * C::kSlots;
  const int b = cur.b, hk = cur.hk, hg = cur.hg, t0 = cur.t0, t1 = cur.t1;
  const int app_pos = cur.app_pos, ws_index = cur.ws_index;
  const bool direct = cur.direct;
  const int head0 = hk * a.gq + hg * a.heads_per_cta;
  const int nh = min(a.heads_per_cta, a.gq - hg * a.heads_per_cta);
  const int n_tok = t1 - t0;
  const size_t slot = static_cast<size_t>(b) * a.kv_heads + hk;
  const bool paged = paged_layout<FUSED, PAGED>(a);

  // ---- this warp's copy pipeline: positions [it*kStageTokens + 16*TPW*warp, +16*TPW)
  // of a span for it = 0 .. iters-1, kSlots copies in flight.
  const int my_first = warp * 16 * C::TPW;
  auto iters_of = [&](const Span& s) {
    const int n = s.t1 - s.t0;
    return n > my_first ? (n - my_first + C::kStageTokens - 1) / C::kStageTokens : 0;
  };
  const int my_iters = iters_of(cur);
  uint8_t* wring = smem + warp * C::kSlots * C::SLOT_BYTES;
  // A stage's 16*TPW positions start at a multiple of 16*TPW, so they never
  // span two pages of the paged layout (pages hold a power of two >= 32).
  static_assert(32 % (16 * C::TPW) == 0, "a stage must fit in the smallest page");
  // Position tb of this slot (the first of a stage).  Slot layout: row
  // slot * capacity + tb of the per-position arrays.  Paged layout: its page
  // (block-table entry, looked up ahead by page_of) and the row inside
  // (page, kv head); a page outside the pool is never read.
  auto page_of = [&](const Span& s, int it) -> int {
    const int tb = s.t0 + it * C::kStageTokens + my_first;
    return a.block_table[static_cast<size_t>(s.b) * a.pages_per_seq + (tb >> a.page_shift)];
  };
  auto issue = [&](const Span& s, int it, int sl, int page) {
    const int base = it * C::kStageTokens + my_first;  // multiple of 16
    const int n16 = (min(16 * C::TPW, s.t1 - s.t0 - base) + 15) & ~15;
    const int tb = s.t0 + base;
    uint8_t* dst = wring + sl * C::SLOT_BYTES;
    size_t r = (static_cast<size_t>(s.b) * a.kv_heads + s.hk) * a.capacity + tb;
    if (paged) {
      if (page < 0 || page >= a.num_pages) {
        // no page: nothing is read (the row's output is unspecified); the
        // stage completes at once so that the pipeline keeps going
        flag_error(a.err, KVQ_DEVERR_BAD_PAGE);
        mbar_arrive_expect_tx(&wfull[sl], 0);
        return;
      }
      const int local = tb & ((1 << a.page_shift) - 1);
      r = ((static_cast<size_t>(page) * a.kv_heads + s.hk) << a.page_shift) + local;
    }
    const uint32_t kbytes = n16 * C::KROW, vbytes = (n16 / 16) * C::VTILE;
    const uint32_t pkbytes = n16 * C::PROWK, pvbytes = n16 * C::PROWV;
    mbar_arrive_expect_tx(&wfull[sl], kbytes + vbytes + pkbytes + pvbytes);
    bulk_copy_g2s(dst, a.k_codes + r * C::KROW, kbytes, &wfull[sl]);
    bulk_copy_g2s(dst + C::SLOT_K, a.v_codes + (r / 16) * C::VTILE, vbytes, &wfull[sl]);
    bulk_copy_g2s(dst + C::SLOT_K + C::SLOT_V,
                  reinterpret_cast<const uint8_t*>(a.k_params) + r * C::PROWK, pkbytes,
                  &wfull[sl]);
    bulk_copy_g2s(dst + C::SLOT_K + C::SLOT_V + C::SLOT_PK,
                  reinterpret_cast<const uint8_t*>(a.v_params) + r * C::PROWV, pvbytes,
                  &wfull[sl]);
  };
  int issued = pre;  // stages of the stream from g0 on that are in flight or consumed
  // Test knob (kvq_debug_inject_wait_timeout): stage `fault_stage` (0 or 1)
  // of the first warp's stream in the first CTA expects 16 bytes more than
  // its copies bring, so that the wait on it runs out.  Checked only where
  // the first stages are requested, never in the main loop.
  auto knob = [&](int stream_stage, int sl) {
    if (stream_stage == a.fault_stage && warp == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&
        blockIdx.z == 0)
      mbar_expect_tx(&wfull[sl], 16);
  };
  // the next span's query rows
  const bool q_bulk = !a.rotate_q;
  uint8_t* qbuf = smem + C::QBUF_OFF;
  // ctl[0]: spans begun before cur; ctl[1]: the next span's rows are in
  // flight; ctl[2]: a query wait ran out (the CTA stops after this span)
  int* ctl = reinterpret_cast<int*>(smem + C::CTL_OFF);
  if (q_bulk && threadIdx.x == 0) {
    Span s;
    const int qs = ctl[0];
    ctl[1] = 0;
    if (peek(s)) {
      issue_q_rows<C>(a, s, qbuf + ((qs + 1) & 1) * C::QBUF_BYTES, &qfull[(qs + 1) & 1]);
      ctl[1] = 1;
    }
  }
  // this warp's view of the next span for the refills at cur's end (b, hk,
  // t0, t1; b < 0: none), kept in shared memory rather than registers (read
  // through a volatile pointer, so that the reads stay where they are used)
  volatile int* wnext = ctl + 4 + 4 * warp;
  if (!FUSED && !paged && lane == 0) {
    Span s;
    const bool any = peek(s);
    wnext[0] = any ? s.b : -1;
    wnext[1] = s.hk;
    wnext[2] = s.t0;
    wnext[3] = s.t1;
  }
  // The fused append's input rows are requested into L2 before anything
  // else, so that the append's loads below find them there.
  if (FUSED && app_pos >= 0 && threadIdx.x == 0) {
    const int p0 = max(app_pos, t0);
    if (p0 < t1) {
      const int es = a.in_dtype == KVQ_F32 ? 4 : 2;
      const size_t row0 = slot * a.n_new + (p0 - app_pos);
      const uint32_t bytes = static_cast<uint32_t>((t1 - p0) * D * es);
      bulk_prefetch_l2(static_cast<const uint8_t*>(a.k_new) + row0 * D * es, bytes);
      bulk_prefetch_l2(static_cast<const uint8_t*>(a.v_new) + row0 * D * es, bytes);
    }
  }
  // First stages (those the previous span has not issued).  With a fused
  // append, the stages that end before the new positions go out first, so
  // that their copies overlap the append.
  int first_pending = min(C::kSlots, my_iters);
  if (lane == 0) {
    if constexpr (FUSED) {
      for (int it = 0; it < min(C::kSlots, my_iters); ++it) {
        if (app_pos >= 0 && t0 + it * C::kStageTokens + my_first + 16 * C::TPW > app_pos) {
          first_pending = it;
          break;
        }
        knob(g0 + it, (g0 + it) % C::kSlots);
        issue(cur, it, (g0 + it) % C::kSlots, paged ? page_of(cur, it) : 0);
      }
    } else {
      for (; issued < min(C::kSlots, my_iters); ++issued) {
        knob(g0 + issued, (g0 + issued) % C::kSlots);
        issue(cur, issued, (g0 + issued) % C::kSlots,
              paged ? page_of(cur, issued) : 0);
      }
    }
  }
  if constexpr (FUSED) {
    // ---- fused append of the new positions in this split (every head-group
    // CTA of the slot writes the same bytes), made visible to the bulk
    // copies of the remaining stages before they are issued.  Scratch: the
    // weight staging buffer, unused until the first tile.
    if (app_pos >= 0) {
      const int p0 = max(app_pos, t0), p1 = t1;
      if (p0 < p1) {
        auto row_of_pos = [&](int p) -> long long {
          if (!paged) return static_cast<long long>(slot) * a.capacity + p;
          const int page =
              a.block_table[static_cast<size_t>(b) * a.pages_per_seq + (p >> a.page_shift)];
          if (page < 0 || page >= a.num_pages) return -1;
          return ((static_cast<long long>(page) * a.kv_heads + hk) << a.page_shift) +
                 (p & ((1 << a.page_shift) - 1));
        };
        append_rows<C>(a, b, hk, app_pos, p0, p1,
                       reinterpret_cast<uint8_t*>(wbuf) + warp * C::APPEND_SCRATCH, row_of_pos);
        fence_proxy_async_global();
        __syncthreads();
        fence_proxy_async_global();
      }
    }
    if (lane == 0)
      for (int it = first_pending; it < min(C::kSlots, my_iters); ++it) {
        knob(g0 + it, (g0 + it) % C::kSlots);
        issue(cur, it, (g0 + it) % C::kSlots, paged ? page_of(cur, it) : 0);
      }
    issued = min(C::kSlots, my_iters);
  }
  __syncwarp();

  // ------------------------------------------------------------ consumers
  const int g = lane >> 2, c = lane & 3;
  bool timed_out = false;
  int consumed = 0;  // stages of cur this warp has consumed
  float m_run[HT], l_run[HT];
  float oacc[KSTEPS][NP][4];
  float2 zacc[HT][NGV];  // zero term, score layout: (row g, row g+8) partials
  // Power-of-two exponent applied to the output weights p * scale_v so that
  // their binary16 parts stay normal; only ever decreases (see below).
  int u_run = 100;
  float u_bound = pow2i(7 - 100);  // value scales below this keep the weights < 2^15
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
  for (int hs = 0; hs < HT; ++hs)
#pragma unroll
    for (int gr = 0; gr < NGV; ++gr) zacc[hs][gr] = make_float2(0.0f, 0.0f);

  {
    // -------- query fragments (B operand of the score product), once per span
    // With rotated keys (KVQ_FLAG_ROTATE_KEYS) the query becomes H q / D: the
    // CTA's query rows are transformed in shared memory first (the weight
    // staging buffer is unused until the first tile).
    const float* qrot = nullptr;
    if (a.rotate_q) {
      float* qs = reinterpret_cast<float*>(wbuf);  // [head][D]
      for (int i = threadIdx.x; i < nh * D; i += C::kThreads)
        qs[i] = load_elem(a.q, a.q_dtype,
                          (static_cast<size_t>(b) * a.q_heads + head0 + i / D) * D + i % D);
      __syncthreads();
#pragma unroll 1
      for (int h = 1; h < D; h *= 2) {
        for (int i = threadIdx.x; i < nh * D / 2; i += C::kThreads) {
          const int r = i % (D / 2);
          float* x = qs + (i / (D / 2)) * D + (r / h) * 2 * h + (r % h);
          const float x0 = x[0], x1 = x[h];
          x[0] = x0 + x1;
          x[h] = x0 - x1;
        }
        __syncthreads();
      }
      qrot = qs;
    }
    // the query buffer, or the rotated rows
    const int qs = ctl[0];
    uint8_t* qcur = qbuf + (qs & 1) * C::QBUF_BYTES;
    if (q_bulk) {
      // (a wait that runs out is flagged, noted in ctl[2], and stops the
      // CTA at the span's end; the span runs on meanwhile)
      if (!mbar_wait_bounded(&qfull[qs & 1], (qs >> 1) & 1, a.err, a.wait_limit_ns))
        ctl[2] = 1;
    }
    float qraw[NQ][KSTEPS][4];
    float amax = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NQ; ++nt) {
      const int n = 8 * nt + g;
      const int head = QS == 2 ? n / 2 : n;
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float2 v;
          if (qrot != nullptr) {
            // elements d, d+1 with d = 16j + 2c + 8r
            constexpr float kInvD = 1.0f / D;  // exact: D is a power of two
            const float* x = qrot + head * D + 16 * j + 2 * c + 8 * r;
            const bool in = head < nh;
            v = in ? make_float2(x[0] * kInvD, x[1] * kInvD) : make_float2(0.0f, 0.0f);
          } else {
            // elements d, d+1 with d = 16j + 2c + 8r of this head's row
            const int d = head * D + 16 * j + 2 * c + 8 * r;
            const bool in = head < nh;
            uint32_t u = 0u, u1 = 0u;
            if (a.q_dtype == KVQ_F32) {
              const uint2 w = in ? *reinterpret_cast<const uint2*>(qcur + 4 * d) : make_uint2(0u, 0u);
              u = w.x;
              u1 = w.y;
            } else {
              u = in ? *reinterpret_cast<const uint32_t*>(qcur + 2 * d) : 0u;
            }
            v = a.q_dtype == KVQ_F32
                    ? make_float2(__uint_as_float(u), __uint_as_float(u1))
                : a.q_dtype == KVQ_BF16
                    ? make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u))
                    : unpack_half2(u);
          }
          qraw[nt][j][2 * r] = v.x;
          qraw[nt][j][2 * r + 1] = v.y;
          amax = fmaxf(amax, fmaxf(fabsf(qraw[nt][j][2 * r]), fabsf(qraw[nt][j][2 * r + 1])));
        }
    }
    if (qrot != nullptr) __syncthreads();  // every warp has read qs before any stages weights
    amax = warp_max_xor(amax, 1);
    const int eq = amax > 0.0f ? max(-100, min(100, 14 - ilogbf(amax))) : 0;
    uint32_t bq[NQ][KSTEPS][2];
#pragma unroll
    for (int nt = 0; nt < NQ; ++nt) {
      const bool lo_col = QS == 2 && (g & 1);
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int e = (2 * j + r) % (16 / C::BK);
          const float f = pow2i(eq - field_pos<C::BK>(e));
          const float v0 = qraw[nt][j][2 * r] * f, v1 = qraw[nt][j][2 * r + 1] * f;
          const uint32_t hi = f2_to_h2(v0, v1);
          const float2 h = unpack_half2(hi);
          const uint32_t lo = f2_to_h2(v0 - h.x, v1 - h.y);
          bq[nt][j][r] = lo_col ? lo : hi;
        }
    }
    // Sum of q over each group, in the same units as the code products (the
    // score product of an all-ones code matrix), times the softmax scale.
    // qz[gr][nt] = {col 2c, col 2c+1}; for QS == 2 both columns of a lane
    // belong to one head and are summed.
    const float F = a.sm_scale_log2 * pow2i(24 - eq);
    float2 qz[NGK][NQ];
    {
      float qsum[NGK][NQ][4];
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j) {
        const int gr = 16 * j / GK;
        const uint32_t one0 = 0x00010001u << field_pos<C::BK>((2 * j) % (16 / C::BK));
        const uint32_t one1 = 0x00010001u << field_pos<C::BK>((2 * j + 1) % (16 / C::BK));
#pragma unroll
        for (int nt = 0; nt < NQ; ++nt) {
          if (j % (GK / 16) == 0)
            mma_f16_16816_zc(qsum[gr][nt], one0, one0, one1, one1, bq[nt][j][0], bq[nt][j][1]);
          else
            mma_f16_16816(qsum[gr][nt], one0, one0, one1, one1, bq[nt][j][0], bq[nt][j][1]);
        }
      }
#pragma unroll
      for (int gr = 0; gr < NGK; ++gr)
#pragma unroll
        for (int nt = 0; nt < NQ; ++nt)
          qz[gr][nt] = QS == 2 ? make_float2((qsum[gr][nt][0] + qsum[gr][nt][1]) * F, 0.0f)
                               : make_float2(qsum[gr][nt][0] * F, qsum[gr][nt][1] * F);
    }

    // ------------------------------------------------------ main loop
    // Softmax reference: m_run[hs] may lag the true running maximum by up to
    // kLazy (log2 units), so weights p = 2^(logit - m_run) stay <= 2^kLazy;
    // only a score above m_run + kLazy triggers the warp-wide maximum and
    // the rescale of the accumulators.
    constexpr float kLazy = 8.0f;
    constexpr int TPW = C::TPW;
    uint16_t* wb = wbuf + warp * TPW * C::WB_HALVES;
    float* walph = alph + warp * 8;
    // lane offsets inside a stage (tile tt of this warp adds tt * 16 rows)
    const int k_off = g * C::KROW + c * C::KSLICE;
    const int v_off = C::SLOT_K + lane * C::VP;
    const int kp_off = C::SLOT_K + C::SLOT_V + g * C::PROWK;
    const int vp_off = C::SLOT_K + C::SLOT_V + C::SLOT_PK + g * C::PROWV;
    uint32_t* const err = a.err;

    // Process NTL consecutive tiles of this warp (tile indices t_first ..),
    // phase by phase so that their dependency chains interleave.  FULL:
    // every position valid; otherwise a single tile with nvalid positions.
    auto tiles_step = [&](auto full_tag, auto ntl_tag, const uint8_t* st, int t_first, int nvalid) {
      constexpr bool FULL = decltype(full_tag)::value;
      constexpr int NTL = decltype(ntl_tag)::value;
      uint32_t kw[NTL][2 * C::KW];
      uint32_t kpa[NTL][NGK], kpb[NTL][NGK], vpa[NTL][NGV], vpb[NTL][NGV];
#pragma unroll
      for (int tt = 0; tt < NTL; ++tt) {
        const int tix = t_first + tt;
        lds_words<C::KSLICE>(st + k_off + tix * 16 * C::KROW, kw[tt], 0);
        lds_words<C::KSLICE>(st + k_off + (tix * 16 + 8) * C::KROW, kw[tt], C::KW);
        // (scale, zero) words of rows g and g+8: one vector load per row
        const uint8_t* kp = st + kp_off + tix * 16 * C::PROWK;
        const uint8_t* vp = st + vp_off + tix * 16 * C::PROWV;
        lds_words<C::PROWK>(kp, kpa[tt], 0);
        lds_words<C::PROWK>(kp + 8 * C::PROWK, kpb[tt], 0);
        lds_words<C::PROWV>(vp, vpa[tt], 0);
        lds_words<C::PROWV>(vp + 8 * C::PROWV, vpb[tt], 0);
      }
      // ---- scores: S^T[token][col] = codes . q'
      float acc[NTL][NGK][NQ][4];
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j) {
        const int gr = 16 * j / GK;
#pragma unroll
        for (int tt = 0; tt < NTL; ++tt) {
          const uint32_t a0 = extract_codes<C::BK>(kw[tt], 0, 2 * j);
          const uint32_t a1 = extract_codes<C::BK>(kw[tt], C::KW, 2 * j);
          const uint32_t a2 = extract_codes<C::BK>(kw[tt], 0, 2 * j + 1);
          const uint32_t a3 = extract_codes<C::BK>(kw[tt], C::KW, 2 * j + 1);
#pragma unroll
          for (int nt = 0; nt < NQ; ++nt) {
            if (j % (GK / 16) == 0)
              mma_f16_16816_zc(acc[tt][gr][nt], a0, a1, a2, a3, bq[nt][j][0], bq[nt][j][1]);
            else
              mma_f16_16816(acc[tt][gr][nt], a0, a1, a2, a3, bq[nt][j][0], bq[nt][j][1]);
          }
        }
      }
      // logits (log2 units) lg[tt][hs][row]: F * sum_g (scale_g acc_g + zero_g qsum_g)
      float lg[NTL][HT][2];
#pragma unroll
      for (int tt = 0; tt < NTL; ++tt) {
        if constexpr (QS == 2) {
#pragma unroll
          for (int nt = 0; nt < NQ; ++nt) {
            float2 t = make_float2(0.0f, 0.0f), z = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int gr = 0; gr < NGK; ++gr) {
              // rows (g, g+8): high + low columns
              const float2 sum = __fadd2_rn(make_float2(acc[tt][gr][nt][0], acc[tt][gr][nt][2]),
                                            make_float2(acc[tt][gr][nt][1], acc[tt][gr][nt][3]));
              t = __ffma2_rn(scales_of(kpa[tt][gr], kpb[tt][gr]), sum, t);
              z = __ffma2_rn(zeros_of(kpa[tt][gr], kpb[tt][gr]),
                             make_float2(qz[gr][nt].x, qz[gr][nt].x), z);
            }
            const float2 l2 = __ffma2_rn(t, make_float2(F, F), z);
            lg[tt][nt][0] = l2.x;
            lg[tt][nt][1] = l2.y;
          }
        } else {
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
#pragma unroll
            for (int nt = 0; nt < NQ; ++nt) {
              float2 t = make_float2(0.0f, 0.0f), z = make_float2(0.0f, 0.0f);
#pragma unroll
              for (int gr = 0; gr < NGK; ++gr) {
                const float2 sz = unpack_half2(rr ? kpb[tt][gr] : kpa[tt][gr]);
                t = __ffma2_rn(make_float2(sz.x, sz.x),
                               make_float2(acc[tt][gr][nt][2 * rr], acc[tt][gr][nt][2 * rr + 1]), t);
                z = __ffma2_rn(make_float2(sz.y, sz.y), qz[gr][nt], z);
              }
              const float2 l2 = __ffma2_rn(t, make_float2(F, F), z);
              lg[tt][2 * nt][rr] = l2.x;
              lg[tt][2 * nt + 1][rr] = l2.y;
            }
          }
        }
      }
      if (!FULL) {
        // positions past the end: no score, and scale = zero = 0 for values
#pragma unroll
        for (int hs = 0; hs < HT; ++hs) {
          if (g >= nvalid) lg[0][hs][0] = -INFINITY;
          if (g + 8 >= nvalid) lg[0][hs][1] = -INFINITY;
        }
#pragma unroll
        for (int gr = 0; gr < NGV; ++gr) {
          if (g >= nvalid) vpa[0][gr] = 0u;
          if (g + 8 >= nvalid) vpb[0][gr] = 0u;
        }
      }

      // ---- lazy online softmax (exp2 domain)
      float lmax[HT];
#pragma unroll
      for (int hs = 0; hs < HT; ++hs) {
        lmax[hs] = fmaxf(lg[0][hs][0], lg[0][hs][1]);
#pragma unroll
        for (int tt = 1; tt < NTL; ++tt) lmax[hs] = fmaxf(lmax[hs], fmaxf(lg[tt][hs][0], lg[tt][hs][1]));
      }
      bool need = false;
#pragma unroll
      for (int hs = 0; hs < HT; ++hs) need |= lmax[hs] > m_run[hs] + kLazy;
      const bool changed = __any_sync(0xffffffffu, need);
      if (changed) {
#pragma unroll
        for (int hs = 0; hs < HT; ++hs) {
          const int head = QS == 2 ? 4 * hs + c : 8 * (hs / 2) + 2 * c + (hs & 1);
          const float mt = warp_max_xor(lmax[hs], 4);
          const float mnew = fmaxf(m_run[hs], mt);
          const float alpha = mnew == -INFINITY ? 1.0f : exp2_approx(m_run[hs] - mnew);
          l_run[hs] *= alpha;
#pragma unroll
          for (int gr = 0; gr < NGV; ++gr)
            zacc[hs][gr] = __fmul2_rn(zacc[hs][gr], make_float2(alpha, alpha));
          m_run[hs] = mnew;
          if (g == 0) walph[head] = alpha;
        }
      }
      float2 pr[NTL][HT];  // weights of rows (g, g+8)
#pragma unroll
      for (int hs = 0; hs < HT; ++hs) {
        const float mref = m_run[hs] == -INFINITY ? 0.0f : m_run[hs];
#pragma unroll
        for (int tt = 0; tt < NTL; ++tt) {
          pr[tt][hs] = make_float2(exp2_approx(lg[tt][hs][0] - mref), exp2_approx(lg[tt][hs][1] - mref));
          l_run[hs] += pr[tt][hs].x + pr[tt][hs].y;
        }
      }
      // ---- exponent u of the output weights: keep p*scale*2^u < 2^15
      {
        uint32_t hm = vpa[0][0];
#pragma unroll
        for (int tt = 0; tt < NTL; ++tt)
#pragma unroll
          for (int gr = 0; gr < NGV; ++gr) {
            __half2 r = __hmax2(*reinterpret_cast<__half2*>(&hm), *reinterpret_cast<__half2*>(&vpa[tt][gr]));
            r = __hmax2(r, *reinterpret_cast<__half2*>(&vpb[tt][gr]));
            hm = *reinterpret_cast<uint32_t*>(&r);
          }
        float smax = unpack_half2(hm).x;
        if (__any_sync(0xffffffffu, smax >= u_bound)) {
          smax = warp_max_xor(smax, 4);
          const int u_need = min(u_run, 6 - ilogbf(smax));
          const float shift = pow2i(u_need - u_run);
          u_run = u_need;
          u_bound = pow2i(7 - u_run);
#pragma unroll
          for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
            for (int pt = 0; pt < NP; ++pt)
#pragma unroll
              for (int r = 0; r < 4; ++r) oacc[j][pt][r] *= shift;
        }
      }
      // ---- weights p * scale_v * 2^u of rows (g, g+8), binary16 high and
      // low parts, staged so that each B-fragment register is one load;
      // zero term accumulated here.
      if constexpr (QS == 2) {
        // Weight matrix of a tile, per (n-tile pt, group): 16 tokens x 8
        // columns (head 4pt + c/2 ... : column 2c = high, 2c+1 = low part),
        // i.e. the score fragment layout itself; stored as two 8x8 b16
        // matrices (tokens 0-7, 8-15) with one stmatrix per four matrices.
        const float fu = pow2i(u_run);
#pragma unroll
        for (int tt = 0; tt < NTL; ++tt) {
          uint32_t mr[2 * NGV * NP];
#pragma unroll
          for (int gr = 0; gr < NGV; ++gr) {
            const float2 sc = scales_of(vpa[tt][gr], vpb[tt][gr]);
            const float2 zr = zeros_of(vpa[tt][gr], vpb[tt][gr]);
#pragma unroll
            for (int hs = 0; hs < HT; ++hs) {
              const float2 P = __fmul2_rn(__fmul2_rn(pr[tt][hs], make_float2(fu, fu)), sc);
              const uint32_t hi = f2_to_h2(P.x, P.y);
              const float2 hf = unpack_half2(hi);
              const uint32_t lo = f2_to_h2(P.x - hf.x, P.y - hf.y);
              mr[2 * (hs * NGV + gr)] = __byte_perm(hi, lo, 0x5410);      // row g: (high, low)
              mr[2 * (hs * NGV + gr) + 1] = __byte_perm(hi, lo, 0x7632);  // row g + 8
              zacc[hs][gr] = __ffma2_rn(pr[tt][hs], zr, zacc[hs][gr]);
            }
          }
          uint8_t* wbt = reinterpret_cast<uint8_t*>(wb + (t_first + tt) * C::WB_HALVES);
#pragma unroll
          for (int m0 = 0; m0 < 2 * NGV * NP; m0 += 4) {
            if constexpr (2 * NGV * NP >= 4)
              stmatrix_b16<4>(wbt + m0 * 128 + lane * 16, mr + m0);
            else
              stmatrix_b16<2>(wbt + m0 * 128 + lane * 16, mr + m0);
          }
        }
      } else {
        const float fu = pow2i(u_run);
#pragma unroll
        for (int tt = 0; tt < NTL; ++tt) {
          uint16_t* wbt = wb + (t_first + tt) * C::WB_HALVES;
#pragma unroll
          for (int gr = 0; gr < NGV; ++gr) {
            const float2 sc = scales_of(vpa[tt][gr], vpb[tt][gr]);
            const float2 zr = zeros_of(vpa[tt][gr], vpb[tt][gr]);
#pragma unroll
            for (int hs = 0; hs < HT; ++hs) {
              const int head = QS == 2 ? 4 * hs + c : 8 * (hs / 2) + 2 * c + (hs & 1);
              const float2 P = __fmul2_rn(__fmul2_rn(pr[tt][hs], make_float2(fu, fu)), sc);
              const uint32_t hi = f2_to_h2(P.x, P.y);
              const float2 hf = unpack_half2(hi);
              const uint32_t lo = f2_to_h2(P.x - hf.x, P.y - hf.y);
              uint16_t* row = wbt + (gr * 8 + head) * 2 * C::WB_RS;
              row[g] = static_cast<uint16_t>(hi);
              row[g + 8] = static_cast<uint16_t>(hi >> 16);
              row[C::WB_RS + g] = static_cast<uint16_t>(lo);
              row[C::WB_RS + g + 8] = static_cast<uint16_t>(lo >> 16);
              zacc[hs][gr] = __ffma2_rn(pr[tt][hs], zr, zacc[hs][gr]);
            }
          }
        }
      }
      __syncwarp();
      if (changed) {
#pragma unroll
        for (int pt = 0; pt < NP; ++pt) {
          const float ao = walph[4 * pt + c];
#pragma unroll
          for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) oacc[j][pt][r] *= ao;
        }
      }
      // ---- output: O^T[dim][col] += codes^T . (p * scale_v)
      uint32_t bp[NTL][NP][NGV][2];
      uint32_t vw[NTL][C::VW];
#pragma unroll
      for (int tt = 0; tt < NTL; ++tt) {
        if constexpr (QS == 2) {
          // transposed loads give the B fragments (tokens 2c, 2c+1 | +8, +9; column g)
          const uint8_t* wbt = reinterpret_cast<const uint8_t*>(wb + (t_first + tt) * C::WB_HALVES);
          uint32_t d[2 * NGV * NP];
#pragma unroll
          for (int m0 = 0; m0 < 2 * NGV * NP; m0 += 4) {
            if constexpr (2 * NGV * NP >= 4)
              ldmatrix_trans_b16<4>(wbt + m0 * 128 + lane * 16, d + m0);
            else
              ldmatrix_trans_b16<2>(wbt + m0 * 128 + lane * 16, d + m0);
          }
#pragma unroll
          for (int pt = 0; pt < NP; ++pt)
#pragma unroll
            for (int gr = 0; gr < NGV; ++gr) {
              bp[tt][pt][gr][0] = d[2 * (pt * NGV + gr)];
              bp[tt][pt][gr][1] = d[2 * (pt * NGV + gr) + 1];
            }
        } else {
          const uint16_t* rd = wb + (t_first + tt) * C::WB_HALVES + g * C::WB_RS + 2 * c;
#pragma unroll
          for (int pt = 0; pt < NP; ++pt)
#pragma unroll
            for (int gr = 0; gr < NGV; ++gr) {
              const uint16_t* row = rd + (gr * 8 + 4 * pt) * 2 * C::WB_RS;
              bp[tt][pt][gr][0] = *reinterpret_cast<const uint32_t*>(row);
              bp[tt][pt][gr][1] = *reinterpret_cast<const uint32_t*>(row + 8);
            }
        }
#pragma unroll
        for (int pc = 0; pc < C::VN / C::VP; ++pc)
          lds_words<C::VP>(st + v_off + (t_first + tt) * C::VTILE + pc * 32 * C::VP, vw[tt],
                           pc * (C::VP / 4));
      }
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j) {
        const int gr = 16 * j / GV;
#pragma unroll
        for (int tt = 0; tt < NTL; ++tt) {
          const uint32_t a0 = extract_codes<C::BV>(vw[tt], 0, 2 * j);
          const uint32_t a1 = extract_codes<C::BV>(vw[tt], 0, 2 * j + 1);
          const uint32_t a2 = extract_codes<C::BV>(vw[tt], C::WV, 2 * j);
          const uint32_t a3 = extract_codes<C::BV>(vw[tt], C::WV, 2 * j + 1);
#pragma unroll
          for (int pt = 0; pt < NP; ++pt)
            mma_f16_16816(oacc[j][pt], a0, a1, a2, a3, bp[tt][pt][gr][0], bp[tt][pt][gr][1]);
        }
      }
      __syncwarp();
    };

    int sl = g0 % C::kSlots;
    uint32_t phase = (g0 / C::kSlots) & 1;
    int it = 0;
    for (; it < my_iters; ++it) {
      // the stage this slot is refilled with (this span's or, past its end,
      // the next span's); paged layout: its page, looked up before the
      // arithmetic so that the block-table read overlaps it
      const bool refill = it + C::kSlots < my_iters;
      int next_page = 0;
      if (paged && lane == 0 && refill) next_page = page_of(cur, it + C::kSlots);
      if (!mbar_wait_bounded(&wfull[sl], phase, err, a.wait_limit_ns)) break;
      const uint8_t* st = wring + sl * C::SLOT_BYTES;
      const int base = it * C::kStageTokens + my_first;  // first position of this slot
      if (base + 16 * TPW <= n_tok) {
        tiles_step(std::true_type{}, std::integral_constant<int, TPW>{}, st, 0, 16);
      } else {
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
          const int rem = n_tok - (base + 16 * tt);
          if (rem >= 16)
            tiles_step(std::true_type{}, std::integral_constant<int, 1>{}, st, tt, 16);
          else if (rem > 0)
            tiles_step(std::false_type{}, std::integral_constant<int, 1>{}, st, tt, rem);
        }
      }
      __syncwarp();
      if (lane == 0) {
        // the warp's reads of this slot are done (registers); hand it back
        // to the copy engine for a later stage: cur's, or past its end the
        // next span's (in order: stage `issued` of the stream)
        if (refill) {
          fence_proxy_async_shared();
          issue(cur, it + C::kSlots, sl, next_page);
          ++issued;
        } else if (!FUSED && !paged && it + C::kSlots == issued &&
                   wnext[0] >= 0) {
          Span s;
          s.b = wnext[0];
          s.hk = wnext[1];
          s.t0 = wnext[2];
          s.t1 = wnext[3];
          if (issued - my_iters < iters_of(s)) {
            fence_proxy_async_shared();
            issue(s, issued - my_iters, sl, 0);
            ++issued;
          }
        }
      }
      if (++sl == C::kSlots) {
        sl = 0;
        phase ^= 1u;
      }
    }
    timed_out = it < my_iters;
    consumed = it;
  }
  // the next span: its first stages and its query elements are requested
  // before the merge, so that they arrive during it (the elements always,
  // so that their registers are free during the main loop; without a next
  // span they are cur's again, unused)
  has_next = next(nxt);
  if (!FUSED && has_next && !timed_out && lane == 0) {
    const int n = min(C::kSlots, iters_of(nxt));
    for (; issued < my_iters + n; ++issued)
      issue(nxt, issued - my_iters, (g0 + issued) % C::kSlots,
            paged ? page_of(nxt, issued - my_iters) : 0);
  }

  // ------------------------------------------------------------ epilogue
  // all stages consumed; a wait that ran out stops the CTA, after the copies
  // still in flight (this span's and the next one's) have landed: shared
  // memory must not be left to them; bounded in any case
  const bool aborted = __syncthreads_or(timed_out || ctl[2] != 0);
  // (query rows still in flight are waited for at the kernel's end)
  if (aborted && lane == 0)
    for (int k = g0 + consumed; k < g0 + issued; ++k)
      mbar_wait_bounded(&wfull[k % C::kSlots], (k / C::kSlots) & 1, a.err, a.wait_limit_ns);
  g0 += my_iters;
  pre = issued - my_iters;
  float* ob = reinterpret_cast<float*>(wbuf);  // [warp][OB_HEADS][D]
  float* mb = mrg;                             // [warp][8]
  float* lb = mb + C::kWarps * 8;              // [warp][8]
  float* zb = lb + C::kWarps * 8;              // [warp][8][NGV]
  float* wt = zb + C::kWarps * 8 * NGV;         // [head][warp] merge weights
  float* rden = wt + 8 * C::kWarps;            // [head] 1 / denominator
  {
#pragma unroll
    for (int hs = 0; hs < HT; ++hs) {
      const int head = QS == 2 ? 4 * hs + c : 8 * (hs / 2) + 2 * c + (hs & 1);
      float l = l_run[hs];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      float z[NGV];
#pragma unroll
      for (int gr = 0; gr < NGV; ++gr) {
        z[gr] = zacc[hs][gr].x + zacc[hs][gr].y;
        z[gr] += __shfl_xor_sync(0xffffffffu, z[gr], 4);
        z[gr] += __shfl_xor_sync(0xffffffffu, z[gr], 8);
        z[gr] += __shfl_xor_sync(0xffffffffu, z[gr], 16);
      }
      if (g == 0) {
        mb[warp * 8 + head] = m_run[hs];
        lb[warp * 8 + head] = l;
#pragma unroll
        for (int gr = 0; gr < NGV; ++gr) zb[(warp * 8 + head) * NGV + gr] = z[gr];
      }
    }
#pragma unroll
    for (int pt = 0; pt < NP; ++pt) {
      const int head = 4 * pt + c;
#pragma unroll
      for (int j = 0; j < KSTEPS; ++j) {
        const float s0 = pow2i(24 - u_run - field_pos<C::BV>((2 * j) % (16 / C::BV)));
        const float s1 = pow2i(24 - u_run - field_pos<C::BV>((2 * j + 1) % (16 / C::BV)));
        ob[(warp * C::OB_HEADS + head) * D + 16 * j + g] = (oacc[j][pt][0] + oacc[j][pt][1]) * s0;
        ob[(warp * C::OB_HEADS + head) * D + 16 * j + 8 + g] = (oacc[j][pt][2] + oacc[j][pt][3]) * s1;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < nh) {
    const int head = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) M = fmaxf(M, mb[w * 8 + head]);
    float den = 0.0f;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) {
      const float mw = mb[w * 8 + head];
      const float x = mw == -INFINITY ? 0.0f : exp2_approx(mw - M);
      wt[head * C::kWarps + w] = x;
      den = fmaf(x, lb[w * 8 + head], den);
    }
    rden[head] = __frcp_rn(den);
    if (!direct) {
      const size_t row = (static_cast<size_t>(b) * a.q_heads + head0 + head) * ws_stride + ws_index;
      a.ws_lse[row] = M + __log2f(den);
    }
  }
  if (threadIdx.x == 0) ++ctl[0];  // every thread read it in the prologue
  __syncthreads();
  for (int idx = threadIdx.x; idx < nh * D; idx += C::kThreads) {
    const int head = idx / D, d = idx % D;
    float num = 0.0f;
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w)
      num = fmaf(wt[head * C::kWarps + w], ob[(w * C::OB_HEADS + head) * D + d] + zb[(w * 8 + head) * NGV + d / GV], num);
    if (direct) {
      store_out(a.out, a.out_dtype, (static_cast<size_t>(b) * a.q_heads + head0 + head) * D + d,
                num * rden[head]);
    } else {
      const size_t row = (static_cast<size_t>(b) * a.q_heads + head0 + head) * ws_stride + ws_index;
      a.ws_o[row * D + d] = num * rden[head];
    }
  }
  return aborted;
}

// The decode kernel: one span per CTA on the per-row split grid (grid =
// (splits, kv heads x head groups, batch rows)), or, with stream_q > 0, the
// balanced (stream-K) schedule: the positions of every
// (batch row, kv head, head group) unit are cut into stages of kStageTokens;
// the units' stages, row after row, form one sequence of S stages, and CTA c
// of the one-wave grid takes stages [c*Q, (c+1)*Q), Q = max(stream_q,
// ceil(S / grid)), so that every CTA streams the same number of stages
// whatever the row lengths.  A unit that one CTA covers whole is written
// directly; the others leave one partial result per covering CTA (index:
// the CTA's rank among them) for the combine kernel.  The balanced schedule
// takes at most kStreamRows rows.
template <class C, bool FUSED, bool PAGED>
__global__ void __launch_bounds__(C::kThreads, C::kMinBlocks)
    decode_kernel(const DecodeArgs a) {
  constexpr int D = C::D, T = C::kStageTokens;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);  // [warp][slot]
  uint64_t* qfull = full + C::kWarps * C::kSlots;                   // [query buffer]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* wfull = full + warp * C::kSlots;
  if (lane == 0) {
    for (int sl = 0; sl < C::kSlots; ++sl) mbar_init(&wfull[sl], 1);
    if (warp == 0) {
      mbar_init(&qfull[0], 1);
      mbar_init(&qfull[1], 1);
      reinterpret_cast<int*>(smem + C::CTL_OFF)[0] = 0;  // spans begun
      reinterpret_cast<int*>(smem + C::CTL_OFF)[1] = 0;  // next span's query rows in flight
      reinterpret_cast<int*>(smem + C::CTL_OFF)[2] = 0;  // a query wait ran out
    }
    fence_barrier_init();
  }
  // the query buffers' barriers and the control words are shared by all
  // warps: initialised before any warp uses them
  __syncthreads();
  const int lim = min(a.max_seq_len, a.capacity);
  const bool stream = a.stream_q > 0;

  // balanced schedule: the rows' lengths and the prefix sums of their stages,
  // built before the wait for the previous grid (no kernel of this library
  // writes the lengths; the ring is free scratch until the first span)
  int* lens = reinterpret_cast<int*>(smem + C::SMEM_BYTES - 4 * (2 * kStreamRows + 1));
  int* off = lens + kStreamRows;
  const int U = a.kv_heads * a.head_groups;
  int p = 0, p_end = 0, Q = 1, rb = 0;
  if (stream) {
    stream_row_offsets(a.seq_lens, a.batch, lim, U, T, off, lens, reinterpret_cast<int*>(smem));
    const int S = off[kStreamRows];  // rows past the batch count no stages
    Q = max(a.stream_q, (S + gridDim.x - 1) / gridDim.x);
    p = blockIdx.x * Q;
    p_end = min(p + Q, S);
    // the row holding stage p (rows with no stages are skipped)
    while (rb < a.batch - 1 && off[rb + 1] <= p) ++rb;
  }
  pdl_wait();
  pdl_trigger();
  if (stream && blockIdx.x == 0)
    for (int r = threadIdx.x; r < a.batch; r += C::kThreads)
      if (lens[r] < 0 || lens[r] > lim) flag_error(a.err, KVQ_DEVERR_SEQ_LEN);

  // Span of the balanced schedule at stage p of row rb: stages [j0, j1) of
  // unit u; adv = j1 - j0.
  auto stream_span = [&](int pp, int r, Span& s, int& adv) {
    const int ns = (off[r + 1] - off[r]) / U;  // stages of each unit of row r
    const int q0 = pp - off[r];
    const int u = q0 / ns;
    const int j0 = q0 % ns;
    const int j1 = min(ns, j0 + (p_end - pp));
    s.b = r;
    s.hk = u / a.head_groups;
    s.hg = u % a.head_groups;
    s.t0 = j0 * T;
    const int len_raw = lens[r];
    s.t1 = min(max(0, min(len_raw, lim)), j1 * T);
    // fused append: as on the split grid; a row shorter than the new rows
    // is flagged once (by the CTA holding its first unit's first stage)
    s.app_pos = -1;
    if (FUSED && a.k_new != nullptr && len_raw <= lim) {
      if (len_raw >= a.n_new)
        s.app_pos = len_raw - a.n_new;
      else if (u == 0 && j0 == 0 && threadIdx.x == 0)
        flag_error(a.err, KVQ_DEVERR_BAD_POS);
    }
    const int ubase = off[r] + u * ns;  // the unit's first stage
    s.ws_index = blockIdx.x - ubase / Q;
    s.direct = ubase / Q == (ubase + ns - 1) / Q;
    adv = j1 - j0;
  };

  Span cur;
  int adv = 0;
  // the first span's query rows are requested first (query buffer 0)
  const bool q_bulk = !a.rotate_q;
  auto first_q = [&]() {
    if (q_bulk && threadIdx.x == 0) issue_q_rows<C>(a, cur, smem + C::QBUF_OFF, &qfull[0]);
  };
  if (stream) {
    if (p >= p_end) return;
    stream_span(p, rb, cur, adv);
    first_q();
  } else {
    // Grid (splits, kv heads x head groups, batch rows).  The fused instance
    // is launched as (kv heads x head groups, batch rows, k) instead, split
    // = the row's last split - k: the splits holding the new positions
    // (longer than the others by their append) are the first ones the block
    // scheduler starts and places.  Same splits, same results; only the
    // launch order differs.
    const int unit = FUSED ? blockIdx.x : blockIdx.y;
    const int k = FUSED ? blockIdx.z : blockIdx.x;  // k == 0: one CTA per row flags
    cur.hk = unit / a.head_groups;
    cur.hg = unit % a.head_groups;
    cur.b = FUSED ? blockIdx.y : blockIdx.z;
    int len = a.seq_lens[cur.b];
    // fused append: positions [len - n_new, len) are written first; a row
    // whose length is out of range appends nothing
    cur.app_pos = -1;
    if (FUSED && a.k_new != nullptr && len <= lim) {
      if (len < a.n_new) {
        if (k == 0 && unit == 0 && threadIdx.x == 0) flag_error(a.err, KVQ_DEVERR_BAD_POS);
      } else {
        cur.app_pos = len - a.n_new;
      }
    }
    if (len < 0 || len > lim) {
      if (k == 0 && unit == 0 && threadIdx.x == 0) flag_error(a.err, KVQ_DEVERR_SEQ_LEN);
      len = max(0, min(len, lim));
    }
    int split = k;
    if constexpr (FUSED) {
      const int ns = (len + a.split_tokens - 1) / a.split_tokens;
      if (k < ns) split = ns - 1 - k;  // (k >= ns: past the row, empty as on the plain grid)
    }
    cur.t0 = split * a.split_tokens;
    if (cur.t0 >= len) {
      // an empty sequence attends to nothing: its output rows are zero
      const int head0 = cur.hk * a.gq + cur.hg * a.heads_per_cta;
      const int nh = min(a.heads_per_cta, a.gq - cur.hg * a.heads_per_cta);
      if (a.direct && len == 0 && split == 0)
        for (int i = threadIdx.x; i < nh * D; i += C::kThreads)
          store_out(a.out, a.out_dtype,
                    (static_cast<size_t>(cur.b) * a.q_heads + head0 + i / D) * D + i % D, 0.0f);
      return;
    }
    cur.t1 = min(cur.t0 + a.split_tokens, len);
    cur.ws_index = split;
    cur.direct = a.direct;
    first_q();
  }

  int g0 = 0, pre = 0;  // this warp's copy stream (see decode_span)
  // the CTA's span after the one at stage p (split grid: none): peek only
  // looks, next moves on
  auto peek = [&](Span& s) {
    if (!stream) return false;
    const int pp = p + adv;
    if (pp >= p_end) return false;
    int r = rb;
    while (r < a.batch - 1 && off[r + 1] <= pp) ++r;
    int ad;
    stream_span(pp, r, s, ad);
    return true;
  };
  auto next = [&](Span& s) {
    if (!stream) return false;
    p += adv;
    while (rb < a.batch - 1 && off[rb + 1] <= p) ++rb;
    if (p >= p_end) return false;
    stream_span(p, rb, s, adv);
    return true;
  };
  for (bool first = true;; first = false) {
    // the previous span's merge is done with shared memory before this
    // span's prologue and first tile reuse it
    if (!first) __syncthreads();
    Span nxt = cur;
    bool has_next = false;
    if (decode_span<C, FUSED, PAGED>(a, smem, cur, peek, next, nxt, has_next, a.num_splits, g0,
                                     pre) ||
        !has_next)
      break;
    cur = nxt;
  }
  // after a wait ran out: query rows still in flight land before the CTA
  // ends (the last span's, if its wait ran out, and the next span's)
  const int* ctl = reinterpret_cast<const int*>(smem + C::CTL_OFF);
  if (threadIdx.x == 0 && (ctl[1] != 0 || ctl[2] != 0)) {
    const int last = ctl[0] - 1;
    if (ctl[2]) mbar_wait_bounded(&qfull[last & 1], (last >> 1) & 1, a.err, a.wait_limit_ns);
    if (ctl[1]) mbar_wait_bounded(&qfull[(last + 1) & 1], ((last + 1) >> 1) & 1, a.err, a.wait_limit_ns);
  }
}

template <class C, bool FUSED, bool PAGED>
cudaError_t launch_decode(const DecodeArgs& a, dim3 grid, cudaStream_t stream) {
  return launch_pdl(decode_kernel<C, FUSED, PAGED>, grid, dim3(C::kThreads), C::SMEM_BYTES,
                    stream, a);
}

template <class C, bool PAGED>
DecodeKernel make_decode_kernel() {
  DecodeKernel k;
  k.fn = reinterpret_cast<const void*>(&decode_kernel<C, false, PAGED>);
  k.fn_fused = reinterpret_cast<const void*>(&decode_kernel<C, true, PAGED>);
  k.threads = C::kThreads;
  k.smem_bytes = C::SMEM_BYTES;
  k.launch = &launch_decode<C, false, PAGED>;
  k.launch_fused = &launch_decode<C, true, PAGED>;
  k.tile = 64;
  k.max_per_sm = 0;
  k.stage_tokens = C::kStageTokens;
  return k;
}

// Instances for one (bits_k, bits_v) pair: D in {64, 128}; groups per row of
// keys and values, equal or with finer key groups (the page's group-size
// finding: keys gain from smaller groups, values do not need them); and the
// query variants: up to 4 heads per CTA (any query type: one head per lane,
// high/low columns), 5..8 heads with 16-bit queries (two heads per lane),
// 5..8 heads with binary32 queries (high/low columns, two n-tiles).
// PAGED: the paged layout's instances (compiled in their own translation
// units, so that the two families build in parallel).
template <int BK, int BV, bool PAGED>
bool get_decode_kernel_bits(int head_dim, int groups_k, int groups_v, int variant,
                            DecodeKernel* out) {
#define KVQ_VARIANTS(D, NGK, NGV)                                                          \
  switch (variant) {                                                                       \
    case 0:                                                                                \
    case 1: *out = make_decode_kernel<DecodeCfg<D, BK, BV, NGK, NGV, 2, 1, 1>, PAGED>(); return true; \
    case 2: *out = make_decode_kernel<DecodeCfg<D, BK, BV, NGK, NGV, 1, 1, 2>, PAGED>(); return true; \
    case 3: *out = make_decode_kernel<DecodeCfg<D, BK, BV, NGK, NGV, 2, 2, 2>, PAGED>(); return true; \
    default: return false;                                                                 \
  }
#define KVQ_GROUPS(D, NGK, NGV) \
  if (groups_k == NGK && groups_v == NGV) { KVQ_VARIANTS(D, NGK, NGV) }
  if (head_dim == 128) {
    KVQ_GROUPS(128, 1, 1)
    KVQ_GROUPS(128, 2, 2)
    KVQ_GROUPS(128, 4, 4)
    KVQ_GROUPS(128, 2, 1)
    KVQ_GROUPS(128, 4, 2)
    KVQ_GROUPS(128, 4, 1)
  } else if (head_dim == 64) {
    KVQ_GROUPS(64, 1, 1)
    KVQ_GROUPS(64, 2, 2)
    KVQ_GROUPS(64, 2, 1)
  }
#undef KVQ_GROUPS
#undef KVQ_VARIANTS
  return false;
}

}  // namespace kvq
