// Quantize-and-append kernel: group-wise asymmetric min-max quantization of
// new K/V rows into the packed cache ("Quantize What Counts: More for Keys,
// Less for Values", summary page, "Problem statement" / "Key contributions":
// keys at b_k bits, values at b_v bits; "Results", "Group-size sensitivity":
// one scale/zero per group of head_dim elements).
//
// A persistent grid walks the 16-position tiles of every (batch row, kv
// head) slot; each CTA stages the input rows of its next tiles in shared
// memory with cp.async (16-byte pieces, each warp reading contiguous global
// memory) several tiles ahead of the one it quantizes.  Inside a tile each
// thread owns a "chunk" of 8*(16/b) consecutive elements of one token:
// exactly the elements whose codes fill one 32-bit word of each of the four
// K slices (keys), or one 16-bit half-word of each of eight V lanes (values),
// so every packed word is built inside one thread without shuffles.
//
// Per element the arithmetic is the binary32 formula of the format with
// explicit round-to-nearest operations (the adds packed f32x2 on sm_100):
//   d = x - min,  t = d * inv,  code = rint(t)
// rint is taken by adding 1.5*2^23 (the sum's rounding is the IEEE
// round-half-even of t, and the code lands in the low mantissa bits); the
// codes of a half-word are packed by shift-and-add (Horner), whose carries of
// the constant's upper bits only ever reach bits >= 22.  No clamp is needed:
// for x in [min, max], t <= fl(range * inv) < 2^b - 1/2.
// Group min/max runs on packed bf16x2/f16x2 pairs (exact), across threads
// by xor-shuffles when a group spans several chunks.
//
// A tile fully covered by the append is assembled in shared memory and
// written with 16-byte stores; a tile at the edge of the appended range is
// written element by element so that positions outside it stay untouched.
#pragma once

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace kvq {

template <int D_, int BK_, int BV_, int G_>
struct QCfg {
  static constexpr int D = D_, BK = BK_, BV = BV_, G = G_;
  static constexpr int NG = D / G;
  static constexpr int EK = 16 / BK, EV = 16 / BV;
  static constexpr int CHK = 8 * EK, CHV = 8 * EV;  // elements per chunk
  static constexpr int CK = D / CHK, CV = D / CHV;  // chunks per token
  static constexpr int KT = (16 * CK + 31) / 32 * 32;  // threads for K items
  static constexpr int VT = (16 * CV + 31) / 32 * 32;  // threads for V items
  static constexpr int THREADS = KT + VT;
  static constexpr int KROW = D * BK / 8;
  static constexpr int KSLICE = D * BK / 32;
  static constexpr int VTILE = 2 * D * BV;
  static constexpr int VN = D * BV / 16;
  static constexpr int VP = VN < 16 ? VN : 16;
  static constexpr int WV = D * BV / 128;
  static_assert(G % 8 == 0 && D % CHK == 0 && D % CHV == 0, "shape");
};

// Raw input pairs and their conversions.
template <typename TIn>
struct InPair;

template <>
struct InPair<__nv_bfloat16> {
  using raw = uint32_t;
  static constexpr int PER16 = 4;  // pairs per 16-byte load
  static __device__ __forceinline__ float2 to_f2(raw w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  static __device__ __forceinline__ raw pmin(raw a, raw b) {
    __nv_bfloat162 r = __hmin2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<raw*>(&r);
  }
  static __device__ __forceinline__ raw pmax(raw a, raw b) {
    __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<raw*>(&r);
  }
  static __device__ __forceinline__ void lds16(const void* p, raw* out) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    out[0] = u.x; out[1] = u.y; out[2] = u.z; out[3] = u.w;
  }
  static __device__ __forceinline__ raw zero() { return 0u; }
};

template <>
struct InPair<__half> {
  using raw = uint32_t;
  static constexpr int PER16 = 4;
  static __device__ __forceinline__ float2 to_f2(raw w) {
    return __half22float2(*reinterpret_cast<__half2*>(&w));
  }
  static __device__ __forceinline__ raw pmin(raw a, raw b) {
    __half2 r = __hmin2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<raw*>(&r);
  }
  static __device__ __forceinline__ raw pmax(raw a, raw b) {
    __half2 r = __hmax2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<raw*>(&r);
  }
  static __device__ __forceinline__ void lds16(const void* p, raw* out) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    out[0] = u.x; out[1] = u.y; out[2] = u.z; out[3] = u.w;
  }
  static __device__ __forceinline__ raw zero() { return 0u; }
};

template <>
struct InPair<float> {
  using raw = float2;
  static constexpr int PER16 = 2;
  static __device__ __forceinline__ float2 to_f2(raw w) { return w; }
  static __device__ __forceinline__ raw pmin(raw a, raw b) {
    return make_float2(fminf(a.x, b.x), fminf(a.y, b.y));
  }
  static __device__ __forceinline__ raw pmax(raw a, raw b) {
    return make_float2(fmaxf(a.x, b.x), fmaxf(a.y, b.y));
  }
  static __device__ __forceinline__ void lds16(const void* p, raw* out) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    out[0] = make_float2(u.x, u.y);
    out[1] = make_float2(u.z, u.w);
  }
  static __device__ __forceinline__ raw zero() { return make_float2(0.0f, 0.0f); }
};

// Packed binary32 add with round-to-nearest-even.  The multiply between the
// two adds of the code formula stays a scalar __fmul_rn: a packed multiply
// followed by a packed add was fused into one multiply-add on sm_100 (the
// exact product then decides the rounding and codes next to a tie change).
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rc, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// Quantize one chunk (CH elements of one token) at B bits.  Outputs the
// per-slice (keys) or per-lane (values) half-words as Horner accumulators:
// acc[x] holds the packed half-word in its low 16 bits.  K: acc[2c] is the
// low and acc[2c+1] the high half of slice c's word; V: acc[g] is lane g's
// half.  par[] receives the (scale, zero) binary16 pairs of the groups that
// this thread reports (n_par of them), first_group their index in the row.
template <int B, int G, int CH, typename TIn>
__device__ __forceinline__ void quantize_chunk(const typename InPair<TIn>::raw (&raw)[CH / 2],
                                               uint32_t (&acc)[8], uint32_t (&par)[CH / G > 0 ? CH / G : 1]) {
  using P = InPair<TIn>;
  constexpr int E = 16 / B;
  constexpr int GC = G < CH ? G : CH;  // elements of one group inside the chunk
  constexpr int NGC = CH / GC;         // groups inside the chunk
  constexpr int TPG = G > CH ? G / CH : 1;  // threads sharing one group
  const float levels = static_cast<float>((1 << B) - 1);
  float2 nmn2[NGC], inv2[NGC];
#pragma unroll
  for (int sg = 0; sg < NGC; ++sg) {
    typename P::raw lo = raw[sg * GC / 2], hi = raw[sg * GC / 2];
#pragma unroll
    for (int p = 1; p < GC / 2; ++p) {
      lo = P::pmin(lo, raw[sg * GC / 2 + p]);
      hi = P::pmax(hi, raw[sg * GC / 2 + p]);
    }
    const float2 l2 = P::to_f2(lo), h2 = P::to_f2(hi);
    float mn = fminf(l2.x, l2.y), mx = fmaxf(h2.x, h2.y);
#pragma unroll
    for (int m = 1; m < TPG; m <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    }
    mn = (mn == 0.0f) ? 0.0f : mn;  // a zero extreme is stored as +0
    mx = (mx == 0.0f) ? 0.0f : mx;
    const float scale = __fdiv_rn(__fsub_rn(mx, mn), levels);
    const float inv = __fdiv_rn(1.0f, scale);
    const bool degenerate = (scale == 0.0f) || !isfinite(scale) || !isfinite(inv);
    // degenerate groups: every code 0 (d * 0 = 0 for the finite inputs)
    nmn2[sg] = degenerate ? make_float2(0.0f, 0.0f) : make_float2(-mn, -mn);
    inv2[sg] = degenerate ? make_float2(0.0f, 0.0f) : make_float2(inv, inv);
    if (sg < (CH / G > 0 ? CH / G : 1)) par[sg] = pack_half2(__float2half_rn(scale), __float2half_rn(mn));
  }
  const float2 magic = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
#pragma unroll
  for (int x = 0; x < 8; ++x) acc[x] = 0u;
  // fields from the highest (e = E-1) down to e = 0: Horner leaves field e
  // at bits [e*B, e*B+B) of the half-word
#pragma unroll
  for (int e = E - 1; e >= 0; --e) {
    const int sg = (8 * e) / GC;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 x = P::to_f2(raw[4 * e + c]);
      const float2 d = add2_rn(x, nmn2[sg]);
      // scalar multiplies: guaranteed never to be fused with the add below
      const float2 t = make_float2(__fmul_rn(d.x, inv2[sg].x), __fmul_rn(d.y, inv2[sg].y));
      const float2 s = add2_rn(t, magic);
      acc[2 * c] = (acc[2 * c] << B) + __float_as_uint(s.x);
      acc[2 * c + 1] = (acc[2 * c + 1] << B) + __float_as_uint(s.y);
    }
  }
}

// Shared-memory staging of the input rows.  A stage holds one tile's K and V
// rows, stored chunk by chunk (the chunk of thread ti at ti * stride) with 16
// bytes of padding after each chunk, so that the 16-byte reads of a chunk's
// owner hit distinct banks across each 8-lane phase.
template <class C, typename TIn>
struct QPipe {
  static constexpr int ES = sizeof(TIn);
  static constexpr int ROWB = C::D * ES;  // bytes per input row
  static constexpr int PPR = ROWB / 16;   // 16-byte pieces per row
  static constexpr int NPK = C::CHK * ES / 16, NPV = C::CHV * ES / 16;  // pieces per chunk
  static constexpr int SK = 16 * (NPK + 1), SV = 16 * (NPV + 1);       // padded chunk strides
  static constexpr int KBYTES = 16 * C::CK * SK, VBYTES = 16 * C::CV * SV;
  static constexpr int STAGE = KBYTES + VBYTES;
  static constexpr int STAGES = ES == 4 ? 2 : 4;  // tiles in flight per CTA
  static constexpr int OUT = 16 * C::KROW + C::VTILE + 2 * 16 * C::NG * 4;
  static constexpr int SMEM = STAGES * STAGE + OUT;
  static_assert(C::CHK * ES % 16 == 0 && C::CHV * ES % 16 == 0, "chunks of whole pieces");
  static_assert(STAGE % 16 == 0 && (16 * C::KROW) % 16 == 0 && C::VTILE % 16 == 0, "alignment");
};

// One tile of the walk: slot (b, h), cache tile index, and the rows [r0, r1)
// of the tile that the append covers.
struct QTile {
  int b, h, x, tile, r0, r1, pos;
  bool ok;   // the tile has rows to write
  bool bad;  // pos[b] is negative or the append overruns the capacity
};

__device__ __forceinline__ QTile q_tile(const QuantizeArgs& a, int idx) {
  QTile t;
  const uint32_t sh = fast_div(static_cast<uint32_t>(idx), a.div_ntps);
  t.x = idx - static_cast<int>(sh) * a.ntps;
  const uint32_t b = fast_div(sh, a.div_heads);
  t.h = static_cast<int>(sh - b * a.kv_heads);
  t.b = static_cast<int>(b);
  t.pos = a.pos[t.b];
  t.bad = t.pos < 0 || static_cast<long long>(t.pos) + a.n_new > a.capacity;
  t.ok = false;
  t.tile = t.r0 = t.r1 = 0;
  if (t.bad) return t;
  t.tile = t.pos / 16 + t.x;
  const int end = t.pos + a.n_new;
  if (t.tile * 16 >= end) return t;
  t.r0 = max(t.tile * 16, t.pos) - t.tile * 16;
  t.r1 = min(t.tile * 16 + 16, end) - t.tile * 16;
  t.ok = true;
  return t;
}

// The 16-byte pieces of a tile's 16 input rows (K and V alike) that one
// thread copies: pieces q = threadIdx.x + i * THREADS.  Consecutive threads
// copy consecutive pieces of a row (coalesced); each piece lands in the
// padded chunk of the thread that will quantize it.  The offsets depend only
// on the thread, so they are computed once per CTA.
template <class C, typename TIn>
struct QCopySlots {
  using Pp = QPipe<C, TIn>;
  static constexpr int PIECES = 16 * Pp::PPR;
  static constexpr int N = (PIECES + C::THREADS - 1) / C::THREADS;
  uint32_t koff[N], voff[N];  // shared-memory offsets within a stage
  int row[N];                 // tile row of the piece (16: none)

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const int q = threadIdx.x + i * C::THREADS;
      const int r = q / Pp::PPR, c = q % Pp::PPR;
      row[i] = q < PIECES ? r : 16;
      koff[i] = (r * C::CK + c / Pp::NPK) * Pp::SK + 16 * (c % Pp::NPK);
      voff[i] = Pp::KBYTES + (r * C::CV + c / Pp::NPV) * Pp::SV + 16 * (c % Pp::NPV);
    }
  }

  // Copies the appended rows [r0, r1) of tile t into `stage`.
  __device__ __forceinline__ void issue(const QuantizeArgs& a, const QTile& t, uint8_t* stage) const {
    if (!t.ok) return;
    // input row of tile row r: slot * n_new + (tile * 16 + r - pos)
    const long long row0 = (static_cast<long long>(t.b) * a.kv_heads + t.h) * a.n_new +
                           (t.tile * 16 - t.pos);
    const uint8_t* kin = reinterpret_cast<const uint8_t*>(a.k) + row0 * Pp::ROWB;
    const uint8_t* vin = reinterpret_cast<const uint8_t*>(a.v) + row0 * Pp::ROWB;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if (row[i] >= t.r0 && row[i] < t.r1) {
        const uint32_t g = (threadIdx.x + i * C::THREADS) * 16u;
        cp_async16(stage + koff[i], kin + g);
        cp_async16(stage + voff[i], vin + g);
      }
    }
  }
};

template <class C, typename TIn>
__global__ void __launch_bounds__(C::THREADS) quantize_append_kernel(const QuantizeArgs a) {
  constexpr int D = C::D, G = C::G, NG = C::NG;
  using P = InPair<TIn>;
  using Pp = QPipe<C, TIn>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sk = smem + Pp::STAGES * Pp::STAGE;
  uint8_t* sv = sk + 16 * C::KROW;
  uint32_t* skp = reinterpret_cast<uint32_t*>(sv + C::VTILE);
  uint32_t* svp = skp + 16 * NG;

  pdl_wait();
  pdl_trigger();

  const int first = blockIdx.x, step = gridDim.x;
  const int my_n = first < a.total_tiles ? (a.total_tiles - 1 - first) / step + 1 : 0;
  QCopySlots<C, TIn> cs;
  cs.init();

  const int t = threadIdx.x;
  const bool is_v = t >= C::KT;  // warp-uniform
  const int ti = is_v ? t - C::KT : t;
  const int chunks = is_v ? C::CV : C::CK;
  const int k = ti / chunks;  // position within the tile
  const int w = ti % chunks;  // chunk index within the row

#pragma unroll 1
  for (int s = 0; s < Pp::STAGES - 1; ++s) {
    if (s < my_n) cs.issue(a, q_tile(a, first + s * step), smem + s * Pp::STAGE);
    cp_async_commit();
  }

#pragma unroll 1
  for (int i = 0; i < my_n; ++i) {
    {
      const int ahead = i + Pp::STAGES - 1;
      if (ahead < my_n)
        cs.issue(a, q_tile(a, first + ahead * step), smem + (ahead % Pp::STAGES) * Pp::STAGE);
      cp_async_commit();
    }
    cp_async_wait<Pp::STAGES - 1>();
    __syncthreads();  // tile i's rows are in its stage

    const QTile tl = q_tile(a, first + i * step);
    if (tl.bad && tl.x == 0 && tl.h == 0 && t == 0)
      flag_error(a.err, tl.pos < 0 ? KVQ_DEVERR_BAD_POS : KVQ_DEVERR_CAPACITY);
    const bool full_tile = tl.ok && tl.r0 == 0 && tl.r1 == 16;
    const size_t slot = static_cast<size_t>(tl.b) * a.kv_heads + tl.h;
    const uint8_t* stage = smem + (i % Pp::STAGES) * Pp::STAGE;

    if (tl.ok) {
      const int p = tl.tile * 16 + k;
      const bool valid = k < 16 && k >= tl.r0 && k < tl.r1;
      if (!is_v) {
        // ------------------------------------------------------------ keys
        constexpr int CH = C::CHK;
        typename P::raw raw[CH / 2];
        if (valid) {
          const uint8_t* src = stage + ti * Pp::SK;
#pragma unroll
          for (int i2 = 0; i2 < Pp::NPK; ++i2) P::lds16(src + 16 * i2, raw + i2 * P::PER16);
        } else {
#pragma unroll
          for (int i2 = 0; i2 < CH / 2; ++i2) raw[i2] = P::zero();
        }
        uint32_t acc[8];
        uint32_t par[CH / G > 0 ? CH / G : 1];
        quantize_chunk<C::BK, G, CH, TIn>(raw, acc, par);
        constexpr int NPAR = CH / G > 0 ? CH / G : 1;
        const bool reports = G > CH ? (w % (G / CH)) == 0 : true;
        const int first_group = (CH * w) / G;
        if (full_tile && k < 16) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint32_t*>(sk + k * C::KROW + c * C::KSLICE + 4 * w) =
                __byte_perm(acc[2 * c], acc[2 * c + 1], 0x5410);
          if (reports)
#pragma unroll
            for (int q = 0; q < NPAR; ++q) skp[k * NG + first_group + q] = par[q];
        } else if (valid) {
          uint8_t* row = a.k_codes + (slot * a.capacity + p) * C::KROW;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint32_t*>(row + c * C::KSLICE + 4 * w) =
                __byte_perm(acc[2 * c], acc[2 * c + 1], 0x5410);
          if (reports)
#pragma unroll
            for (int q = 0; q < NPAR; ++q)
              a.k_params[(slot * a.capacity + p) * NG + first_group + q] = par[q];
        }
      } else {
        // ---------------------------------------------------------- values
        constexpr int CH = C::CHV;
        typename P::raw raw[CH / 2];
        if (valid) {
          const uint8_t* src = stage + Pp::KBYTES + ti * Pp::SV;
#pragma unroll
          for (int i2 = 0; i2 < Pp::NPV; ++i2) P::lds16(src + 16 * i2, raw + i2 * P::PER16);
        } else {
#pragma unroll
          for (int i2 = 0; i2 < CH / 2; ++i2) raw[i2] = P::zero();
        }
        uint32_t acc[8];
        uint32_t par[CH / G > 0 ? CH / G : 1];
        quantize_chunk<C::BV, G, CH, TIn>(raw, acc, par);
        constexpr int NPAR = CH / G > 0 ? CH / G : 1;
        const bool reports = G > CH ? (w % (G / CH)) == 0 : true;
        const int first_group = (CH * w) / G;
        // half-word of position k in lane 4g + (k mod 8)/2, word (k/8)*WV + w
        const int n = 4 * ((k / 8) * C::WV + w) + 2 * (k % 2);
        const int lane0 = (k % 8) / 2;
        const int off0 = (n / C::VP) * 32 * C::VP + lane0 * C::VP + (n % C::VP);
        if (full_tile && k < 16) {
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<uint16_t*>(sv + off0 + 4 * g * C::VP) = static_cast<uint16_t>(acc[g]);
          if (reports)
#pragma unroll
            for (int q = 0; q < NPAR; ++q) svp[k * NG + first_group + q] = par[q];
        } else if (valid) {
          uint8_t* gt = a.v_codes + (slot * (a.capacity / 16) + tl.tile) * C::VTILE;
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<uint16_t*>(gt + off0 + 4 * g * C::VP) = static_cast<uint16_t>(acc[g]);
          if (reports)
#pragma unroll
            for (int q = 0; q < NPAR; ++q)
              a.v_params[(slot * a.capacity + p) * NG + first_group + q] = par[q];
        }
      }
    }
    __syncthreads();  // the stage is free; a full tile's packed output is complete
    if (full_tile) {
      uint4* gk = reinterpret_cast<uint4*>(a.k_codes + (slot * a.capacity + tl.tile * 16) * C::KROW);
      uint4* gv = reinterpret_cast<uint4*>(a.v_codes + (slot * (a.capacity / 16) + tl.tile) * C::VTILE);
      uint4* gkp = reinterpret_cast<uint4*>(a.k_params + (slot * a.capacity + tl.tile * 16) * NG);
      uint4* gvp = reinterpret_cast<uint4*>(a.v_params + (slot * a.capacity + tl.tile * 16) * NG);
      for (int i2 = t; i2 < 16 * C::KROW / 16; i2 += C::THREADS) gk[i2] = reinterpret_cast<const uint4*>(sk)[i2];
      for (int i2 = t; i2 < C::VTILE / 16; i2 += C::THREADS) gv[i2] = reinterpret_cast<const uint4*>(sv)[i2];
      for (int i2 = t; i2 < NG * 4; i2 += C::THREADS) {  // 16 * NG words = 4 * NG uint4
        gkp[i2] = reinterpret_cast<const uint4*>(skp)[i2];
        gvp[i2] = reinterpret_cast<const uint4*>(svp)[i2];
      }
    }
  }
  cp_async_wait<0>();  // no copy may land after the CTA has exited
}

// Persistent launch: as many CTAs as fit on the device at once (queried
// once per device), each walking tiles blockIdx.x, blockIdx.x + gridDim.x, ...
template <int D, int BK, int BV, int G, typename TIn>
cudaError_t launch_q(const QuantizeArgs& a, cudaStream_t stream) {
  using C = QCfg<D, BK, BV, G>;
  using Pp = QPipe<C, TIn>;
  constexpr int kMaxDevices = 64;
  static std::atomic<int> per_sm_cache[kMaxDevices];
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (dev < kMaxDevices) per_sm = per_sm_cache[dev].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    e = cudaFuncSetAttribute(quantize_append_kernel<C, TIn>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Pp::SMEM);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_append_kernel<C, TIn>,
                                                        C::THREADS, Pp::SMEM);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    if (dev < kMaxDevices) per_sm_cache[dev].store(per_sm, std::memory_order_relaxed);
  }
  QuantizeArgs w = a;
  w.ntps = (a.n_new + 30) / 16;  // tiles an append of n_new can touch
  const long long total = static_cast<long long>(w.ntps) * a.kv_heads * a.batch;
  if (total >= (1ll << 31)) return cudaErrorInvalidValue;
  w.total_tiles = static_cast<int>(total);
  w.div_ntps = make_fast_div(static_cast<uint32_t>(w.ntps));
  w.div_heads = make_fast_div(static_cast<uint32_t>(a.kv_heads));
  const long long cap = static_cast<long long>(sms) * per_sm;
  const dim3 grid(static_cast<unsigned>(total < cap ? total : cap));
  return launch_pdl(quantize_append_kernel<C, TIn>, grid, dim3(C::THREADS), Pp::SMEM, stream, w);
}

// Dispatch over (D, G, bits) for one input type.
template <typename TIn>
cudaError_t launch_quantize_typed(const QuantizeArgs& a, cudaStream_t stream) {
#define KVQ_Q_BITS(D, G)                                                            \
  switch (a.bits_k * 16 + a.bits_v) {                                                \
    case 0x22: return launch_q<D, 2, 2, G, TIn>(a, stream);                          \
    case 0x24: return launch_q<D, 2, 4, G, TIn>(a, stream);                          \
    case 0x28: return launch_q<D, 2, 8, G, TIn>(a, stream);                          \
    case 0x42: return launch_q<D, 4, 2, G, TIn>(a, stream);                          \
    case 0x44: return launch_q<D, 4, 4, G, TIn>(a, stream);                          \
    case 0x48: return launch_q<D, 4, 8, G, TIn>(a, stream);                          \
    case 0x82: return launch_q<D, 8, 2, G, TIn>(a, stream);                          \
    case 0x84: return launch_q<D, 8, 4, G, TIn>(a, stream);                          \
    case 0x88: return launch_q<D, 8, 8, G, TIn>(a, stream);                          \
    default: return cudaErrorInvalidValue;                                           \
  }
  if (a.head_dim == 128) {
    if (a.group == 32) { KVQ_Q_BITS(128, 32) }
    if (a.group == 64) { KVQ_Q_BITS(128, 64) }
    if (a.group == 128) { KVQ_Q_BITS(128, 128) }
  } else {
    if (a.group == 32) { KVQ_Q_BITS(64, 32) }
    if (a.group == 64) { KVQ_Q_BITS(64, 64) }
  }
#undef KVQ_Q_BITS
  return cudaErrorInvalidValue;
}

}  // namespace kvq
