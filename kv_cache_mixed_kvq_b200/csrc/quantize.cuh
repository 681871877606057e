// Quantize-and-append kernel: group-wise asymmetric min-max quantization of
// new K/V rows into the packed cache ("Quantize What Counts: More for Keys,
// Less for Values", summary page, "Problem statement" / "Key contributions":
// keys at b_k bits, values at b_v bits; "Results", "Group-size sensitivity":
// one scale/zero per group of head_dim elements; keys and values may use
// different group sizes, GK and GV).
//
// One CTA handles one 16-position tile of one (batch row, kv head) slot;
// each thread issues all its 16-byte loads before any arithmetic, and about
// ten 96-thread CTAs stay resident per SM.  (A persistent grid that staged
// the next tiles in shared memory with cp.async measured slower on B200:
// more instructions per tile and fewer resident warps.)
// Each thread owns a "chunk" of 8*(16/b) consecutive elements of one token:
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
// In the paged layout a tile (16 positions) never spans two pages; its page
// comes from the block table and its rows and V tile are addressed inside
// (page, kv head) exactly as inside a slot.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace kvq {

// GK / GV: group sizes of the keys / values.
template <int D_, int BK_, int BV_, int GK_, int GV_>
struct QCfg {
  static constexpr int D = D_, BK = BK_, BV = BV_, GK = GK_, GV = GV_;
  static constexpr int NGK = D / GK, NGV = D / GV;
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
  static_assert(GK % 8 == 0 && GV % 8 == 0 && D % CHK == 0 && D % CHV == 0, "shape");
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
  static __device__ __forceinline__ void load16(const void* p, raw* out) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
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
  static __device__ __forceinline__ void load16(const void* p, raw* out) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
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
  static __device__ __forceinline__ void load16(const void* p, raw* out) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(p));
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

// Walsh-Hadamard transform of a key row held as CK chunks of CH binary32
// values (chunk w of the row in the lane whose chunk index is w, the row's
// chunks in consecutive lanes): the butterfly stages h = 1, 2, ..., D/2 in
// that order, (x[i], x[i+h]) <- (x[i] + x[i+h], x[i] - x[i+h]) for i & h == 0;
// stages with h < CH stay in the thread, the others exchange with lane xor
// h/CH (key rotation of the cache format, KVQ_FLAG_ROTATE_KEYS).  Stages
// h >= 2 pair whole float2s and use the packed add; a - b is computed as
// a + (-b) (the same IEEE operation), the negation a sign flip.
__device__ __forceinline__ float2 neg2(float2 a) {
  return make_float2(__uint_as_float(__float_as_uint(a.x) ^ 0x80000000u),
                     __uint_as_float(__float_as_uint(a.y) ^ 0x80000000u));
}

template <int CH, int CK>
__device__ __forceinline__ void rotate_row_chunk(float2 (&f)[CH / 2], int w) {
#pragma unroll
  for (int i = 0; i < CH / 2; ++i) f[i] = make_float2(f[i].x + f[i].y, f[i].x - f[i].y);  // h = 1
#pragma unroll
  for (int hh = 1; hh < CH / 2; hh *= 2)  // h = 2 hh
#pragma unroll
    for (int i = 0; i < CH / 2; ++i)
      if ((i & hh) == 0) {
        const float2 x = f[i], y = f[i + hh];
        f[i] = add2_rn(x, y);
        f[i + hh] = add2_rn(x, neg2(y));
      }
#pragma unroll
  for (int m = 1; m < CK; m *= 2) {  // h = m * CH: partner chunk w ^ m
    const bool upper = (w & m) != 0;
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {
      const float2 y = make_float2(__shfl_xor_sync(0xffffffffu, f[i].x, m),
                                   __shfl_xor_sync(0xffffffffu, f[i].y, m));
      // lower chunk: own + partner; upper chunk: partner (lower index) - own
      f[i] = add2_rn(y, upper ? neg2(f[i]) : f[i]);
    }
  }
}

template <class C, typename TIn, bool ROT>
__global__ void __launch_bounds__(C::THREADS) quantize_append_kernel(const QuantizeArgs a) {
  constexpr int D = C::D, NGK = C::NGK, NGV = C::NGV;
  using P = InPair<TIn>;
  __shared__ __align__(16) uint8_t sk[16 * C::KROW];
  __shared__ __align__(16) uint8_t sv[C::VTILE];
  __shared__ __align__(16) uint32_t skp[16 * NGK];
  __shared__ __align__(16) uint32_t svp[16 * NGV];

  const int b = blockIdx.z;
  const int h = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const int pos = a.pos[b];
  if (pos < 0 || static_cast<long long>(pos) + a.n_new > a.capacity) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0)
      flag_error(a.err, pos < 0 ? KVQ_DEVERR_BAD_POS : KVQ_DEVERR_CAPACITY);
    return;
  }
  const int tile = pos / 16 + static_cast<int>(blockIdx.x);
  const int end = pos + a.n_new;
  if (tile * 16 >= end) return;
  const bool full_tile = tile * 16 >= pos && tile * 16 + 16 <= end;
  const size_t slot = static_cast<size_t>(b) * a.kv_heads + h;
  // destination: row index of the tile's first position in the per-position
  // arrays (K rows, parameters) and index of its V tile
  size_t row0, vt;
  if (a.block_table == nullptr) {
    row0 = slot * a.capacity + tile * 16;
    vt = slot * (a.capacity / 16) + tile;
  } else {
    const int j = (tile * 16) >> a.page_shift;
    const int page = a.block_table[static_cast<size_t>(b) * a.pages_per_seq + j];
    if (page < 0 || page >= a.num_pages) {
      if (threadIdx.x == 0) flag_error(a.err, KVQ_DEVERR_BAD_PAGE);
      return;
    }
    const size_t vslot = static_cast<size_t>(page) * a.kv_heads + h;
    const int local = tile * 16 - (j << a.page_shift);
    row0 = (vslot << a.page_shift) + local;
    vt = (vslot << (a.page_shift - 4)) + local / 16;
  }

  const int t = threadIdx.x;
  const bool is_v = t >= C::KT;  // warp-uniform
  const int ti = is_v ? t - C::KT : t;
  const int chunks = is_v ? C::CV : C::CK;
  const int k = ti / chunks;  // position within the tile
  const int w = ti % chunks;  // chunk index within the row
  const int p = tile * 16 + k;
  const bool valid = k < 16 && p >= pos && p < end;

  if (!is_v) {
    // ------------------------------------------------------------ keys
    constexpr int CH = C::CHK;
    typename P::raw raw[CH / 2];
    if (valid) {
      const TIn* src = reinterpret_cast<const TIn*>(a.k) +
                       (slot * a.n_new + (p - pos)) * D + static_cast<size_t>(CH) * w;
#pragma unroll
      for (int i = 0; i < CH / 2 / P::PER16; ++i) P::load16(src + i * 2 * P::PER16, raw + i * P::PER16);
    } else {
#pragma unroll
      for (int i = 0; i < CH / 2; ++i) raw[i] = P::zero();
    }
    uint32_t acc[8];
    uint32_t par[CH / C::GK > 0 ? CH / C::GK : 1];
    if constexpr (ROT) {
      // rotated keys: quantize H k, computed in binary32 (exact widening first)
      float2 f[CH / 2];
#pragma unroll
      for (int i = 0; i < CH / 2; ++i) f[i] = P::to_f2(raw[i]);
      rotate_row_chunk<CH, C::CK>(f, w);
      quantize_chunk<C::BK, C::GK, CH, float>(f, acc, par);
    } else {
      quantize_chunk<C::BK, C::GK, CH, TIn>(raw, acc, par);
    }
    constexpr int NPAR = CH / C::GK > 0 ? CH / C::GK : 1;
    const bool reports = C::GK > CH ? (w % (C::GK / CH)) == 0 : true;
    const int first_group = (CH * w) / C::GK;
    if (full_tile && k < 16) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint32_t*>(sk + k * C::KROW + c * C::KSLICE + 4 * w) =
            __byte_perm(acc[2 * c], acc[2 * c + 1], 0x5410);
      if (reports)
#pragma unroll
        for (int q = 0; q < NPAR; ++q) skp[k * NGK + first_group + q] = par[q];
    } else if (valid) {
      uint8_t* row = a.k_codes + (row0 + k) * C::KROW;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint32_t*>(row + c * C::KSLICE + 4 * w) =
            __byte_perm(acc[2 * c], acc[2 * c + 1], 0x5410);
      if (reports)
#pragma unroll
        for (int q = 0; q < NPAR; ++q)
          a.k_params[(row0 + k) * NGK + first_group + q] = par[q];
    }
  } else {
    // ---------------------------------------------------------- values
    constexpr int CH = C::CHV;
    typename P::raw raw[CH / 2];
    if (valid) {
      const TIn* src = reinterpret_cast<const TIn*>(a.v) +
                       (slot * a.n_new + (p - pos)) * D + static_cast<size_t>(CH) * w;
#pragma unroll
      for (int i = 0; i < CH / 2 / P::PER16; ++i) P::load16(src + i * 2 * P::PER16, raw + i * P::PER16);
    } else {
#pragma unroll
      for (int i = 0; i < CH / 2; ++i) raw[i] = P::zero();
    }
    uint32_t acc[8];
    uint32_t par[CH / C::GV > 0 ? CH / C::GV : 1];
    quantize_chunk<C::BV, C::GV, CH, TIn>(raw, acc, par);
    constexpr int NPAR = CH / C::GV > 0 ? CH / C::GV : 1;
    const bool reports = C::GV > CH ? (w % (C::GV / CH)) == 0 : true;
    const int first_group = (CH * w) / C::GV;
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
        for (int q = 0; q < NPAR; ++q) svp[k * NGV + first_group + q] = par[q];
    } else if (valid) {
      uint8_t* gt = a.v_codes + vt * C::VTILE;
#pragma unroll
      for (int g = 0; g < 8; ++g)
        *reinterpret_cast<uint16_t*>(gt + off0 + 4 * g * C::VP) = static_cast<uint16_t>(acc[g]);
      if (reports)
#pragma unroll
        for (int q = 0; q < NPAR; ++q)
          a.v_params[(row0 + k) * NGV + first_group + q] = par[q];
    }
  }

  if (full_tile) {
    __syncthreads();
    uint4* gk = reinterpret_cast<uint4*>(a.k_codes + row0 * C::KROW);
    uint4* gv = reinterpret_cast<uint4*>(a.v_codes + vt * C::VTILE);
    uint4* gkp = reinterpret_cast<uint4*>(a.k_params + row0 * NGK);
    uint4* gvp = reinterpret_cast<uint4*>(a.v_params + row0 * NGV);
    for (int i = t; i < 16 * C::KROW / 16; i += C::THREADS) gk[i] = reinterpret_cast<const uint4*>(sk)[i];
    for (int i = t; i < C::VTILE / 16; i += C::THREADS) gv[i] = reinterpret_cast<const uint4*>(sv)[i];
    for (int i = t; i < NGK * 4; i += C::THREADS)  // 16 * NGK words = 4 * NGK uint4
      gkp[i] = reinterpret_cast<const uint4*>(skp)[i];
    for (int i = t; i < NGV * 4; i += C::THREADS)
      gvp[i] = reinterpret_cast<const uint4*>(svp)[i];
  }
}

template <int D, int BK, int BV, int GK, int GV, typename TIn>
cudaError_t launch_q(const QuantizeArgs& a, cudaStream_t stream) {
  using C = QCfg<D, BK, BV, GK, GV>;
  const dim3 grid((a.n_new + 30) / 16, a.kv_heads, a.batch);
  if (a.rotate_keys)
    return launch_pdl(quantize_append_kernel<C, TIn, true>, grid, dim3(C::THREADS), 0, stream, a);
  return launch_pdl(quantize_append_kernel<C, TIn, false>, grid, dim3(C::THREADS), 0, stream, a);
}

// Dispatch over (D, key and value groups, bits) for one input type: equal
// groups, or coarser value groups (the combinations the decode kernel has).
template <typename TIn>
cudaError_t launch_quantize_typed(const QuantizeArgs& a, cudaStream_t stream) {
#define KVQ_Q_BITS(D, GK, GV)                                                       \
  switch (a.bits_k * 16 + a.bits_v) {                                                \
    case 0x22: return launch_q<D, 2, 2, GK, GV, TIn>(a, stream);                     \
    case 0x24: return launch_q<D, 2, 4, GK, GV, TIn>(a, stream);                     \
    case 0x28: return launch_q<D, 2, 8, GK, GV, TIn>(a, stream);                     \
    case 0x42: return launch_q<D, 4, 2, GK, GV, TIn>(a, stream);                     \
    case 0x44: return launch_q<D, 4, 4, GK, GV, TIn>(a, stream);                     \
    case 0x48: return launch_q<D, 4, 8, GK, GV, TIn>(a, stream);                     \
    case 0x82: return launch_q<D, 8, 2, GK, GV, TIn>(a, stream);                     \
    case 0x84: return launch_q<D, 8, 4, GK, GV, TIn>(a, stream);                     \
    case 0x88: return launch_q<D, 8, 8, GK, GV, TIn>(a, stream);                     \
    default: return cudaErrorInvalidValue;                                           \
  }
#define KVQ_Q_GROUPS(D, GK, GV) \
  if (a.group == GK && a.group_v == GV) { KVQ_Q_BITS(D, GK, GV) }
  if (a.head_dim == 128) {
    KVQ_Q_GROUPS(128, 32, 32)
    KVQ_Q_GROUPS(128, 64, 64)
    KVQ_Q_GROUPS(128, 128, 128)
    KVQ_Q_GROUPS(128, 32, 64)
    KVQ_Q_GROUPS(128, 32, 128)
    KVQ_Q_GROUPS(128, 64, 128)
  } else {
    KVQ_Q_GROUPS(64, 32, 32)
    KVQ_Q_GROUPS(64, 64, 64)
    KVQ_Q_GROUPS(64, 32, 64)
  }
#undef KVQ_Q_GROUPS
#undef KVQ_Q_BITS
  return cudaErrorInvalidValue;
}

}  // namespace kvq
