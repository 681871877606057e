/*
 * kvq_oracle.c — plain, slow, obviously-correct CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * constant with the CUDA library: the cache format and the quantizer below
 * are written again from their textual definitions.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no fused multiply-add, IEEE binary32 arithmetic on SSE, default
 * round-to-nearest-even mode).
 *
 * What it computes, with the passage each step follows:
 *   - ora_quantize_group: the group-wise asymmetric min-max quantizer that
 *     the summary page "Quantize What Counts: More for Keys, Less for Values"
 *     leaves open ("Problem statement": BF16 cache stored at INT4 or fewer
 *     bits; "Results", "Group-size sensitivity": one quantizer per group of
 *     head_dim elements).  Steps in binary32, in this order: min/max
 *     (signed zeros made +0), range/(2^b-1), reciprocal, (x-min)*reciprocal, round half to even,
 *     clamp; stored scale and min rounded to binary16.
 *   - ora_k_code_place / ora_v_code_place: where a code lives in the packed
 *     cache (the library's documented format; see the header of the library
 *     for the definition this restates).
 *   - ora_decode_attention: softmax(q k^T * sm_scale) v in binary64 on the
 *     dequantised cache (plain definition of one decode step of attention).
 *   - ora_attention_dense: the same on unquantised K/V (the full-precision
 *     baseline of "Results", "Downstream accuracy").
 *   - separate group sizes (the *_g2 variants): "Results", "Group-size
 *     sensitivity": finer groups (32) help the keys, coarser ones (64 or 128)
 *     are enough for the values; keys use groups of Gk elements and values
 *     groups of Gv, each array's (scale, zero) pairs indexed by its own
 *     group count D/Gk or D/Gv.
 *   - ora_fwht and the *_ex variants: key-only rotation ("Results",
 *     "Integration with rotation": rotating only the keys in a K4V2 setting
 *     comes close to K4V4; the page names no transform, the plainest reading
 *     is a Walsh-Hadamard rotation of each key row along head_dim).  Keys are
 *     stored as H k (H the unnormalised Sylvester Hadamard matrix, computed
 *     by the butterfly below in binary32); the query is rotated the same way
 *     and divided by D, so that (H q / D) . (H k) = q . k.
 *
 * Every function here is pinned by the -m "not gpu" tests (closed forms,
 * brute force, library routines, invariants); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- numbers */

/* Round a binary32 value to the nearest binary16 (ties to even) and return
 * its bit pattern.  Written from the IEEE 754 definition: find the spacing
 * of binary16 numbers at |f|, round |f|/spacing to an integer, re-encode. */
uint16_t ora_f32_to_f16(float f) {
  uint32_t bits;
  memcpy(&bits, &f, sizeof bits);
  uint16_t sign = (bits >> 31) ? 0x8000u : 0u;
  if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
  if (isinf(f)) return (uint16_t)(sign | 0x7c00u);
  double a = fabs((double)f);
  /* 65504 is the largest finite binary16; the midpoint to the next power of
   * two, 65520, and everything above rounds to infinity. */
  if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
  double spacing;
  if (a < 0x1p-14) {
    spacing = 0x1p-24; /* subnormal range */
  } else {
    int e;
    frexp(a, &e); /* a in [2^(e-1), 2^e) */
    spacing = ldexp(1.0, (e - 1) - 10);
  }
  double n = nearbyint(a / spacing); /* exact quotient; ties to even */
  double r = n * spacing;
  if (r == 0.0) return sign;
  if (r < 0x1p-14) return (uint16_t)(sign | (uint16_t)(r / 0x1p-24));
  int e;
  frexp(r, &e);
  int E = e - 1; /* r in [2^E, 2^(E+1)) */
  uint16_t man = (uint16_t)((r / ldexp(1.0, E) - 1.0) * 1024.0);
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | man);
}

float ora_f16_to_f32(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25);
  return (float)(s ? -v : v);
}

float ora_bf16_to_f32(uint16_t b) {
  uint32_t bits = (uint32_t)b << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return f;
}

/* Element i of an array of dtype 0 = binary32, 1 = bfloat16, 2 = binary16. */
static float load_elem(const void* base, int dtype, size_t i) {
  if (dtype == 0) return ((const float*)base)[i];
  if (dtype == 1) return ora_bf16_to_f32(((const uint16_t*)base)[i]);
  return ora_f16_to_f32(((const uint16_t*)base)[i]);
}

/* -------------------------------------------------------------- quantizer */

/* Quantize one group of n binary32 values to b-bit codes.
 * Outputs: codes[n], the binary32 scale and minimum the codes were computed
 * from, and the stored binary16 scale and zero (bit patterns). */
void ora_quantize_group(const float* x, int n, int bits, uint8_t* codes,
                        float* scale32, float* min32, uint16_t* scale16,
                        uint16_t* zero16) {
  float mn = x[0], mx = x[0];
  for (int i = 1; i < n; ++i) {
    if (x[i] < mn) mn = x[i];
    if (x[i] > mx) mx = x[i];
  }
  mn = mn + 0.0f; /* a -0 minimum becomes +0 */
  mx = mx + 0.0f; /* and so does a -0 maximum */
  float levels = (float)((1 << bits) - 1);
  float range = mx - mn;
  float scale = range / levels;
  float inv = 1.0f / scale;
  int degenerate = (scale == 0.0f) || !isfinite(scale) || !isfinite(inv);
  for (int i = 0; i < n; ++i) {
    if (degenerate) {
      codes[i] = 0;
      continue;
    }
    float t = (x[i] - mn) * inv;
    float r = nearbyintf(t);
    if (r < 0.0f) r = 0.0f;
    if (r > levels) r = levels;
    codes[i] = (uint8_t)r;
  }
  *scale32 = scale;
  *min32 = mn;
  *scale16 = ora_f32_to_f16(scale);
  *zero16 = ora_f32_to_f16(mn);
}

/* ------------------------------------------------------------ cache format */

/* Byte offset (within one K row of D*b/8 bytes) and bit shift (within that
 * byte) of the code of element d.  Definition: E = 16/b codes per 16-bit
 * half-word; slice c = (d mod 8)/2 of D*b/32 bytes; 32-bit little-endian
 * word (d/8)/E of the slice; bit 16*(d mod 2) + b*((d/8) mod E) of it. */
void ora_k_code_place(int D, int b, int d, int* byte_off, int* shift) {
  int E = 16 / b;
  int slice = (d % 8) / 2;
  int word = (d / 8) / E;
  int bit = 16 * (d % 2) + b * ((d / 8) % E);
  *byte_off = slice * (D * b / 32) + 4 * word + bit / 8;
  *shift = bit % 8;
}

/* Byte offset (within one 16-position V tile of 2*D*b bytes) and bit shift
 * of the code of (position k within the tile, element d).  Definition:
 * lane 4*(d mod 8) + (k mod 8)/2 owns N = D*b/16 bytes stored in pieces of
 * P = min(16, N) bytes (lane byte n at (n/P)*32*P + lane*P + n mod P); word
 * (k/8)*W + (d/8)/E of the lane with W = D*b/128; bit
 * 16*(k mod 2) + b*((d/8) mod E) of that word. */
void ora_v_code_place(int D, int b, int k, int d, int* byte_off, int* shift) {
  int E = 16 / b;
  int W = D * b / 128;
  int N = D * b / 16;
  int P = N < 16 ? N : 16;
  int lane = 4 * (d % 8) + (k % 8) / 2;
  int word = (k / 8) * W + (d / 8) / E;
  int bit = 16 * (k % 2) + b * ((d / 8) % E);
  int n = 4 * word + bit / 8;
  *byte_off = (n / P) * 32 * P + lane * P + (n % P);
  *shift = bit % 8;
}

static void put_code(uint8_t* byte, int shift, int b, unsigned code) {
  unsigned mask = ((1u << b) - 1u) << shift;
  *byte = (uint8_t)((*byte & ~mask) | ((code << shift) & mask));
}

static unsigned get_code(const uint8_t* byte, int shift, int b) {
  return ((unsigned)*byte >> shift) & ((1u << b) - 1u);
}

static int valid_shape(int D, int cap, int bk, int bv, int G) {
  if (D != 64 && D != 128) return 0;
  if (cap < 16 || cap % 16) return 0;
  if (bk != 2 && bk != 4 && bk != 8) return 0;
  if (bv != 2 && bv != 4 && bv != 8) return 0;
  if (G != 32 && G != 64 && G != 128) return 0;
  if (G > D) return 0;
  return 1;
}

/* In-place unnormalised Walsh-Hadamard transform of n = 2^m binary32 values:
 * for h = 1, 2, 4, ..., n/2 and every pair (i, i+h) with i & h == 0,
 * (x[i], x[i+h]) <- (x[i] + x[i+h], x[i] - x[i+h]), each a binary32
 * operation rounded to nearest even.  The result is H x with
 * H[i][j] = (-1)^popcount(i & j); the stage order fixes the rounding. */
void ora_fwht(float* x, int n) {
  for (int h = 1; h < n; h *= 2)
    for (int i = 0; i < n; ++i)
      if ((i & h) == 0) {
        float a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
}

/* The same transform in binary64 (used on queries). */
static void fwht_d(double* x, int n) {
  for (int h = 1; h < n; h *= 2)
    for (int i = 0; i < n; ++i)
      if ((i & h) == 0) {
        double a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
}

/* Quantize-append into host copies of the four cache arrays, with the same
 * argument meaning as the library call: k, v are [B][Hkv][n_new][D] of
 * dtype, batch row b writes positions pos[b] .. pos[b]+n_new-1.  A batch row
 * whose range leaves [0, cap) is skipped.  Returns the flags: 1 = past
 * capacity, 8 = negative position; -1 for an invalid shape. */
int ora_quantize_append_g2(int B, int Hkv, int D, int cap, int bk, int bv, int Gk, int Gv,
                           uint8_t* k_codes, uint8_t* v_codes, uint16_t* k_params,
                           uint16_t* v_params, const void* k, const void* v,
                           int dtype, const int32_t* pos, int n_new, int rotate_keys) {
  if (!valid_shape(D, cap, bk, bv, Gk) || !valid_shape(D, cap, bk, bv, Gv)) return -1;
  int flags = 0;
  size_t krow = (size_t)D * bk / 8;
  size_t vtile = (size_t)2 * D * bv;
  float* x = (float*)malloc(sizeof(float) * D);
  uint8_t* codes = (uint8_t*)malloc(D);
  for (int b = 0; b < B; ++b) {
    if (pos[b] < 0) {
      flags |= 8;
      continue;
    }
    if ((long)pos[b] + n_new > cap) {
      flags |= 1;
      continue;
    }
    for (int h = 0; h < Hkv; ++h) {
      size_t slot = (size_t)b * Hkv + h;
      for (int i = 0; i < n_new; ++i) {
        int p = pos[b] + i;
        size_t src = ((slot * n_new) + i) * D;
        for (int which = 0; which < 2; ++which) {
          const void* in = which == 0 ? k : v;
          int bits = which == 0 ? bk : bv;
          int G = which == 0 ? Gk : Gv;
          int NG = D / G;
          uint16_t* params = which == 0 ? k_params : v_params;
          for (int d = 0; d < D; ++d) x[d] = load_elem(in, dtype, src + d);
          if (which == 0 && rotate_keys) ora_fwht(x, D);
          for (int g = 0; g < NG; ++g) {
            float s32, m32;
            uint16_t s16, z16;
            ora_quantize_group(x + g * G, G, bits, codes + g * G, &s32, &m32,
                               &s16, &z16);
            size_t pp = ((slot * cap + p) * NG + g) * 2;
            params[pp] = s16;
            params[pp + 1] = z16;
          }
          for (int d = 0; d < D; ++d) {
            int off, sh;
            if (which == 0) {
              ora_k_code_place(D, bits, d, &off, &sh);
              put_code(k_codes + slot * cap * krow + (size_t)p * krow + off,
                       sh, bits, codes[d]);
            } else {
              ora_v_code_place(D, bits, p % 16, d, &off, &sh);
              put_code(v_codes + slot * cap / 16 * vtile + (size_t)(p / 16) * vtile + off,
                       sh, bits, codes[d]);
            }
          }
        }
      }
    }
  }
  free(x);
  free(codes);
  return flags;
}

int ora_quantize_append_ex(int B, int Hkv, int D, int cap, int bk, int bv, int G,
                           uint8_t* k_codes, uint8_t* v_codes, uint16_t* k_params,
                           uint16_t* v_params, const void* k, const void* v,
                           int dtype, const int32_t* pos, int n_new, int rotate_keys) {
  return ora_quantize_append_g2(B, Hkv, D, cap, bk, bv, G, G, k_codes, v_codes, k_params,
                                v_params, k, v, dtype, pos, n_new, rotate_keys);
}

int ora_quantize_append(int B, int Hkv, int D, int cap, int bk, int bv, int G,
                        uint8_t* k_codes, uint8_t* v_codes, uint16_t* k_params,
                        uint16_t* v_params, const void* k, const void* v,
                        int dtype, const int32_t* pos, int n_new) {
  return ora_quantize_append_ex(B, Hkv, D, cap, bk, bv, G, k_codes, v_codes, k_params,
                                v_params, k, v, dtype, pos, n_new, 0);
}

/* Codes of position p of slot (b, h): which = 0 for K, 1 for V. */
void ora_read_codes(int Hkv, int D, int cap, int bk, int bv, const uint8_t* k_codes,
                    const uint8_t* v_codes, int which, int b, int h, int p,
                    uint8_t* codes) {
  size_t slot = (size_t)b * Hkv + h;
  int bits = which == 0 ? bk : bv;
  for (int d = 0; d < D; ++d) {
    int off, sh;
    if (which == 0) {
      size_t krow = (size_t)D * bk / 8;
      ora_k_code_place(D, bits, d, &off, &sh);
      codes[d] = (uint8_t)get_code(k_codes + slot * cap * krow + (size_t)p * krow + off, sh, bits);
    } else {
      size_t vtile = (size_t)2 * D * bv;
      ora_v_code_place(D, bits, p % 16, d, &off, &sh);
      codes[d] = (uint8_t)get_code(v_codes + slot * cap / 16 * vtile + (size_t)(p / 16) * vtile + off,
                                   sh, bits);
    }
  }
}

/* Dequantised row: x^_d = code_d * scale16 + zero16, in binary32.  G is the
 * group size of the array read (which = 0: keys, 1: values). */
void ora_dequant_row(int Hkv, int D, int cap, int bk, int bv, int G,
                     const uint8_t* k_codes, const uint8_t* v_codes,
                     const uint16_t* k_params, const uint16_t* v_params,
                     int which, int b, int h, int p, float* out) {
  uint8_t codes[128];
  ora_read_codes(Hkv, D, cap, bk, bv, k_codes, v_codes, which, b, h, p, codes);
  const uint16_t* params = which == 0 ? k_params : v_params;
  int NG = D / G;
  size_t slot = (size_t)b * Hkv + h;
  for (int d = 0; d < D; ++d) {
    size_t pp = ((slot * cap + p) * NG + d / G) * 2;
    float scale = ora_f16_to_f32(params[pp]);
    float zero = ora_f16_to_f32(params[pp + 1]);
    float prod = (float)codes[d] * scale;
    out[d] = prod + zero;
  }
}

/* ------------------------------------------------------------- attention */

/* softmax(s) v for one query head, binary64.  k_rows/v_rows are len x D. */
static void attend(int D, int len, const double* q, const float* k_rows,
                   const float* v_rows, double sm_scale, double* out) {
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (len <= 0) return;
  double* s = (double*)malloc(sizeof(double) * len);
  double m = -INFINITY;
  for (int t = 0; t < len; ++t) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += q[d] * (double)k_rows[(size_t)t * D + d];
    s[t] = acc * sm_scale;
    if (s[t] > m) m = s[t];
  }
  double l = 0.0;
  for (int t = 0; t < len; ++t) {
    double p = exp(s[t] - m);
    l += p;
    for (int d = 0; d < D; ++d) out[d] += p * (double)v_rows[(size_t)t * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= l;
  free(s);
}

/* One decode step over the packed cache: out[B][Hq][D] in binary64.
 * Batch row b attends to positions [0, min(seq_lens[b], max_len, cap)).
 * sm_scale <= 0 selects 1/sqrt(D).  Returns 2 if a length was clamped,
 * -1 on an invalid shape, else 0. */
int ora_decode_attention_g2(int B, int Hkv, int D, int cap, int bk, int bv, int Gk, int Gv,
                            const uint8_t* k_codes, const uint8_t* v_codes,
                            const uint16_t* k_params, const uint16_t* v_params,
                            const void* q, int q_dtype, int Hq,
                            const int32_t* seq_lens, int max_len, float sm_scale,
                            int rotate_keys, double* out) {
  if (!valid_shape(D, cap, bk, bv, Gk) || !valid_shape(D, cap, bk, bv, Gv) || Hq % Hkv)
    return -1;
  int flags = 0;
  int gq = Hq / Hkv;
  double scale = sm_scale > 0.0f ? (double)sm_scale : 1.0 / sqrt((double)D);
  double* qd = (double*)malloc(sizeof(double) * D);
  for (int b = 0; b < B; ++b) {
    int len = seq_lens[b];
    if (len < 0) len = 0;
    int lim = max_len < cap ? max_len : cap;
    if (len > lim) {
      len = lim;
      flags |= 2;
    }
    for (int h = 0; h < Hkv; ++h) {
      float* kr = (float*)malloc(sizeof(float) * (size_t)(len > 0 ? len : 1) * D);
      float* vr = (float*)malloc(sizeof(float) * (size_t)(len > 0 ? len : 1) * D);
      for (int t = 0; t < len; ++t) {
        ora_dequant_row(Hkv, D, cap, bk, bv, Gk, k_codes, v_codes, k_params, v_params,
                        0, b, h, t, kr + (size_t)t * D);
        ora_dequant_row(Hkv, D, cap, bk, bv, Gv, k_codes, v_codes, k_params, v_params,
                        1, b, h, t, vr + (size_t)t * D);
      }
      for (int j = 0; j < gq; ++j) {
        int hq = h * gq + j;
        for (int d = 0; d < D; ++d)
          qd[d] = load_elem(q, q_dtype, ((size_t)b * Hq + hq) * D + d);
        if (rotate_keys) {
          /* keys are stored rotated: use H q / D */
          fwht_d(qd, D);
          for (int d = 0; d < D; ++d) qd[d] /= (double)D;
        }
        attend(D, len, qd, kr, vr, scale, out + ((size_t)b * Hq + hq) * D);
      }
      free(kr);
      free(vr);
    }
  }
  free(qd);
  return flags;
}

int ora_decode_attention_ex(int B, int Hkv, int D, int cap, int bk, int bv, int G,
                            const uint8_t* k_codes, const uint8_t* v_codes,
                            const uint16_t* k_params, const uint16_t* v_params,
                            const void* q, int q_dtype, int Hq,
                            const int32_t* seq_lens, int max_len, float sm_scale,
                            int rotate_keys, double* out) {
  return ora_decode_attention_g2(B, Hkv, D, cap, bk, bv, G, G, k_codes, v_codes, k_params,
                                 v_params, q, q_dtype, Hq, seq_lens, max_len, sm_scale,
                                 rotate_keys, out);
}

int ora_decode_attention(int B, int Hkv, int D, int cap, int bk, int bv, int G,
                         const uint8_t* k_codes, const uint8_t* v_codes,
                         const uint16_t* k_params, const uint16_t* v_params,
                         const void* q, int q_dtype, int Hq,
                         const int32_t* seq_lens, int max_len, float sm_scale,
                         double* out) {
  return ora_decode_attention_ex(B, Hkv, D, cap, bk, bv, G, k_codes, v_codes, k_params,
                                 v_params, q, q_dtype, Hq, seq_lens, max_len, sm_scale, 0, out);
}

/* Attention on unquantised K/V, [B][Hkv][T][D] of kv_dtype, binary64. */
int ora_attention_dense(int B, int Hkv, int D, int T, const void* k,
                        const void* v, int kv_dtype, const void* q, int q_dtype,
                        int Hq, const int32_t* seq_lens, float sm_scale,
                        double* out) {
  if (Hq % Hkv) return -1;
  int gq = Hq / Hkv;
  double scale = sm_scale > 0.0f ? (double)sm_scale : 1.0 / sqrt((double)D);
  double* qd = (double*)malloc(sizeof(double) * D);
  for (int b = 0; b < B; ++b) {
    int len = seq_lens[b] < T ? seq_lens[b] : T;
    for (int h = 0; h < Hkv; ++h) {
      size_t n = (size_t)(len > 0 ? len : 1) * D;
      float* kr = (float*)malloc(sizeof(float) * n);
      float* vr = (float*)malloc(sizeof(float) * n);
      size_t base = ((size_t)b * Hkv + h) * (size_t)T * D;
      for (size_t i = 0; i < (size_t)len * D; ++i) {
        kr[i] = load_elem(k, kv_dtype, base + i);
        vr[i] = load_elem(v, kv_dtype, base + i);
      }
      for (int j = 0; j < gq; ++j) {
        int hq = h * gq + j;
        for (int d = 0; d < D; ++d)
          qd[d] = load_elem(q, q_dtype, ((size_t)b * Hq + hq) * D + d);
        attend(D, len, qd, kr, vr, scale, out + ((size_t)b * Hq + hq) * D);
      }
      free(kr);
      free(vr);
    }
  }
  free(qd);
  return 0;
}
