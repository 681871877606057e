// Device helpers shared by the kvq kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "internal.h"
#include "kvq.h"

namespace kvq {

// ------------------------------------------------------------------ inputs
// Eight consecutive elements of an input row widened exactly to binary32.
template <typename T>
struct Load8;

template <>
struct Load8<float> {
  static __device__ __forceinline__ void run(const float* p, float x[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

template <>
struct Load8<__nv_bfloat16> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* p, float x[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

template <>
struct Load8<__half> {
  static __device__ __forceinline__ void run(const __half* p, float x[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 f = __half22float2(h);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
};

// One element of Q (or any input) widened to binary32.
__device__ __forceinline__ float load_elem(const void* base, int dtype, size_t i) {
  if (dtype == KVQ_F32) return __ldg(reinterpret_cast<const float*>(base) + i);
  const unsigned short u = __ldg(reinterpret_cast<const unsigned short*>(base) + i);
  if (dtype == KVQ_BF16) return __uint_as_float(static_cast<uint32_t>(u) << 16);
  return __half2float(__ushort_as_half(u));
}

// One attention output element in the caller's type.
__device__ __forceinline__ void store_out(void* out, int dtype, size_t i, float v) {
  if (dtype == KVQ_F32)
    reinterpret_cast<float*>(out)[i] = v;
  else if (dtype == KVQ_BF16)
    reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<__half*>(out)[i] = __float2half_rn(v);
}

// --------------------------------------------------------------- error word
__device__ __forceinline__ void flag_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

// ------------------------------------------------ balanced decode schedule
// off[r] = units * sum_{r' < r} ceil(len_r' / T) for r = 0 .. kStreamRows,
// with each length clamped to [0, lim] (rows past `batch` count nothing);
// lens (when not NULL): the raw lengths, kStreamRows entries (0 past
// `batch`).  Reads only the lengths, so it may run before the wait for the
// previous grid.  Called by all 128 threads of the CTA; wsum: 4 ints of
// shared scratch.  Ends with a CTA barrier.
__device__ __forceinline__ void stream_row_offsets(const int32_t* seq_lens, int batch, int lim,
                                                   int units, int T, int* off, int* lens,
                                                   int* wsum) {
  constexpr int R = kStreamRows / 128;
  int cnt[R], tot = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int r = R * threadIdx.x + i;
    const int raw = r < batch ? seq_lens[r] : 0;
    if (lens != nullptr) lens[r] = raw;
    const int len = max(0, min(raw, lim));
    cnt[i] = units * ((len + T - 1) / T);
    tot += cnt[i];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = tot;  // inclusive scan of the threads' totals within the warp
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, m);
    if (lane >= m) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = incl - tot;
  for (int w = 0; w < warp; ++w) before += wsum[w];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    off[R * threadIdx.x + i] = before;
    before += cnt[i];
  }
  if (threadIdx.x == 127) off[kStreamRows] = before;
  __syncthreads();
}

// ------------------------------------------------- mbarrier / bulk copies
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
      : "memory");
}

// Raises the current phase's expected transaction bytes without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_addr(bar)),
      "r"(bytes)
      : "memory");
}

// Test for the completion of the phase with the given parity; the thread may
// be suspended (up to the hint, in nanoseconds) until it completes, so that
// waiting warps do not spin on the issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Longest a pipeline wait may take before the kernel gives up (1 s), unless
// the launch carries a shorter limit (the failure-detection test knob).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Slow path of mbar_wait_bounded: keep waiting, up to limit_ns.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, uint32_t* err,
                                                   uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      flag_error(err, KVQ_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait on an mbarrier phase: returns false (and flags
// KVQ_DEVERR_TIMEOUT) if the phase did not complete within limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t* err,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, err, limit_ns);
}

// Programmatic dependent launch.  pdl_wait() blocks until every grid this
// one depends on has completed and its writes are visible; it returns at once
// when the launch carried no such dependency.  Every global read of an input
// and every global write comes after it.  pdl_trigger() lets the next grid in
// the stream begin launching; its blocks then hold in their own pdl_wait().
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The same for global memory: generic-proxy stores to the cache before later
// bulk copies that read them.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 1-D bulk copy global -> shared (no multicast), completion counted in bytes
// on `bar`.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, a multiple
// of 16 bytes); no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------------------ tensor cores
// D = A * B + C, m16n8k16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^e as a binary32 value, for e in [-126, 127] (exact).
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// 2^x, hardware approximation (relative error ~2^-22; results below 2^-126
// flush to zero), for softmax weights.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two binary32 values rounded to binary16 (nearest even) in one register:
// lo in bits 0..15, hi in bits 16..31.
__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return static_cast<uint32_t>(__half_as_ushort(lo)) |
         (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t u) {
  __half2 h = *reinterpret_cast<__half2*>(&u);
  return __half22float2(h);
}

}  // namespace kvq
