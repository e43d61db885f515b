// fs_device.cuh -- small sm_100a device helpers: packed fp32x2 arithmetic, the MUFU
// base-2 exponential, TMA bulk copies with mbarrier completion, and bounded waits.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fs {

typedef unsigned long long u64;

// Error bits OR-ed into the workspace error word by kernels.
constexpr unsigned kErrTimeout = 1u;

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Finite stand-in for log2(0): a zero weight or a padding column. Any exponent built
// on it stays near -1e30, so its term vanishes once a real column sets the row max.
constexpr float kLogZero = -1.0e30f;

// ---- packed fp32x2 (one instruction, two IEEE fp32 lanes) -------------------------------

__device__ __forceinline__ u64 pk(float lo, float hi) {
  u64 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk(u64 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ u64 add2(u64 a, u64 b) {
  u64 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 sub2(u64 a, u64 b) {
  u64 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
  u64 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x on the MUFU unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^t of both lanes on the FMA and integer pipes instead of the MUFU unit, for kernels whose
// MUFU unit is the bound while issue slots are free. t is clamped to [-125, ...) (smaller
// exponents give 2^-125 where ex2.approx.ftz gives 0: a term below 2^-125 of any sum that
// matters), rounded to the nearest integer j by adding 1.5 * 2^23 (j then sits in the low
// mantissa bits), and 2^(t - j), t - j in [-1/2, 1/2], is a degree-5 polynomial fitted to
// 2^f on that interval by iteratively reweighted least squares at Chebyshev nodes (relative
// error 2.1e-7 evaluated in fp32 by Horner's rule, checked over [-125, 9]); 2^j is added to
// its exponent field.
__device__ __forceinline__ u64 ex2_poly2(u64 t) {
  float a, b;
  upk(t, a, b);
  t = pk(fmaxf(a, -125.0f), fmaxf(b, -125.0f));
  const u64 magic = pk(12582912.0f, 12582912.0f);
  const u64 tm = add2(t, magic);
  const u64 f = sub2(t, sub2(tm, magic));
  u64 p = pk(1.327645150013268e-3f, 1.327645150013268e-3f);
  p = fma2(p, f, pk(9.675540961325169e-3f, 9.675540961325169e-3f));
  p = fma2(p, f, pk(5.550713464617729e-2f, 5.550713464617729e-2f));
  p = fma2(p, f, pk(2.4022120237350464e-1f, 2.4022120237350464e-1f));
  p = fma2(p, f, pk(6.931469440460205e-1f, 6.931469440460205e-1f));
  p = fma2(p, f, pk(1.0000001192092896f, 1.0000001192092896f));
  float pa, pb, ma, mb;
  upk(p, pa, pb);
  upk(tm, ma, mb);
  return pk(__uint_as_float(__float_as_uint(pa) + (__float_as_uint(ma) << 23)),
            __uint_as_float(__float_as_uint(pb) + (__float_as_uint(mb) << 23)));
}

// Asks L2 to fetch the line holding p (no register result, nothing waits for it).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---- shared-memory addresses, mbarriers and bulk copies ----------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Global -> shared bulk copy (TMA, no tensor map, no multicast); completion is
// signalled on `bar` as transaction bytes. dst, src and bytes must be 16-byte multiples.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_try_wait with a suspend-time hint: a waiting thread may sleep in hardware for up to
// hint_ns (until the phase completes) instead of returning at once, so a spinning warp
// issues far fewer instructions while it waits.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, giving up after `limit_ns` nanoseconds of
// %globaltimer (kWaitLimitNs unless a caller asks for less).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// ---- reductions -----------------------------------------------------------------------------

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_or(int v) {
  return __reduce_or_sync(0xffffffffu, static_cast<unsigned>(v));
}

// Max of nonnegative doubles via their bit patterns (order-preserving for x >= 0).
__device__ __forceinline__ void atomic_max_nonneg(double* addr, double v) {
  atomicMax(reinterpret_cast<unsigned long long*>(addr),
            static_cast<unsigned long long>(__double_as_longlong(v)));
}

}  // namespace fs
