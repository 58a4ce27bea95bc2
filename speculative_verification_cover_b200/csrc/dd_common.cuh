// Shared device-side pieces of libdd: the device error word, bounded
// waits, the Philox4x32-10 generator, and small numeric helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dd.h"

namespace dd {

// ---------------------------------------------------------------------------
// Device error word: a kernel whose bounded wait runs out records a dd_status
// here (first writer wins) and returns; dd_get_device_error() reads and clears
// it from the host. (libdd is built as one translation unit, libdd.cu, so the
// definition lives here.)
__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_error(unsigned int code) {
  atomicCAS(&g_device_error, 0u, code);
}

// ---------------------------------------------------------------------------
// mbarrier helpers (shared::cta). Every wait is bounded by `limit`
// iterations and by kWaitNs of wall time (a try_wait may suspend the thread
// for a while, so iterations alone do not bound the time); on expiry it
// records DD_ERR_TIMEOUT and returns false.
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// A waiting thread is suspended by the hardware until the phase completes or
// the hint (ns) runs out, so waiting warps take no issue slots from the warps
// that share their SM sub-partition.
constexpr uint32_t kSuspendHintNs = 1000000u;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t phase, uint32_t limit) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1; it < limit; ++it) {
    if (mbar_try_wait(bar, phase)) return true;
    if (global_ns() - t0 > kWaitNs) break;
  }
  record_error(DD_ERR_TIMEOUT);
  return false;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of
//   (x0,x1,x2,x3) -> (hi(M1*x2)^x1^k0, lo(M1*x2), hi(M0*x0)^x3^k1, lo(M0*x0))
// with the key bumped by the Weyl increments after each round.
struct PhiloxOut { uint32_t w[4]; };

__device__ __forceinline__ PhiloxOut philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                   uint32_t c3, uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = M0 * c0, hi0 = __umulhi(M0, c0);
    const uint32_t lo1 = M1 * c2, hi1 = __umulhi(M1, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += W0; k1 += W1;
  }
  PhiloxOut o;
  o.w[0] = c0; o.w[1] = c1; o.w[2] = c2; o.w[3] = c3;
  return o;
}

// U = (2*(w >> 9) + 1) * 2^-24, exact in fp32, in (0, 1).
__device__ __forceinline__ float uniform_from_word(uint32_t w) {
  return __uint2float_rn(2u * (w >> 9) + 1u) * 5.9604644775390625e-08f;
}

// g = -ln(-ln U). The inner log must be accurate in *relative* terms near
// U = 1 (where -ln U is tiny and the Gumbel value is large), so it uses the
// full-precision logf; the outer one only needs absolute accuracy.
__device__ __forceinline__ float gumbel_from_word(uint32_t w) {
  const float u = uniform_from_word(w);
  const float e = -logf(u);
  return -__logf(e);
}

// An upper bound of gumbel_from_word(w) as computed above (its fp32 result),
// cheap enough to screen every entry: -ln(-ln U) <= -ln(1 - U) since
// -ln U >= 1 - U on (0, 1). With k = w >> 9, 1 - U = (j + 1/2) 2^-23 exactly for
// j = 2^23 - 1 - k, so -ln(1 - U) = ln2 (23 - log2(j + 1/2)); j + 1/2 is formed
// exactly from the float with bits (2^23 + j) minus (2^23 - 1/2). The 0.01
// margin covers the approximate log2 here (about 4e-6 absolute) and the fp32
// rounding of the exact path (about 1e-5): the bound is never below it.
__device__ __forceinline__ float gumbel_bound_from_word(uint32_t w) {
  const float jh = __uint_as_float((w >> 9) ^ 0x4B7FFFFFu) - 8388607.5f;
  return fmaf(__log2f(jh), -0.69314718f, 23.f * 0.69314718f + 0.01f);
}

// Monotone map of floats (no NaN) onto signed integers, for integer max reductions.
__device__ __forceinline__ int float_to_ordered(float x) {
  const int i = __float_as_int(x);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ordered_to_float(int i) {
  return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF);
}

// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace dd
