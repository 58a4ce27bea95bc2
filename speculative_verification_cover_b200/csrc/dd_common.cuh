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

// Programmatic dependent launch. A kernel launched by launch_dependent() may be
// scheduled while the previous kernel on its stream is still finishing (once every
// CTA of that kernel has started); it calls pdl_wait() before it reads anything that
// kernel writes, or writes anything it reads. Without the launch attribute the wait
// returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel on the stream (launched with launch_dependent) be scheduled
// now, before this one finishes; it still waits in pdl_wait() for this kernel's data.
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;"); }

// Index checks of the checked build (compiled with DD_CHECK_BOUNDS). Written as
// `if (DD_IN_BOUNDS(i < n)) access;`: a false condition records DD_ERR_BOUNDS and
// the access is skipped. Without DD_CHECK_BOUNDS the macro is the constant true
// and the condition is not evaluated, so normal builds carry no cost.
#ifdef DD_CHECK_BOUNDS
__device__ __forceinline__ bool in_bounds_checked(bool ok) {
  if (!ok) record_error(DD_ERR_BOUNDS);
  return ok;
}
#define DD_IN_BOUNDS(cond) (::dd::in_bounds_checked(cond))
#else
#define DD_IN_BOUNDS(cond) true
#endif

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

// Hint: fetch the 128-byte line holding p into L2 (no register result, no fault on
// the addresses the kernels pass, which lie inside their input arrays).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// ---------------------------------------------------------------------------
// Philox4x32-10 split for a streaming pass over one row. In the counter
// (c0 = v >> 2, c1 = pos, c2 = b, c3 = step) only c0 changes along a row, and
// rounds 1 and 2 of the generator combine it with the fixed words in a way that
// leaves four of their eight products independent of c0. PhiloxRow holds those
// per-row parts (already xor-ed with the round keys), so a counter of the row
// costs 18 wide multiplies instead of 20; philox_row_counter() then runs
// rounds 3..10. The words are bit-identical to philox4x32_10().
constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u, kPhiloxW1 = 0xBB67AE85u;

struct PhiloxRow {
  uint32_t s1;   // c3 ^ k1 (round 1)
  uint32_t r1k;  // lo(M1 c2) ^ round-2 key 0
  uint32_t h2k;  // hi(M0 (hi(M1 c2) ^ c1 ^ k0)) ^ round-2 key 1
  uint32_t l2;   // lo(M0 (hi(M1 c2) ^ c1 ^ k0))
};

__device__ __forceinline__ PhiloxRow philox_row(uint32_t c1, uint32_t c2, uint32_t c3,
                                                uint32_t k0, uint32_t k1) {
  const uint64_t pb = (uint64_t)kPhiloxM1 * c2;
  const uint32_t x0 = (uint32_t)(pb >> 32) ^ c1 ^ k0;  // word 0 after round 1
  const uint32_t x1 = (uint32_t)pb;                    // word 1 after round 1
  const uint64_t p0 = (uint64_t)kPhiloxM0 * x0;        // round 2's first product
  PhiloxRow r;
  r.s1 = c3 ^ k1;
  r.r1k = x1 ^ (k0 + kPhiloxW0);
  r.h2k = (uint32_t)(p0 >> 32) ^ (k1 + kPhiloxW1);
  r.l2 = (uint32_t)p0;
  return r;
}

__device__ __forceinline__ PhiloxOut philox_row_counter(const PhiloxRow& r, uint32_t c0,
                                                        uint32_t k0, uint32_t k1) {
  // round 1: words 0, 1 are row constants; words 2, 3 come from M0 * c0
  const uint64_t p = (uint64_t)kPhiloxM0 * c0;
  const uint32_t x2 = (uint32_t)(p >> 32) ^ r.s1, x3 = (uint32_t)p;
  // round 2: M0 * word 0 is a row constant; M1 * word 2 is not
  const uint64_t q = (uint64_t)kPhiloxM1 * x2;
  uint32_t y0 = (uint32_t)(q >> 32) ^ r.r1k, y1 = (uint32_t)q;
  uint32_t y2 = r.h2k ^ x3, y3 = r.l2;
#pragma unroll
  for (int rd = 2; rd < 10; ++rd) {
    const uint32_t key0 = k0 + (uint32_t)rd * kPhiloxW0, key1 = k1 + (uint32_t)rd * kPhiloxW1;
    const uint64_t a = (uint64_t)kPhiloxM0 * y0, b = (uint64_t)kPhiloxM1 * y2;
    const uint32_t n0 = (uint32_t)(b >> 32) ^ y1 ^ key0, n2 = (uint32_t)(a >> 32) ^ y3 ^ key1;
    y0 = n0; y1 = (uint32_t)b; y2 = n2; y3 = (uint32_t)a;
  }
  PhiloxOut o;
  o.w[0] = y0; o.w[1] = y1; o.w[2] = y2; o.w[3] = y3;
  return o;
}

// ---------------------------------------------------------------------------
// Screening the Gumbel noise of a group of entries without computing it.
//
// gumbel_from_word(w) never exceeds kGumbelMax: U <= 1 - 2^-24, so
// -ln(-ln U) <= -ln(2^-24 (1 + 2^-25)) < 16.6356, and the fp32 evaluation adds
// far less than the 0.015 of headroom. An entry whose score could only beat a
// threshold with g > kGumbelMax needs no noise at all.
constexpr float kGumbelMax = 16.65f;

// For a required noise level G: every word w with gumbel_from_word(w) > G has
// j(w) + 1/2 < gumbel_screen_limit(G), where j(w) = 2^23 - 1 - (w >> 9) (so
// that 1 - U = (j + 1/2) 2^-23). Derivation: g > G means
//   1 - U < 1 - exp(-e^-G) <= e^-G,  i.e.  j + 1/2 < e^-G 2^23,
// and the limit returned is e^-(G - 0.01) 2^23: the 0.01 covers the fp32
// evaluation of gumbel_from_word (about 1e-6) and the approximate exp2 here
// (relative error below 2^-21). Words at or above the limit (in j) are screened
// out. Checked on the device over all 2^23 noise values by dd_selftest_gumbel_screen.
constexpr float kScreenSlack = 0.01f;
__device__ __forceinline__ float gumbel_screen_limit(float G) {
  return fast_exp2(fmaf(-G, 1.4426950408889634f, 23.f + kScreenSlack * 1.4426950408889634f));
}
// j of the largest word among several (the one whose noise could be largest), as
// an exact float: words w with larger w >> 9 have smaller j.
__device__ __forceinline__ float gumbel_screen_j(uint32_t wmax) {
  return __uint_as_float((0x7FFFFFu - (wmax >> 9)) | 0x4B000000u) - 8388608.f;
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


constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace dd
