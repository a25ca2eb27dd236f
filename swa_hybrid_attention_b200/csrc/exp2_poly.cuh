// 2^x on the FMA pipe, used for part of the softmax exponentials so that the
// MUFU (special-function) pipe is not the bottleneck of the attention kernel.
//
// Method: Cody–Waite style range reduction x = n + f with n = round(x) and
// f in [-1/2, 1/2] (the rounding uses the 1.5 * 2^23 shifter), a cubic
// polynomial p(f) ~ 2^f whose coefficients minimise the maximum relative
// error on [-1/2, 1/2] (found here with a Remez exchange: max relative error
// 7.5e-5, evaluated by Horner in fp32), and 2^n applied by adding n to the
// exponent field.  Valid for x <= 127; inputs below -125 return 0 (the
// softmax feeds x <= 8 and -inf for masked keys).  The attention
// probabilities are rounded to bf16 (relative step 2^-8) right after, so the
// polynomial error is far below what reaches the MMA.
#pragma once
#include <cstdint>

namespace rtp {

__device__ __forceinline__ float exp2_poly(float x) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  const float xc = fmaxf(x, -125.0f);
  const float t = __fadd_rn(xc, kShift);
  const int n = __float_as_int(t) - 0x4B400000;
  const float f = __fsub_rn(xc, __fsub_rn(t, kShift));
  float p = fmaf(0.0551716685f, f, 0.242611125f);
  p = fmaf(p, f, 0.693260968f);
  p = fmaf(p, f, 0.999928057f);
  const float r = __int_as_float(__float_as_int(p) + static_cast<int>(static_cast<unsigned>(n) << 23));
  return x < -125.0f ? 0.0f : r;
}

// ------------------------------------------------------------------ packed
// Two fp32 values in one 64-bit register pair, for the sm_100 packed f32x2
// instructions (one issue slot for two lanes' worth of arithmetic).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2_poly on two values at once (same method and error as exp2_poly; the
// inputs are clamped to >= -125, so tiny results come out as ~2^-125, not 0).
__device__ __forceinline__ uint64_t exp2_poly2(float xa, float xb) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  const uint64_t x = pack2(fmaxf(xa, -125.0f), fmaxf(xb, -125.0f));
  const uint64_t t = add2(x, pack2(kShift, kShift));       // round to integer n
  const uint64_t n = add2(t, pack2(-kShift, -kShift));     // n, exact
  const uint64_t f = fma2(n, pack2(-1.0f, -1.0f), x);      // x - n, exact, in [-1/2, 1/2]
  uint64_t p = fma2(pack2(0.0551716685f, 0.0551716685f), f, pack2(0.242611125f, 0.242611125f));
  p = fma2(p, f, pack2(0.693260968f, 0.693260968f));
  p = fma2(p, f, pack2(0.999928057f, 0.999928057f));
  // 2^n: the low bits of t hold n + 2^22; shifting by 23 leaves n << 23 (mod 2^32)
  const uint32_t lo = static_cast<uint32_t>(p) + (static_cast<uint32_t>(t) << 23);
  const uint32_t hi = static_cast<uint32_t>(p >> 32) + (static_cast<uint32_t>(t >> 32) << 23);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

}  // namespace rtp
