// Packed fp32 arithmetic (sm_100 f32x2 instructions) and an exp2 that runs on
// the FMA pipe instead of the MUFU unit, used by the attention softmax to
// split the exponentials between the two pipes.
#pragma once
#include <cstdint>

namespace h3 {

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Hardware 2^x (MUFU).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for two values at once on the FMA/ALU pipes (inputs clamped at -125).
// Range reduction 2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2]
// (Cody & Waite style, the rounding done by adding 1.5 * 2^23), then 2^f from a
// cubic fitted to 2^f on [-1/2, 1/2] (Lawson-weighted least squares on
// Chebyshev nodes toward the minimax fit; max relative error 7.5e-5, far
// below the bf16 rounding the probabilities get next), and 2^n applied by
// adding n to the exponent field.
__device__ __forceinline__ uint64_t ex2_poly2(uint64_t x2) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  constexpr float kC0 = 0.99992806f, kC1 = 0.69326097f, kC2 = 0.24261113f, kC3 = 0.05517166f;
  float xl, xh;
  f2_unpack(x2, xl, xh);
  xl = fmaxf(xl, -125.0f);
  xh = fmaxf(xh, -125.0f);
  const uint64_t xc = f2_pack(xl, xh);
  const uint64_t magic = f2_pack(kMagic, kMagic);
  const uint64_t xr = f2_add(xc, magic);          // n in the low mantissa bits
  const uint64_t f = f2_sub(xc, f2_sub(xr, magic));
  uint64_t pl = f2_fma(f2_pack(kC3, kC3), f, f2_pack(kC2, kC2));
  pl = f2_fma(pl, f, f2_pack(kC1, kC1));
  pl = f2_fma(pl, f, f2_pack(kC0, kC0));
  float rl, rh, pl_lo, pl_hi;
  f2_unpack(xr, rl, rh);
  f2_unpack(pl, pl_lo, pl_hi);
  const uint32_t lo = __float_as_uint(pl_lo) + (__float_as_uint(rl) << 23);
  const uint32_t hi = __float_as_uint(pl_hi) + (__float_as_uint(rh) << 23);
  return f2_pack(__uint_as_float(lo), __uint_as_float(hi));
}

}  // namespace h3
