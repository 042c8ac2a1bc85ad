// pa_fastmath.cuh -- packed fp32 arithmetic and exp2 for the softmax of the
// tensor-core prefill kernel (sm_100a).
//
// sm_100a executes fp32 add / sub / mul / fma on a pair of values held in one
// 64-bit register pair (the .f32x2 forms), and max over three fp32 operands,
// in one instruction each; the softmax uses them to halve its instruction
// count.  The exponential unit (ex2) delivers 16 results per clock per SM,
// which for a 128 x 128 score tile pair is as many cycles as the tensor cores
// need for the tile's two MMAs, so exp2_poly2 evaluates part of the
// exponentials on the FMA pipe instead.
#pragma once

#include <stdint.h>

namespace pa {

// ------------------------------------------------------------ packed pairs
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ void u2_split(uint64_t v, uint32_t& lo, uint32_t& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t u2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// the same fp32 constant in both lanes
__host__ __device__ constexpr uint64_t dup_bits(uint32_t bits) {
  return ((uint64_t)bits << 32) | bits;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// exponential unit, flushing subnormal results to zero (ex2(-inf) = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x in both lanes, without the exponential unit.
//
// Range reduction after Cody and Waite (1980): x = n + f with n = round(x)
// and f in [-1/2, 1/2].  Adding 1.5 * 2^23 rounds x to an integer (the fp32
// spacing there is 1) and leaves n in the low mantissa bits; subtracting it
// again gives n exactly, and x - n gives f exactly.  2^f is a degree-3
// polynomial whose coefficients minimise the relative error on [-1/2, 1/2]
// (Remez exchange; the fit is reproduced by fit_exp2_poly.py in the package):
// at most 7.5e-5 in fp32 arithmetic, well under the 2^-9 relative rounding of
// the bf16 P that the result becomes.  Multiplying by 2^n adds n to the
// exponent field, as in Schraudolph's exponent-field construction (1999):
// the low 9 bits of the rounded sum's bit pattern are n in two's complement,
// so shifting that bit pattern left by 23 gives n << 23 modulo 2^32.
//
// Inputs are clamped at -126 so that the exponent field stays in range;
// -inf (a masked score) and anything below -126 therefore give at most
// 2^-126 instead of 0, which is below every weight that matters.  Between
// -126 and -125 a polynomial factor just below 1 lands on a subnormal
// encoding (relative error up to 1.5e-4 there).  Inputs
// are at most 2^8 here (scores minus a running max that trails by at most
// 8), far inside the exponent range.
constexpr uint64_t kExp2Round = dup_bits(0x4B400000u);  // 1.5 * 2^23
constexpr uint64_t kExp2C0 = dup_bits(0x3F7FFB49u);     // 0.99992806
constexpr uint64_t kExp2C1 = dup_bits(0x3F31798Du);     // 0.69326097
constexpr uint64_t kExp2C2 = dup_bits(0x3E786F0Du);     // 0.24261113
constexpr uint64_t kExp2C3 = dup_bits(0x3D61FBB0u);     // 0.05517167
constexpr float kExp2Floor = -126.0f;

__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  float x0, x1;
  f2_split(x, x0, x1);
  const uint64_t xc = f2(fmaxf(x0, kExp2Floor), fmaxf(x1, kExp2Floor));
  const uint64_t t = add2(xc, kExp2Round);         // 1.5 * 2^23 + n
  const uint64_t f = sub2(xc, sub2(t, kExp2Round));  // x - n
  uint64_t p = fma2(kExp2C3, f, kExp2C2);
  p = fma2(p, f, kExp2C1);
  p = fma2(p, f, kExp2C0);
  uint32_t t0, t1, p0, p1;
  u2_split(t, t0, t1);
  u2_split(p, p0, p1);
  return u2(p0 + (t0 << 23), p1 + (t1 << 23));
}

}  // namespace pa
