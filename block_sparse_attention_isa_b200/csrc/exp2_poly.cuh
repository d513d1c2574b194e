// Packed fp32x2 arithmetic and a polynomial 2^x on the FMA pipe.
//
// The softmax of the attention kernel needs 2^x for every score. The special
// function unit (ex2.approx) has a fraction of the FMA pipe's throughput, so a
// share of the exponentials is computed here instead, with the classic
// Cody-Waite style split:
//   x = n + f, n = round(x) (by adding and subtracting 1.5 * 2^23), f in [-1/2, 1/2],
//   2^x = 2^n * p(f), p a cubic fitted to 2^f on [-1/2, 1/2] by iteratively
//   reweighted least squares on the relative error (max relative error 7.5e-5
//   in float32 Horner form), 2^n applied by adding n to the exponent field.
// Inputs are clamped to >= -125 so that the result stays a normal float (2^-125
// is far below anything a bfloat16 P can resolve next to the row maximum).
// Accuracy is checked against the CUDA exp2f function in the GPU test suite.
#pragma once
#include <cstdint>

namespace isa {

__device__ __forceinline__ uint64_t pack2(float a, float b) {
  return static_cast<uint64_t>(__float_as_uint(a)) | (static_cast<uint64_t>(__float_as_uint(b)) << 32);
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Coefficients of the cubic p(f) ~ 2^f on [-1/2, 1/2] (own fit, see above).
constexpr float kExp2C0 = 0.99992805719375610f;
constexpr float kExp2C1 = 0.69326096773147583f;
constexpr float kExp2C2 = 0.24261112511157990f;
constexpr float kExp2C3 = 0.05517166852951050f;
constexpr float kRoundShift = 12582912.0f;  // 1.5 * 2^23

// 2^x for a pair of floats (x <= 2^22), both lanes on the FMA / integer pipes.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  const float x0 = fmaxf(lo2(x), -125.0f), x1 = fmaxf(hi2(x), -125.0f);
  const uint64_t xc = pack2(x0, x1);
  const uint64_t j = fadd2(xc, pack2(kRoundShift, kRoundShift));         // round(x) in the low mantissa bits
  const uint64_t n = fadd2(j, pack2(-kRoundShift, -kRoundShift));        // round(x) as a float
  const uint64_t f = ffma2(n, pack2(-1.0f, -1.0f), xc);                  // x - round(x), in [-1/2, 1/2]
  uint64_t p = ffma2(pack2(kExp2C3, kExp2C3), f, pack2(kExp2C2, kExp2C2));
  p = ffma2(p, f, pack2(kExp2C1, kExp2C1));
  p = ffma2(p, f, pack2(kExp2C0, kExp2C0));
  // add n to the exponent field: (bits(j) << 23) == n << 23 modulo 2^32
  const uint32_t r0 = static_cast<uint32_t>(p) + (static_cast<uint32_t>(j) << 23);
  const uint32_t r1 = static_cast<uint32_t>(p >> 32) + (static_cast<uint32_t>(j >> 32) << 23);
  return static_cast<uint64_t>(r0) | (static_cast<uint64_t>(r1) << 32);
}

// Scalar form (used by the self-test).
__device__ __forceinline__ float exp2_poly(float x) {
  return lo2(exp2_poly2(pack2(x, x)));
}

}  // namespace isa
