// Packed two-lane fp32 arithmetic (sm_100a .f32x2) and an exp2 evaluated on
// the FMA pipe, used to take part of the softmax's exponentials off the
// special-function unit.
//
// exp2 method: range reduction x = n + f with n = round(x) (computed by adding
// 1.5 * 2^23, which leaves n in the low mantissa bits) and f in [-1/2, 1/2];
// 2^f from a degree-3 polynomial whose coefficients minimise the maximum
// relative error on [-1/2, 1/2] (Remez exchange; gen_exp2_poly.py prints them:
// max relative error 7.5e-5, far below the 2^-9 rounding of the bf16 P it
// feeds); 2^n is applied by adding n to the exponent field. Inputs must be
// >= -125 (callers clamp), so 2^n stays a normal number.
#pragma once
#include <cstdint>

namespace sa {

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Polynomial coefficients for 2^f on [-1/2, 1/2] (gen_exp2_poly.py 3).
constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426111251e-01f;
constexpr float kExp2C3 = 5.517166853e-02f;

// 2^x for both lanes of x (each lane >= -125).
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x) {
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);       // 1.5 * 2^23
  const uint64_t neg_magic = f2_pack(-12582912.0f, -12582912.0f);
  const uint64_t t = f2_add(x, magic);           // n in the low mantissa bits
  const uint64_t n = f2_add(t, neg_magic);       // round(x) as a float
  const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), x);  // x - n in [-1/2, 1/2]
  uint64_t p = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(kExp2C0, kExp2C0));
  float p_lo, p_hi, t_lo, t_hi;
  f2_unpack(p, p_lo, p_hi);
  f2_unpack(t, t_lo, t_hi);
  // exponent += n; the bits of 1.5 * 2^23 itself shift out of the word
  const uint32_t r_lo = __float_as_uint(p_lo) + (__float_as_uint(t_lo) << 23);
  const uint32_t r_hi = __float_as_uint(p_hi) + (__float_as_uint(t_hi) << 23);
  return f2_pack(__uint_as_float(r_lo), __uint_as_float(r_hi));
}

// Degree-5 coefficients (gen_exp2_poly.py 5): max relative error 1.5e-7
// after rounding them to fp32, on a par with ex2.approx; for sums that must
// keep fp32-level accuracy.
constexpr float kExp2D0 = 1.000000119e+00f;
constexpr float kExp2D1 = 6.931469440e-01f;
constexpr float kExp2D2 = 2.402212024e-01f;
constexpr float kExp2D3 = 5.550713092e-02f;
constexpr float kExp2D4 = 9.675540961e-03f;
constexpr float kExp2D5 = 1.327647245e-03f;

// 2^x for both lanes of x (each lane >= -125), degree-5 polynomial.
__device__ __forceinline__ uint64_t exp2_poly5_x2(uint64_t x) {
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);       // 1.5 * 2^23
  const uint64_t neg_magic = f2_pack(-12582912.0f, -12582912.0f);
  const uint64_t t = f2_add(x, magic);
  const uint64_t n = f2_add(t, neg_magic);
  const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), x);
  uint64_t p = f2_fma(f2_pack(kExp2D5, kExp2D5), f, f2_pack(kExp2D4, kExp2D4));
  p = f2_fma(p, f, f2_pack(kExp2D3, kExp2D3));
  p = f2_fma(p, f, f2_pack(kExp2D2, kExp2D2));
  p = f2_fma(p, f, f2_pack(kExp2D1, kExp2D1));
  p = f2_fma(p, f, f2_pack(kExp2D0, kExp2D0));
  float p_lo, p_hi, t_lo, t_hi;
  f2_unpack(p, p_lo, p_hi);
  f2_unpack(t, t_lo, t_hi);
  const uint32_t r_lo = __float_as_uint(p_lo) + (__float_as_uint(t_lo) << 23);
  const uint32_t r_hi = __float_as_uint(p_hi) + (__float_as_uint(t_hi) << 23);
  return f2_pack(__uint_as_float(r_lo), __uint_as_float(r_hi));
}

}  // namespace sa
