// exp2 for the softmax: the SFU instruction, and a polynomial on the FMA pipe
// for the share of elements the SFU cannot keep up with on sm_100a (the
// tensor cores outrun the 16-per-clock SFU; "the librarian" page, "FA4 --
// Blackwell's asymmetry", idea 1, runs a software exponential for this).
//
// Polynomial path (own implementation of two published methods, see
// gen_exp2_poly.py): Cody-Waite reduction x = n + f, n = round(x) via the
// 1.5 * 2^23 rounding constant, f in [-1/2, 1/2]; 2^f by the Remez minimax
// polynomial of fa_exp2_poly.h in Horner form with packed f32x2 FMAs; 2^n by
// adding n to the exponent field.  Inputs are clamped to >= -125 so that
// the result is always a normal number (at -126 the polynomial's value just
// below 1 would land in the subnormal range, where adding n to the exponent
// field no longer scales it); below the clamp the result is ~2.4e-38
// instead of 0, negligible next to the row sum (>= 1).
#pragma once

#include "fa_exp2_poly.h"
#include "fa_ptx.cuh"

namespace fa {

template <int DEG>
__device__ __forceinline__ float exp2_coef(int k) {
  if constexpr (DEG == 3) return exp2_poly3_coef(k);
  else if constexpr (DEG == 4) return exp2_poly4_coef(k);
  else return exp2_poly5_coef(k);
}

// 2^x for both halves of a packed pair, -125 <= x <= 126 (smaller x: 2^-125).
template <int DEG>
__device__ __forceinline__ uint64_t exp2_poly_f2(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  const uint64_t xc = f2_pack(x0, x1);
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);    // 1.5 * 2^23
  const uint64_t t = f2_add(xc, magic);                      // round(x) in the low bits
  const uint64_t f = f2_sub(xc, f2_sub(t, magic));           // x - round(x)
  uint64_t p = f2_pack(exp2_coef<DEG>(DEG), exp2_coef<DEG>(DEG));
#pragma unroll
  for (int k = DEG - 1; k >= 0; --k) p = f2_fma(p, f, f2_pack(exp2_coef<DEG>(k), exp2_coef<DEG>(k)));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  // bits(t) = bits(1.5 * 2^23) + n; shifting left by 23 leaves n << 23.
  const uint32_t r0 = __float_as_uint(p0) + (__float_as_uint(t0) << 23);
  const uint32_t r1 = __float_as_uint(p1) + (__float_as_uint(t1) << 23);
  return f2_pack(__uint_as_float(r0), __uint_as_float(r1));
}

__device__ __forceinline__ uint64_t exp2_sfu_f2(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  return f2_pack(ex2_sfu(x0), ex2_sfu(x1));
}

}  // namespace fa
