// swa_exp2.cuh - packed fp32 helpers and a base-2 exponential on the FMA pipe
// for the prefill softmax.
//
// The softmax needs one 2^x per visible (query, key) pair.  The SFU's
// MUFU.EX2 is fast per instruction but has only a quarter of the FMA pipe's
// lane throughput, and in a 128x128 tile of the attention it needs as many
// cycles as the tensor core needs for the tile's two matrix products.  So part
// of the exponentials are computed on the FMA pipe instead:
//
//   range reduction (Cody & Waite's split of the argument into an integer part
//   and a remainder):  n = round(x) by adding and subtracting 1.5 * 2^23, which
//   leaves n in the low mantissa bits of the sum;  f = x - n in [-1/2, 1/2];
//   2^f by a cubic  1 + f (c1 + f (c2 + f c3))  whose coefficients were fitted
//   for this file by iteratively reweighted least squares on the relative error
//   over [-1/2, 1/2] with p(0) = 1 (maximum relative error 1.02e-4, well below
//   the 2^-9 relative rounding of the bf16 probabilities that consume it);
//   2^n by adding n to the exponent field (an integer multiply-add of the
//   rounding sum's bit pattern by 2^23).
//
// Inputs must be at most +128.  Arguments below -126 (masked keys are -inf)
// give exactly 0, so a masked key contributes nothing, as on the SFU path;
// the polynomial itself only ever sees arguments in [-126, 128].
#pragma once

#include <stdint.h>

namespace swa {

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t x, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}

// a * b + c on two fp32 lanes at once
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

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x0, 2^x1 on the FMA pipe (see the file comment for the method and bounds).
__device__ __forceinline__ void exp2_fma_pipe(float& x0, float& x1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  constexpr float kC1 = 0.6932827830314636f;
  constexpr float kC2 = 0.2422090768814087f;
  constexpr float kC3 = 0.055008113384246826f;
  const uint64_t x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t round2 = f2_pack(kRound, kRound);
  const uint64_t j = f2_add(x, round2);                       // n in the low mantissa bits
  const uint64_t r = f2_sub(j, round2);                       // n as a float
  const uint64_t f = f2_sub(x, r);                            // remainder in [-1/2, 1/2]
  uint64_t p = f2_fma(f, f2_pack(kC3, kC3), f2_pack(kC2, kC2));
  p = f2_fma(p, f, f2_pack(kC1, kC1));
  p = f2_fma(p, f, f2_pack(1.f, 1.f));
  float p0, p1, j0, j1;
  f2_unpack(p, p0, p1);
  f2_unpack(j, j0, j1);
  // bits(2^n * p) = bits(p) + n * 2^23; the low bits of bits(j) are n (mod 2^9
  // after the shift), and unsigned arithmetic wraps as the two's complement needs.
  const float y0 = __uint_as_float(__float_as_uint(j0) * (1u << 23) + __float_as_uint(p0));
  const float y1 = __uint_as_float(__float_as_uint(j1) * (1u << 23) + __float_as_uint(p1));
  // below the clamp (masked keys are -inf) the result is exactly 0
  x0 = x0 >= -126.f ? y0 : 0.f;
  x1 = x1 >= -126.f ? y1 : 0.f;
}

}  // namespace swa
