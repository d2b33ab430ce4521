// Code decisions and packing shared by the quantize-append kernels: the stored field of a
// rotated coordinate decided on the FMA pipe against norm-scaled thresholds, and the sums
// of codes into exact float half-words that become packed words without per-code shifts.
#pragma once

#include <stdint.h>

#include "isoq_common.cuh"
#include "isoq_ptx.cuh"

namespace isoq {

// The stored field of one rotated coordinate z (scaled by sqrt(d)) on the FMA pipe, with
// TB[k] = n * (positive threshold k) * 2^64 (+inf for a zero vector).  Each
// sat(|z| 2^64 - TB[k]) is 1 when |z| > n t_k and 0 below; a coordinate exactly on a
// threshold (a difference of 0, the only case decided differently from the >= of the
// definition) lies inside any parity band around the thresholds.  With m thresholds
// exceeded, code = half + m for z >= 0 and half - 1 - m for z < 0 (-0 counts as +0, so a
// zero vector codes half), i.e. code = (half - 0.5) + sign(z) (m + 0.5).  4 bits store the
// sign-magnitude nibble m + 8 [z < 0] instead.
template <int BITS>
__device__ __forceinline__ uint32_t code_sat(float z, const float (&TB)[(1 << (BITS - 1)) - 1]) {
  constexpr int NT = (1 << (BITS - 1)) - 1;
  constexpr float kHalf = (float)(1 << (BITS - 1));
  const float zp = z + 0.0f;  // -0 -> +0
  const float a = fabsf(zp);
  float acc = 0.5f;
#pragma unroll
  for (int k = 0; k < NT; ++k) acc += __saturatef(fmaf(a, 0x1p64f, -TB[k]));
  const float sg = copysignf(1.0f, zp);
  const float cf = BITS == 4 ? fmaf(-4.0f, sg, acc + 3.5f) : fmaf(sg, acc, kHalf - 0.5f);
  return __float_as_uint(cf + 8388608.0f) & 0xFu;  // small exact integer in the mantissa
}

// 2-bit layout: the slot (0..15) of dim e (0..15) of a 16-dim word.
__host__ __device__ constexpr int slot2(int e) {
  return e < 8 ? ((e & 1) ? (e >> 1) + 4 : (e >> 1)) : ((e & 1) ? ((e - 8) >> 1) + 12 : ((e - 8) >> 1) + 8);
}

// The same decision as code_sat, added into the sum W = sum coef * code of a 16-bit
// half-word (coef = 16^nibble, or 4^slot at 2 bits): W gains coef * code minus the
// sign-independent part coef * base, which the caller puts in W's initial value
// (base = half - 0.5, or 4 at 4 bits).  z is never -0 here.  W stays an exact binary32
// integer + 0.5 multiple below 2^17, and no per-code conversion or shift is needed.
template <int BITS>
__device__ __forceinline__ float add_code(float W, float z, float coef,
                                          const float (&TB)[(1 << (BITS - 1)) - 1]) {
  constexpr int NT = (1 << (BITS - 1)) - 1;
  const float a = fabsf(z);
  const float c = copysignf(coef, z);
  float s[NT];
#pragma unroll
  for (int k = 0; k < NT; ++k) s[k] = __saturatef(fmaf(a, 0x1p64f, -TB[k]));
  if constexpr (BITS == 2) {
    return fmaf(c, s[0] + 0.5f, W);  // sign(z) (m + 0.5)
  } else if constexpr (BITS == 3) {
    return fmaf(c, (s[0] + s[1]) + (s[2] + 0.5f), W);
  } else {  // m - 4 sign(z)
    const float m = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + s[6]);
    return fmaf(c, -4.0f, fmaf(coef, m, W));
  }
}
template <int BITS>
constexpr float code_base() { return BITS == 4 ? 4.0f : (float)(1 << (BITS - 1)) - 0.5f; }

// add_code<3> for two coordinates za, zb at once, into a pair of partial sums W2 of one
// half-word (the half-word is W2.x + W2.y).  The six saturating decisions stay scalar; the
// sums (s0 + s1) + (s2 + 0.5) and the accumulation run as packed f32x2 pairs with the same
// per-lane rounding, and every value involved is a small exact half-integer, so the sum
// equals the scalar add_code's bit for bit.
__device__ __forceinline__ void add_code3_pair(float2& W2, float za, float zb, float coef_a,
                                               float coef_b, const float (&TB)[3]) {
  float sa[3], sb[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    sa[k] = __saturatef(fmaf(fabsf(za), 0x1p64f, -TB[k]));
    sb[k] = __saturatef(fmaf(fabsf(zb), 0x1p64f, -TB[k]));
  }
  const float2 m = ptx::f2_add(ptx::f2_add(make_float2(sa[0], sb[0]), make_float2(sa[1], sb[1])),
                               ptx::f2_add(make_float2(sa[2], sb[2]), make_float2(0.5f, 0.5f)));
  W2 = ptx::f2_fma(make_float2(copysignf(coef_a, za), copysignf(coef_b, zb)), m, W2);
}


// Two half-word sums, each as the bits of W + 2^23 (0x4B000000 | W), joined into one word:
// the high half's exponent bits leave the 32-bit product.
__device__ __forceinline__ uint32_t join_halves(uint32_t lo, uint32_t hi) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, 65536, %2;" : "=r"(r) : "r"(hi), "r"(lo & 0xffffu));
  return r;
}

}  // namespace isoq
