// Per-32-element int8 quantisation rule shared by the weight and activation
// requantisation kernels and by the decode kernel's fused activation pass.
//
// Rule (the launcher pages fix the layout: one F32 scale per 32 elements,
// signed int8 codes; the rounding conventions are this library's):
//   amax  = max |x| over the group
//   scale = RN_f32(amax / 127)
//   q     = clamp(rint_half_even(RN_f32(x / scale)), -127, 127), or 0 when scale == 0
//
// The division by the scale is exact-rounded float32.  Instead of one IEEE
// division per element, `quant_code` multiplies by RN(1/scale) and only falls
// back to the exact division when the product lies within 2^-15 of a
// half-integer.  Argument: with t = x/scale (|t| <= 127.00001),
// y = RN(x * RN(1/scale)) satisfies |y - t| <= |t| (2^-23 + 2^-48) < 1.52e-5
// and |RN(t) - t| <= 2^-18, so |y - RN(t)| < 1.9e-5 < 2^-15.  When y is more
// than 2^-15 away from every half-integer, RN(t) lies strictly between the
// same two half-integers and rounds to the same integer as y.  This needs
// RN(1/scale) to be a normal float, i.e. scale >= 2^-126; smaller scales use
// the exact division throughout.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace bsr {

constexpr float kQMax = 127.0f;
// 0.5 - 2^-15: distance test for "close to a half-integer".
constexpr float kTieGuard = 0.499969482421875f;
constexpr float kMinNormal = 1.17549435e-38f;  // 2^-126

struct GroupScale {
  float scale;  // RN(amax / 127); 0 for a zero group
  float rcp;    // RN(1 / scale) when scale is normal, else 0 (exact path)
};

__device__ __forceinline__ GroupScale group_scale(float amax) {
  GroupScale g;
  g.scale = __fdiv_rn(amax, kQMax);
  g.rcp = (g.scale >= kMinNormal) ? __frcp_rn(g.scale) : 0.0f;
  return g;
}

// Integer code of x for a group with non-zero scale.
__device__ __forceinline__ int quant_code(float x, const GroupScale& g) {
  float ry;
  if (g.rcp != 0.0f) {
    float y = __fmul_rn(x, g.rcp);
    ry = rintf(y);
    if (fabsf(__fsub_rn(y, ry)) >= kTieGuard) ry = rintf(__fdiv_rn(x, g.scale));
  } else {
    ry = rintf(__fdiv_rn(x, g.scale));
  }
  ry = fminf(fmaxf(ry, -kQMax), kQMax);
  return __float2int_rn(ry);
}

// Pack the low bytes of four ints into one word, element 0 in byte 0.
__device__ __forceinline__ uint32_t pack4_s8(int a, int b, int c, int d) {
  uint32_t lo = __byte_perm((uint32_t)a, (uint32_t)b, 0x0040);
  uint32_t hi = __byte_perm((uint32_t)c, (uint32_t)d, 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// Eight BF16 values (one 16-byte load) to float32 (exact).
__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&x)[8]) {
  x[0] = __uint_as_float(v.x << 16);
  x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16);
  x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  x[4] = __uint_as_float(v.z << 16);
  x[5] = __uint_as_float(v.z & 0xFFFF0000u);
  x[6] = __uint_as_float(v.w << 16);
  x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

// Quantise 8 consecutive values of a group whose 4 lanes are adjacent
// (lane & ~3 .. lane | 3).  Returns the 8 codes packed, and the group scale.
__device__ __forceinline__ uint2 quant8_quad(const float (&x)[8], float& scale_out) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  const GroupScale g = group_scale(amax);
  scale_out = g.scale;
  int q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = (g.scale == 0.0f) ? 0 : quant_code(x[i], g);
  return make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
}

}  // namespace bsr
