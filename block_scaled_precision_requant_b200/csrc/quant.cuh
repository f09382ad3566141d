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

// Four codes in [-127, 127] packed into one word, element 0 in byte 0
// (two saturating pack conversions; the saturation never binds).
__device__ __forceinline__ uint32_t pack4_cvt(int q0, int q1, int q2, int q3) {
  uint32_t hi, d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(q3), "r"(q2));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q1), "r"(q0), "r"(hi));
  return d;
}

// Largest |x| of 16 BF16 pairs, as float32 (exact).  |x| of a BF16 value is
// its bit pattern with the sign cleared, and for non-NaN values the order of
// those patterns as unsigned integers is the order of the magnitudes, so
// the maximum is taken with packed 16-bit unsigned max operations.
__device__ __forceinline__ float bf16x32_amax(const uint4 (&v)[4]) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = __vmaxu2(m, v[i].x & 0x7FFF7FFFu);
    m = __vmaxu2(m, v[i].y & 0x7FFF7FFFu);
    m = __vmaxu2(m, v[i].z & 0x7FFF7FFFu);
    m = __vmaxu2(m, v[i].w & 0x7FFF7FFFu);
  }
  const uint32_t hm = (m >> 16) > (m & 0xFFFFu) ? (m >> 16) : (m & 0xFFFFu);
  return __uint_as_float(hm << 16);
}

// Code of x for a group with a normal reciprocal (g.rcp != 0): the product
// by RN(1/scale) rounded half-even, or the rounded IEEE quotient when the
// product lies within 2^-15 of a half-integer (see the file comment).  The
// result is in [-127, 127] without a clamp: |y| <= 127 (1 + 2^-23)^2 < 127.5.
__device__ __forceinline__ int quant_code_rcp(float x, const GroupScale& g) {
  const float y = __fmul_rn(x, g.rcp);
  float ry = rintf(y);
  if (fabsf(__fsub_rn(y, ry)) >= kTieGuard) ry = rintf(__fdiv_rn(x, g.scale));
  return __float2int_rn(ry);
}

// One whole 32-group in one thread: 32 BF16 values (four 16-byte loads) ->
// 32 codes (two 16-byte words) and the group scale.  Same rule as
// quant_code; all-zero (or underflowing) groups give scale 0 and codes 0.
__device__ __forceinline__ void quant_group32(const uint4 (&v)[4], uint4& c_lo, uint4& c_hi, float& scale_out) {
  const GroupScale g = group_scale(bf16x32_amax(v));
  scale_out = g.scale;
  uint32_t w[8];
  if (g.rcp != 0.0f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t p[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int q0 = quant_code_rcp(__uint_as_float(p[2 * j] << 16), g);
        const int q1 = quant_code_rcp(__uint_as_float(p[2 * j] & 0xFFFF0000u), g);
        const int q2 = quant_code_rcp(__uint_as_float(p[2 * j + 1] << 16), g);
        const int q3 = quant_code_rcp(__uint_as_float(p[2 * j + 1] & 0xFFFF0000u), g);
        w[2 * i + j] = pack4_cvt(q0, q1, q2, q3);
      }
    }
  } else {
    // scale 0 (all-zero group) or subnormal (every code by exact division)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t p[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        int q[4];
        const float x[4] = {__uint_as_float(p[2 * j] << 16), __uint_as_float(p[2 * j] & 0xFFFF0000u),
                            __uint_as_float(p[2 * j + 1] << 16), __uint_as_float(p[2 * j + 1] & 0xFFFF0000u)};
#pragma unroll
        for (int e = 0; e < 4; ++e) q[e] = (g.scale == 0.0f) ? 0 : quant_code(x[e], g);
        w[2 * i + j] = pack4_cvt(q[0], q[1], q[2], q[3]);
      }
    }
  }
  c_lo = make_uint4(w[0], w[1], w[2], w[3]);
  c_hi = make_uint4(w[4], w[5], w[6], w[7]);
}

}  // namespace bsr
