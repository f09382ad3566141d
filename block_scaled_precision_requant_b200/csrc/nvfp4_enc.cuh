// NVFP4 encoders for the W4A4 row quantiser (w4a4_proj/fixed.rs,
// `nvfp4_proj_mx`: each BF16 activation row is quantised to NVFP4 before the
// "mx" GEMV; the page gives no arithmetic).  Reading taken, the encoding the
// weight is stored in, applied per row:
//
//   scale2 = RN(amax_row / 2688)                     (2688 = 6 * 448)
//   s16    = E4M3_RNE(RN(amax16 / RN(6 * scale2)))   (saturating at 448)
//   code   = E2M1_RNE(RN(x / RN(s16 * scale2)))      (saturating at 6)
//
// every RN a float32 operation rounded to nearest even; a block whose s16 or
// whose s16 * scale2 is 0 (a zero row or block) gets code 0 throughout.
// E2M1 ties go to the even mantissa and the sign of the quotient is kept (a
// negative value that rounds to 0 is -0, code 0x8).
//
// The functions are plain arithmetic on float bits, written from the format
// definitions (OCP FP8 E4M3: bias 7, 3 mantissa bits, subnormal step 2^-9,
// largest finite 448; OCP MX E2M1: magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), so
// that the same source compiles, as plain C++, for a host check against the
// CPU reference.  On the GPU quant_block takes the two final roundings from
// the hardware conversions instead (same results, a few instructions per
// value instead of a few dozen).
#pragma once

#include <cstdint>
#include <cstring>

#if defined(__CUDACC__)
#define BSR_HD __host__ __device__ __forceinline__
#else
#include <cmath>
#define BSR_HD inline
#endif

namespace bsr {
namespace nvfp4 {

BSR_HD uint32_t f32_bits(float x) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(x);
#else
  uint32_t u;
  std::memcpy(&u, &x, 4);
  return u;
#endif
}

BSR_HD float bits_f32(uint32_t u) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float(u);
#else
  float x;
  std::memcpy(&x, &u, 4);
  return x;
#endif
}

// IEEE float32 operations rounded to nearest even, never contracted
BSR_HD float mul_rn(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(a, b);
#else
  volatile float r = a * b;
  return r;
#endif
}

BSR_HD float div_rn(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fdiv_rn(a, b);
#else
  volatile float r = a / b;
  return r;
#endif
}

BSR_HD float abs_f(float x) { return bits_f32(f32_bits(x) & 0x7FFFFFFFu); }

// Value of a non-negative E4M3 byte (0x00..0x7E): exponent field 0 gives
// m * 2^-9, otherwise (8 + m) * 2^(e - 10).  Built from bits, so exact.
BSR_HD float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u;
  const uint32_t m = code & 7u;
  if (e == 0) return mul_rn((float)m, bits_f32(0x3B000000u));  // 2^-9
  // float32 with exponent e - 7 and the 3-bit mantissa at the top
  return bits_f32(((e - 7u + 127u) << 23) | (m << 20));
}

// Nearest E4M3 byte to a finite t >= 0, ties to the even code, values at or
// above 448 saturating to 448 (0x7E).
BSR_HD uint32_t e4m3_rne_nonneg(float t) {
  if (!(t < 448.0f)) return 0x7Eu;  // also catches +inf
  if (t < 0.015625f) {  // below 2^-6: subnormal codes 0..8, steps of 2^-9
    // t * 2^9 is exact; round half to even by integer arithmetic on the bits
    const float s = mul_rn(t, 512.0f);  // in [0, 8)
    uint32_t q = (uint32_t)s;           // truncation
    const float frac = s - (float)q;    // exact (s < 8, q integer)
    if (frac > 0.5f || (frac == 0.5f && (q & 1u))) ++q;
    return q;  // q == 8 is exponent field 1, mantissa 0: the smallest normal
  }
  const uint32_t u = f32_bits(t);
  uint32_t e = (u >> 23) - 127u + 7u;  // biased E4M3 exponent, >= 1 here
  uint32_t keep = (u >> 20) & 7u;      // top 3 mantissa bits
  const uint32_t rest = u & 0xFFFFFu;  // the 20 dropped bits
  if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) {
    if (++keep == 8u) {
      keep = 0;
      ++e;
    }
  }
  const uint32_t code = (e << 3) | keep;
  return code > 0x7Eu ? 0x7Eu : code;
}

// E2M1 nibble of y: magnitude index of |y| rounded to {0, .5, 1, 1.5, 2, 3,
// 4, 6}, ties to the even index (even mantissa), saturating at 6; bit 3 is
// the sign bit of y.
BSR_HD uint32_t e2m1_rne(float y) {
  const float a = abs_f(y);
  uint32_t i = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return i | ((f32_bits(y) >> 28) & 8u);
}

// scale2 of a row from its amax
BSR_HD float row_scale2(float amax) { return div_rn(amax, 2688.0f); }

// One 16-element block: its E4M3 scale byte and the 16 codes packed in two
// words (element 2i in the low nibble of byte i).
struct Block {
  uint32_t e4;
  uint32_t lo, hi;
};

#if defined(__CUDA_ARCH__)
// The same two roundings by the hardware conversions (round to nearest even
// on the format's grid, saturating at its largest finite value, the sign of
// zero kept): e2m1_rne of two values, `lo` into the low nibble, and
// e4m3_rne_nonneg.  The GPU tests hold them to the oracle bit for bit on
// every E2M1 and E4M3 midpoint, -0, subnormal and saturating case.
__device__ __forceinline__ uint32_t e2m1x2_rne_hw(float lo, float hi) {
  unsigned short h;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(h)
      : "f"(hi), "f"(lo));
  return h;
}
__device__ __forceinline__ uint32_t e4m3_rne_nonneg_hw(float t) {
  unsigned short h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(t));
  return h & 0xFFu;
}
#endif

BSR_HD Block quant_block(const float (&x)[16], float scale2) {
  float amax16 = 0.0f;
  for (int i = 0; i < 16; ++i) {
    const float v = abs_f(x[i]);
    amax16 = v > amax16 ? v : amax16;
  }
  const float six_s2 = mul_rn(6.0f, scale2);
  const float t = six_s2 > 0.0f ? div_rn(amax16, six_s2) : 0.0f;
  Block b;
#if defined(__CUDA_ARCH__)
  b.e4 = e4m3_rne_nonneg_hw(t);
#else
  b.e4 = e4m3_rne_nonneg(t);
#endif
  const float denom = mul_rn(e4m3_value(b.e4), scale2);
  b.lo = 0;
  b.hi = 0;
  if (denom > 0.0f) {
#if defined(__CUDA_ARCH__)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t c = e2m1x2_rne_hw(div_rn(x[2 * i], denom), div_rn(x[2 * i + 1], denom));
      if (i < 4)
        b.lo |= c << (8 * i);
      else
        b.hi |= c << (8 * (i - 4));
    }
#else
    for (int i = 0; i < 16; ++i) {
      const uint32_t c = e2m1_rne(div_rn(x[i], denom));
      if (i < 8)
        b.lo |= c << (4 * i);
      else
        b.hi |= c << (4 * (i - 8));
    }
#endif
  }
  return b;
}

}  // namespace nvfp4
}  // namespace bsr
