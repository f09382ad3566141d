// Hardware conversions of the OCP FP8 E4M3 and OCP MX E2M1 formats, and the
// mixed-precision FMA, as inline PTX for sm_100a.
//
// cuda_fp8.h / cuda_fp4.h route their conversion intrinsics to these
// instructions only for the family-specific target (sm_100f); built for
// sm_100a they fall back to a software emulation of a few dozen integer
// instructions per value.  The kernels that convert per element call the
// instructions directly instead.
#pragma once

#include <cstdint>

namespace bsr {

// Two E4M3 bytes (the low 16 bits of `two`, the low byte into the low half)
// -> two f16 in one word.  Exact: every E4M3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t d;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(d) : "r"(two));
  return d;
}

__device__ __forceinline__ float f16_lo_to_f32(uint32_t h2) {
  float f;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, lo;\n\t}" : "=f"(f) : "r"(h2));
  return f;
}

__device__ __forceinline__ float f16_hi_to_f32(uint32_t h2) {
  float f;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, hi;\n\t}" : "=f"(f) : "r"(h2));
  return f;
}

// Value of one E4M3 byte (the low byte of `byte`) as float32, exact.
__device__ __forceinline__ float e4m3_to_f32_hw(uint32_t byte) { return f16_lo_to_f32(e4m3x2_to_f16x2(byte & 0xFFu)); }

// The 8 E2M1 codes of one word (element 2i in the low nibble of byte i) ->
// four f16x2 words, word i = (element 2i, element 2i + 1) in (low, high)
// half.  Exact.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t* h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

// c + a.lo * b.lo, then + a.hi * b.hi: f16 operands, float32 accumulation.
// Each f16 x f16 product is exact in float32, so each step rounds once,
// exactly like a float32 FMA on the converted operands.
__device__ __forceinline__ float fma2_f16_f32(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t.reg .f32 t;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 t, al, bl, %3;\n\tfma.rn.f32.f16 %0, ah, bh, t;\n\t}"
      : "=f"(d)
      : "r"(a), "r"(b), "f"(c));
  return d;
}

// float32 sum of the two f16 halves of h2, rounded once.
__device__ __forceinline__ float f16x2_sum_f32(uint32_t h2) {
  float d;
  asm("{\n\t.reg .b16 lo, hi;\n\t.reg .f32 t;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "add.rn.f32.f16 t, lo, 0f00000000;\n\tadd.rn.f32.f16 %0, hi, t;\n\t}"
      : "=f"(d)
      : "r"(h2));
  return d;
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Two float32 -> f16x2 (lo into the low half), rounded to nearest even.
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

}  // namespace bsr
