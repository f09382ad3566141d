// Host build of the NVFP4 encoders the W4A4 kernels use (csrc/nvfp4_enc.cuh,
// compiled as plain C++), exported for the CPU tests: the same source the GPU
// runs, checked against the CPU reference without a GPU.  The row loop below
// follows the kernels' order: row amax, scale2, then each 16-block.
#include <cstdint>
#include <cstring>

#include "nvfp4_enc.cuh"

using namespace bsr::nvfp4;

extern "C" {

void h_e4m3_rne(const float* t, uint8_t* out, long n) {
  for (long i = 0; i < n; ++i) out[i] = (uint8_t)e4m3_rne_nonneg(t[i]);
}

void h_e4m3_value(const uint8_t* code, float* out, long n) {
  for (long i = 0; i < n; ++i) out[i] = e4m3_value(code[i]);
}

void h_e2m1_rne(const float* y, uint8_t* out, long n) {
  for (long i = 0; i < n; ++i) out[i] = (uint8_t)e2m1_rne(y[i]);
}

void h_quant_rows(const uint16_t* a, long m, long k, uint8_t* packed, uint8_t* e4, float* scale2) {
  for (long r = 0; r < m; ++r) {
    const uint16_t* row = a + r * k;
    float amax = 0.0f;
    for (long j = 0; j < k; ++j) {
      const float v = bits_f32((uint32_t)(row[j] & 0x7FFFu) << 16);
      amax = v > amax ? v : amax;
    }
    const float s2 = row_scale2(amax);
    scale2[r] = s2;
    for (long b = 0; b < k / 16; ++b) {
      float x[16];
      for (int i = 0; i < 16; ++i) x[i] = bits_f32((uint32_t)row[16 * b + i] << 16);
      const Block q = quant_block(x, s2);
      uint8_t* dst = packed + r * (k / 2) + 8 * b;
      for (int i = 0; i < 4; ++i) {
        dst[i] = (uint8_t)(q.lo >> (8 * i));
        dst[4 + i] = (uint8_t)(q.hi >> (8 * i));
      }
      e4[r * (k / 16) + b] = (uint8_t)q.e4;
    }
  }
}

}  // extern "C"
