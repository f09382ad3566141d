// SiLU.mul quantiser for the down projection.  The launcher pages name it
// (w8a8_decode/parts.rs: `W8a8Kernels::quant_silu`, "the SiLU.mul quantizer";
// the grouped-decode page's gate+up step writes "quantized products") but
// give no arithmetic.  Reading taken here: the product is the BF16
// activation the down projection would otherwise be given,
//
//     x = bf16_rne(silu(g) * u),   silu(g) = g / (1 + exp(-g)),
//
// and the quantiser is requant_a of x (same code as requant_a, so the fused
// quantiser is bit-identical to the product followed by requant_a).
//
// The kernel evaluates silu(g) without overflow for either sign of g, with
// t = exp(-|g|) in (0, 1]:
//     silu(g) = g / (1 + t)        for g >= 0,
//     silu(g) = (g * t) / (1 + t)  for g < 0,
// and exp by Cody-Waite range reduction with a two-part ln 2 followed by the
// hardware base-2 exponential of the reduced argument:
//     n = rint(x * log2e),  r = (x - n * ln2_hi) - n * ln2_lo,  |r| <= ln2/2
//     exp(x) = 2^(r * log2e) * 2^n           (x = -|g| <= 0)
// The reduced argument keeps the hardware's relative error (about 2^-22) for
// every |g|; with the approximate quotient (2 ulp) and three roundings the
// float32 product is within 2^-20 of the exact silu(g) * u, so its BF16
// rounding equals the exact product's except within 2^-20 of a rounding
// boundary.  For g < -104 the kernel takes t = 0 (e^-104 is below float32's
// range), so its product is a signed zero; the exact product rounds to zero
// in BF16 there unless |u| > 650.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "occupancy.h"
#include "quant.cuh"

namespace bsr {

namespace {

constexpr uint32_t kLog2e = 0x3FB8AA3Bu;  // 1.442695f
constexpr uint32_t kLn2Hi = 0x3F317200u;  // 0.693145751953125f (15 significant bits: n * ln2_hi is exact)
constexpr uint32_t kLn2Lo = 0x35BFBE8Eu;  // ln 2 - kLn2Hi

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// exp(x) for -104 <= x <= 0 (below -126 ln 2 the two-step scaling by
// 2^h1 * 2^h2 reaches the subnormal range)
__device__ __forceinline__ float exp_nonpos(float x) {
  const float n = rintf(__fmul_rn(x, __uint_as_float(kLog2e)));
  float r = __fmaf_rn(-n, __uint_as_float(kLn2Hi), x);
  r = __fmaf_rn(-n, __uint_as_float(kLn2Lo), r);
  const float p = ex2_approx(__fmul_rn(r, __uint_as_float(kLog2e)));
  const int ni = (int)n;                      // in [-150, 0]
  const int h1 = ni >= -126 ? ni : -126;      // 2^h1 normal
  const int h2 = ni - h1;                     // in [-25, 0]
  const float s1 = __uint_as_float((uint32_t)(h1 + 127) << 23);
  const float s2 = __uint_as_float((uint32_t)(h2 + 127) << 23);
  return __fmul_rn(__fmul_rn(p, s1), s2);
}

// bf16(silu(g) * u) as its float32 value (exact)
__device__ __forceinline__ float silu_mul_value(float g, float u) {
  const float ag = fabsf(g);
  const float t = ag <= 104.0f ? exp_nonpos(-ag) : 0.0f;
  const float num = g >= 0.0f ? g : __fmul_rn(g, t);
  const float s = __fdividef(num, __fadd_rn(1.0f, t));
  return __bfloat162float(__float2bfloat16_rn(__fmul_rn(s, u)));
}

__device__ __forceinline__ void silu_mul8(const uint4& gv, const uint4& uv, float (&x)[8]) {
  float g[8], u[8];
  bf16x8_to_f32(gv, g);
  bf16x8_to_f32(uv, u);
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = silu_mul_value(g[i], u[i]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (__float_as_uint(lo) >> 16) | (__float_as_uint(hi) & 0xFFFF0000u);  // values are exact BF16
}

// x = bf16(silu(g) * u), 8 elements (16 bytes) per thread and step.
__global__ void __launch_bounds__(256) silu_mul_kernel(const uint4* __restrict__ g, const uint4* __restrict__ u,
                                                       uint4* __restrict__ x, long long n8) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    float v[8];
    silu_mul8(__ldg(g + i), __ldg(u + i), v);
    x[i] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
  }
}

// requant_a of bf16(silu(g) * u) without writing the product: the task
// layout of requant_a (one thread per 32-group, a warp on 8 rows x 4
// blocks, block-major scales), the 32 products formed after the loads and
// quantised by the same code as requant_a.
__global__ void __launch_bounds__(256) requant_silu_a_kernel(const uint16_t* __restrict__ g,
                                                             const uint16_t* __restrict__ u,
                                                             int8_t* __restrict__ a_i8, float* __restrict__ a_scale_t,
                                                             int m, int k, int ld) {
  const int lane = threadIdx.x & 31;
  const int nb = k >> 5;
  const int nb4 = (nb + 3) >> 2;
  const long long tasks = (long long)((m + 7) >> 3) * nb4;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long t = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < tasks; t += nwarps) {
    const long long r8 = t / nb4;
    const int row = (int)(r8 * 8) + (lane & 7);
    const int blk = (int)(t - r8 * nb4) * 4 + (lane >> 3);
    if (row >= m || blk >= nb) continue;  // no warp-wide operation below
    const size_t off = (size_t)row * k + (size_t)blk * 32;
    const uint4* gs = reinterpret_cast<const uint4*>(g + off);
    const uint4* us = reinterpret_cast<const uint4*>(u + off);
    uint4 gv[4], uv[4], v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      gv[i] = __ldg(gs + i);
      uv[i] = __ldg(us + i);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float x[8];
      silu_mul8(gv[i], uv[i], x);
      v[i] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                        pack_bf16x2(x[6], x[7]));
    }
    uint4 lo, hi;
    float scale;
    quant_group32(v, lo, hi, scale);
    uint4* dst = reinterpret_cast<uint4*>(a_i8 + off);
    dst[0] = lo;
    dst[1] = hi;
    a_scale_t[(size_t)blk * ld + row] = scale;
  }
}

int grid_for(long long work_items, int per_block, int max_blocks) {
  long long gr = (work_items + per_block - 1) / per_block;
  if (gr < 1) gr = 1;
  if (gr > max_blocks) gr = max_blocks;
  return (int)gr;
}

}  // namespace

cudaError_t launch_silu_mul(const uint16_t* g, const uint16_t* u, uint16_t* x, int m, int k, cudaStream_t stream,
                            int num_sms) {
  const long long n8 = (long long)m * k / 8;
  const int grid = grid_for(n8, 256, num_sms * resident_ctas_per_sm((const void*)silu_mul_kernel, 256));
  silu_mul_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(g), reinterpret_cast<const uint4*>(u),
                                            reinterpret_cast<uint4*>(x), n8);
  return cudaGetLastError();
}

cudaError_t launch_requant_silu_a(const uint16_t* g, const uint16_t* u, int8_t* a_i8, float* a_scale_t, int m, int k,
                                  int ld, cudaStream_t stream, int num_sms) {
  const long long tasks = (long long)((m + 7) / 8) * ((k / 32 + 3) / 4);
  const int grid = grid_for(tasks, 8, num_sms * resident_ctas_per_sm((const void*)requant_silu_a_kernel, 256));
  requant_silu_a_kernel<<<grid, 256, 0, stream>>>(g, u, a_i8, a_scale_t, m, k, ld);
  return cudaGetLastError();
}

}  // namespace bsr
