// SiLU.mul quantiser for the down projection.  The launcher pages name it
// (w8a8_decode/parts.rs: `W8a8Kernels::quant_silu`, "the SiLU.mul quantizer";
// the grouped-decode page's gate+up step writes "quantized products") but
// give no arithmetic.  Reading taken here: the product is the BF16
// activation the down projection would otherwise be given,
//
//     x = bf16_rne(silu(g) * u),   silu(g) = g / (1 + exp(-g)),
//
// every step a float32 operation rounded to nearest (intrinsics, so nothing
// is contracted into an FMA), and the quantiser is requant_a of x: one F32
// scale per 32 elements, codes rint(x / scale) clamped to +-127.
//
// exp is computed by explicit steps (Cody-Waite range reduction with a
// two-part ln 2 and a degree-6 Taylor polynomial in Horner form), not by the
// CUDA math library, so that the result is a fixed function of the input:
//
//     n = rint(x * log2e)                     (half-even)
//     r = (x - n * ln2_hi) - n * ln2_lo        (n * ln2_hi exact: ln2_hi has 15 bits)
//     p = 1 + r(1 + r(1/2 + r(1/6 + r(1/24 + r(1/120 + r/720)))))
//     exp(x) = (p * 2^h1) * 2^h2,  h1 = floor(n/2), h2 = n - h1
//
// with x > 88 -> +inf and x < -88 -> +0.  Over [-88, 88] it is within 3 ulp
// of exp.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace bsr {

namespace {

constexpr uint32_t kLog2e = 0x3FB8AA3Bu;  // 1.442695f
constexpr uint32_t kLn2Hi = 0x3F317200u;  // 0.693145751953125f
constexpr uint32_t kLn2Lo = 0x35BFBE8Eu;  // ln 2 - kLn2Hi
// 1/i! for i = 0..6
constexpr uint32_t kC0 = 0x3F800000u, kC1 = 0x3F800000u, kC2 = 0x3F000000u, kC3 = 0x3E2AAAABu,
                   kC4 = 0x3D2AAAABu, kC5 = 0x3C088889u, kC6 = 0x3AB60B61u;

__device__ __forceinline__ float pow2i(int h) {  // 2^h, h in [-126, 127]
  return __uint_as_float((uint32_t)(h + 127) << 23);
}

__device__ __forceinline__ float exp_steps(float x) {
  if (x != x) return x;
  if (x > 88.0f) return __uint_as_float(0x7F800000u);
  if (x < -88.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, __uint_as_float(kLog2e)));
  const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(n, __uint_as_float(kLn2Hi))), __fmul_rn(n, __uint_as_float(kLn2Lo)));
  float p = __uint_as_float(kC6);
  p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(kC5));
  p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(kC4));
  p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(kC3));
  p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(kC2));
  p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(kC1));
  p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(kC0));
  const int ni = (int)n;
  const int h1 = ni >> 1;  // floor(n / 2)
  const int h2 = ni - h1;
  return __fmul_rn(__fmul_rn(p, pow2i(h1)), pow2i(h2));
}

// bf16(silu(g) * u) as its float32 value (exact) and its bit pattern
__device__ __forceinline__ float silu_mul_value(float g, float u) {
  const float e = exp_steps(-g);
  const float s = __fdiv_rn(g, __fadd_rn(1.0f, e));
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
// layout of requant_a (four lanes per 32-group, eight rows per warp at one
// block, block-major scales), with the product formed after the loads.
__global__ void __launch_bounds__(256) requant_silu_a_kernel(const uint4* __restrict__ g, const uint4* __restrict__ u,
                                                             uint2* __restrict__ a_i8, float* __restrict__ a_scale_t,
                                                             int m, int k, int ld) {
  const int lane = threadIdx.x & 31;
  const int nb = k >> 5;
  const long long tasks = (long long)((m + 7) >> 3) * nb;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int sub = lane & 3;
  for (long long t = warp0; t < tasks; t += nwarps) {
    const int r8 = (int)(t / nb);
    const int b = (int)(t - (long long)r8 * nb);
    const int row = r8 * 8 + (lane >> 2);
    const bool valid = row < m;  // uniform per group of 4 lanes
    const long long e = (long long)(valid ? row : 0) * k + (long long)b * 32 + sub * 8;
    uint4 gv = make_uint4(0, 0, 0, 0), uv = make_uint4(0, 0, 0, 0);
    if (valid) {
      gv = __ldg(g + (e >> 3));
      uv = __ldg(u + (e >> 3));
    }
    float x[8];
    silu_mul8(gv, uv, x);
    float s;
    const uint2 c = quant8_quad(x, s);
    if (valid) {
      a_i8[e >> 3] = c;
      if (sub == 0) a_scale_t[(long long)b * ld + row] = s;
    }
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
  const int grid = grid_for(n8, 256, num_sms * 8);
  silu_mul_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(g), reinterpret_cast<const uint4*>(u),
                                            reinterpret_cast<uint4*>(x), n8);
  return cudaGetLastError();
}

cudaError_t launch_requant_silu_a(const uint16_t* g, const uint16_t* u, int8_t* a_i8, float* a_scale_t, int m, int k,
                                  int ld, cudaStream_t stream, int num_sms) {
  const long long tasks = (long long)((m + 7) / 8) * (k / 32);
  const int grid = grid_for(tasks, 8, num_sms * 8);
  requant_silu_a_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(g),
                                                  reinterpret_cast<const uint4*>(u), reinterpret_cast<uint2*>(a_i8),
                                                  a_scale_t, m, k, ld);
  return cudaGetLastError();
}

}  // namespace bsr
