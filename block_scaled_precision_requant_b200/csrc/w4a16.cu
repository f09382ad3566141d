// NVFP4 W4A16 decode GEMV (gemv_sw.rs: `w4a16_gemv` / `w4a16_gemv_sw`, the
// decode GEMV launched with the BF16 input, the packed E2M1 weight, its E4M3
// scales, the F32 scale_2, the BF16 output, n and k).  The page fixes the
// arguments, not the arithmetic; reading taken:
//
//   out[m, n] = bf16( sum_k A[m, k] * (e2m1[n, k] * e4m3[n, k/16]) * scale2 ),
//
// accumulated in float32: per 16-element block p = sum_i a_i * e2m1_i, then
// acc += p * e4m3, and scale2 once at the end.  It reads the NVFP4 weight as
// stored (0.5625 B per element, half the int8 path's 1.125 B), so it is the
// byte-minimal decode; its results are not bit-compatible with the int8
// projection (no requantisation) and are compared within the BF16 tolerance.
//
// One warp per weight row: lane l takes 16-element blocks l, l+32, ... (8
// bytes of nibbles and one E4M3 byte each; the loads of four blocks are
// issued before their arithmetic), the E2M1 pairs are converted by the
// hardware FP4 -> f16 conversion (exact), the activation rows sit in shared
// memory as BF16.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace bsr {

namespace {

constexpr int kW4Unroll = 4;  // 16-blocks per lane in flight

// threads per CTA: one row per warp; more activation rows per CTA need more
// registers per thread, so fewer warps
template <int MR>
constexpr int w4a16_max_threads() { return MR == 1 ? 1024 : 512; }

__device__ __forceinline__ float e4m3_value(uint32_t byte) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3);
  return __half2float(__half(h));
}

// the 16 E2M1 values of one block (8 bytes, element 2i in the low nibble of byte i)
__device__ __forceinline__ void e2m1x16(const uint2 q, float (&w)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t byte = ((i < 4 ? q.x : q.y) >> (8 * (i & 3))) & 0xFFu;
    const __half2_raw h2 = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)byte, __NV_E2M1);
    w[2 * i] = __half2float(__half(__half_raw{h2.x}));
    w[2 * i + 1] = __half2float(__half(__half_raw{h2.y}));
  }
}

__device__ __forceinline__ void bf16x8(const uint4& v, float* x) {
  x[0] = __uint_as_float(v.x << 16);
  x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16);
  x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  x[4] = __uint_as_float(v.z << 16);
  x[5] = __uint_as_float(v.z & 0xFFFF0000u);
  x[6] = __uint_as_float(v.w << 16);
  x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

template <int MR>
__global__ void __launch_bounds__(w4a16_max_threads<MR>(), 1)
    w4a16_decode_kernel(const uint16_t* __restrict__ a, const uint8_t* __restrict__ w_packed,
                        const uint8_t* __restrict__ w_e4m3, float scale2, __nv_bfloat16* __restrict__ out, int m,
                        int n, int k) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* s_a = reinterpret_cast<uint16_t*>(smem);  // [MR][K] BF16
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int m0 = blockIdx.y * MR;
  const int rows = min(MR, m - m0);

  // programmatic dependent launch: the activations may come from the
  // previous kernel on the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int kv = k >> 3;  // 16-byte vectors per activation row
  for (int i = threadIdx.x; i < MR * kv; i += blockDim.x) {
    const int r = i / kv;
    const int c = i - r * kv;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows) v = __ldg(reinterpret_cast<const uint4*>(a + (size_t)(m0 + r) * k) + c);
    reinterpret_cast<uint4*>(s_a + (size_t)r * k)[c] = v;
  }
  __syncthreads();

  const int nb = k >> 4;  // 16-element blocks per row
  // the two 16-byte halves of a block's activations are read in the order
  // h, 1-h (h = (lane >> 2) & 1) so the shared loads of a quarter-warp hit
  // distinct banks
  const int h = (lane >> 2) & 1;
  for (int row = blockIdx.x * nwarps + warp; row < n; row += gridDim.x * nwarps) {
    const uint2* wp = reinterpret_cast<const uint2*>(w_packed + (size_t)row * (size_t)(k >> 1));
    const uint8_t* we = w_e4m3 + (size_t)row * (size_t)nb;
    float acc[MR];
#pragma unroll
    for (int r = 0; r < MR; ++r) acc[r] = 0.0f;
    for (int b0 = lane; b0 < nb; b0 += 32 * kW4Unroll) {
      uint2 q[kW4Unroll];
      uint32_t e[kW4Unroll];
#pragma unroll
      for (int u = 0; u < kW4Unroll; ++u) {
        const int b = b0 + 32 * u;
        q[u] = b < nb ? __ldg(wp + b) : make_uint2(0, 0);
        e[u] = b < nb ? (uint32_t)__ldg(we + b) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kW4Unroll; ++u) {
        const int b = b0 + 32 * u;
        if (b >= nb) break;
        float wv[16];
        e2m1x16(q[u], wv);
        const float s = e4m3_value(e[u]);
#pragma unroll
        for (int r = 0; r < MR; ++r) {
          const uint4* ap = reinterpret_cast<const uint4*>(s_a + (size_t)r * k + (size_t)b * 16);
          float x[16];
          bf16x8(ap[h], x + 8 * h);
          bf16x8(ap[1 - h], x + 8 * (1 - h));
          float p = 0.0f;
#pragma unroll
          for (int i = 0; i < 16; ++i) p = __fmaf_rn(x[i], wv[i], p);
          acc[r] = __fmaf_rn(p, s, acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      float v = acc[r];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
      acc[r] = v;
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < MR; ++r)
        if (r < rows) out[(size_t)(m0 + r) * n + row] = __float2bfloat16_rn(__fmul_rn(acc[r], scale2));
    }
  }
}

template <int MR>
cudaError_t launch_w4a16_t(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                           uint16_t* out, int m, int n, int k, size_t smem_limit, cudaStream_t stream, int num_sms) {
  auto kern = w4a16_decode_kernel<MR>;
  const size_t smem = (size_t)MR * (size_t)k * 2;
  if (smem > smem_limit) return cudaErrorInvalidValue;
  static size_t granted[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (smem > granted[dev] && smem > 48 * 1024) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      granted[dev] = smem;
    }
  }
  // warps (= weight rows in flight) per CTA: spread the rows over all SMs
  int w = (int)((n + (long long)num_sms - 1) / num_sms);
  constexpr int kMaxW = w4a16_max_threads<MR>() / 32;
  w = w < 1 ? 1 : (w > kMaxW ? kMaxW : w);
  const int gy = (m + MR - 1) / MR;
  long long gx = (n + w - 1) / w;
  if (gx * gy > num_sms) gx = ((long long)num_sms + gy - 1) / gy;
  if (gx < 1) gx = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)gx, (unsigned)gy);
  cfg.blockDim = dim3(w * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a, w_packed, w_e4m3, scale2, reinterpret_cast<__nv_bfloat16*>(out), m, n, k);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16_decode(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                                uint16_t* out, int m, int n, int k, size_t smem_limit, cudaStream_t stream,
                                int num_sms) {
  int mr = 1;
  while (mr < m && mr < 16) mr <<= 1;
  while (mr > 1 && (size_t)mr * (size_t)k * 2 > smem_limit) mr >>= 1;
  switch (mr) {
    case 1: return launch_w4a16_t<1>(a, w_packed, w_e4m3, scale2, out, m, n, k, smem_limit, stream, num_sms);
    case 2: return launch_w4a16_t<2>(a, w_packed, w_e4m3, scale2, out, m, n, k, smem_limit, stream, num_sms);
    case 4: return launch_w4a16_t<4>(a, w_packed, w_e4m3, scale2, out, m, n, k, smem_limit, stream, num_sms);
    case 8: return launch_w4a16_t<8>(a, w_packed, w_e4m3, scale2, out, m, n, k, smem_limit, stream, num_sms);
    default: return launch_w4a16_t<16>(a, w_packed, w_e4m3, scale2, out, m, n, k, smem_limit, stream, num_sms);
  }
}

}  // namespace bsr
