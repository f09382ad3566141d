// NVFP4 W4A4 decode route (w4a4_proj/fixed.rs, `nvfp4_proj_mx`: a per-row
// NVFP4 quantiser of the BF16 input, then the "mx" GEMV against the NVFP4
// weight; a row's output bits do not depend on M or on the other rows).
//
// Row quantiser: the encoding of nvfp4_enc.cuh (F32 scale2 per row, E4M3
// scale per 16 elements, E2M1 codes), bit-exact with the CPU reference.
//
// Product (the page gives none; reading taken): for output (m, n)
//
//   out = bf16( (sum_b s16a[m,b] * s16w[n,b] * sum_{i<16} ea[m,16b+i] * ew[n,16b+i])
//               * scale2a[m] * scale2w ),
//
// the shape of a block-scaled FP4 MMA with both F32 scales in the epilogue.
// Per 16-block the E2M1 products are summed in half precision by HFMA2 (even
// and odd elements in the two halves): every product is a multiple of 1/4 of
// magnitude <= 36 and each half sums 8 of them, so |sum| <= 288 in steps of
// 1/4 (1152 steps < 2^11) and every step is exact.  p * (s16a * s16w) is
// exact in float32 too (12 + 8 significant bits); only the float32 sum over
// blocks and the two final scalings round, so results agree with the exact
// product within the BF16 tolerance.
//
// Decode layout: a CTA serves MR activation rows; it quantises them into
// shared memory (all threads: per-row amax, then one 16-block per thread and
// step), then each warp reduces one weight row at a time, lane l taking
// blocks l, l+32, ... (8 bytes of codes and one E4M3 byte each, the loads of
// four blocks issued before their arithmetic).  The weight is read as stored,
// 0.5625 B per element.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include <cstdint>
#include <mutex>

#include "bsr.h"
#include "nvfp4_enc.cuh"

namespace bsr {
// Records the message bsr_last_error() returns on this thread (api.cu).
bsr_status report(bsr_status st, const char* fmt, ...);
}  // namespace bsr

namespace bsr {
namespace {

constexpr int kW4A4Unroll = 4;  // weight blocks per lane in flight
constexpr int kW4A4MaxMR = 16;

template <int MR>
constexpr int w4a4_max_threads() { return MR <= 2 ? 1024 : 512; }

__device__ __forceinline__ void bf16x8_unpack(const uint4& v, float* x) {
  x[0] = __uint_as_float(v.x << 16);
  x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16);
  x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  x[4] = __uint_as_float(v.z << 16);
  x[5] = __uint_as_float(v.z & 0xFFFF0000u);
  x[6] = __uint_as_float(v.w << 16);
  x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

__device__ __forceinline__ float amax8(const uint4& v) {
  // |bf16| as float: clear the sign bit of each half
  const uint32_t w[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, __uint_as_float(w[i] << 16));
    m = fmaxf(m, __uint_as_float(w[i] & 0xFFFF0000u));
  }
  return m;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  return v;
}

// Quantise block b of the BF16 row src (16-byte aligned) with the row's
// scale2; codes to dst_packed[b] (8 bytes), scale byte to dst_e4[b].
__device__ __forceinline__ void quant_block_at(const uint16_t* __restrict__ src, int b, float scale2,
                                               uint2* dst_packed, uint8_t* dst_e4) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src) + 2 * (size_t)b;
  float x[16];
  bf16x8_unpack(__ldg(s4), x);
  bf16x8_unpack(__ldg(s4 + 1), x + 8);
  const nvfp4::Block q = nvfp4::quant_block(x, scale2);
  dst_packed[b] = make_uint2(q.lo, q.hi);
  dst_e4[b] = (uint8_t)q.e4;
}

// Standalone row quantiser: one warp per row.
__global__ void __launch_bounds__(256) nvfp4_quant_rows_kernel(const uint16_t* __restrict__ a,
                                                               uint8_t* __restrict__ a_packed,
                                                               uint8_t* __restrict__ a_e4m3,
                                                               float* __restrict__ a_scale2, int m, int k) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int nv = k >> 3;   // 16-byte vectors per row
  const int nb = k >> 4;   // 16-element blocks per row
  for (long long row = warp0; row < m; row += nwarps) {
    const uint16_t* src = a + (size_t)row * (size_t)k;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    float mx = 0.0f;
    for (int i = lane; i < nv; i += 32) mx = fmaxf(mx, amax8(__ldg(s4 + i)));
    const float scale2 = nvfp4::row_scale2(warp_max(mx));
    uint2* dp = reinterpret_cast<uint2*>(a_packed + (size_t)row * (size_t)(k >> 1));
    uint8_t* de = a_e4m3 + (size_t)row * (size_t)nb;
    for (int b = lane; b < nb; b += 32) quant_block_at(src, b, scale2, dp, de);
    if (lane == 0) a_scale2[row] = scale2;
  }
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ __half2 e2m1x2_to_half2(uint32_t byte) {
  const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(byte & 0xFFu), __NV_E2M1);
  return __half2(h);
}

// Shared-memory layout of the decode kernel for MR rows of K elements.
struct DecodeSmem {
  size_t codes, e4, s2, total;
};

__host__ __device__ __forceinline__ DecodeSmem decode_smem(int mr, int k) {
  DecodeSmem s;
  s.codes = 0;                                                      // [MR][K/2]
  s.e4 = (size_t)mr * (size_t)(k >> 1);                             // [MR][K/16]
  s.s2 = (s.e4 + (size_t)mr * (size_t)(k >> 4) + 15) & ~size_t(15);  // [MR] float
  s.total = s.s2 + 4 * (size_t)mr;
  return s;
}

template <int MR>
__global__ void __launch_bounds__(w4a4_max_threads<MR>(), 1)
    w4a4_decode_kernel(const uint16_t* __restrict__ a, const uint8_t* __restrict__ w_packed,
                       const uint8_t* __restrict__ w_e4m3, float scale2_w, __nv_bfloat16* __restrict__ out, int m,
                       int n, int k) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float s_part[MR][32];  // per-warp row amax partials
  const DecodeSmem lay = decode_smem(MR, k);
  uint8_t* s_codes = smem + lay.codes;
  uint8_t* s_e4 = smem + lay.e4;
  float* s_s2 = reinterpret_cast<float*>(smem + lay.s2);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int m0 = blockIdx.y * MR;
  const int rows = min(MR, m - m0);
  const int kp = k >> 1;
  const int nb = k >> 4;
  const int nv = k >> 3;

  // the activations may come from the previous kernel on the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // 1. row amax (all threads), scale2 per row
  {
    float mx[MR];
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      mx[r] = 0.0f;
      if (r < rows) {
        const uint4* s4 = reinterpret_cast<const uint4*>(a + (size_t)(m0 + r) * (size_t)k);
        for (int i = threadIdx.x; i < nv; i += blockDim.x) mx[r] = fmaxf(mx[r], amax8(__ldg(s4 + i)));
      }
      mx[r] = warp_max(mx[r]);
      if (lane == 0) s_part[r][warp] = mx[r];
    }
  }
  __syncthreads();
  if (threadIdx.x < MR) {
    const int r = threadIdx.x;
    float v = 0.0f;
    for (int w = 0; w < nwarps; ++w) v = fmaxf(v, s_part[r][w]);
    s_s2[r] = r < rows ? nvfp4::row_scale2(v) : 0.0f;
  }
  __syncthreads();

  // 2. quantise the rows into shared memory (rows past m: codes and scales 0)
  for (int i = threadIdx.x; i < MR * nb; i += blockDim.x) {
    const int r = i / nb;
    const int b = i - r * nb;
    uint2* dp = reinterpret_cast<uint2*>(s_codes + (size_t)r * kp);
    uint8_t* de = s_e4 + (size_t)r * nb;
    if (r < rows) {
      quant_block_at(a + (size_t)(m0 + r) * (size_t)k, b, s_s2[r], dp, de);
    } else {
      dp[b] = make_uint2(0u, 0u);
      de[b] = 0;
    }
  }
  __syncthreads();

  // 3. GEMV: one weight row per warp
  for (int row = blockIdx.x * nwarps + warp; row < n; row += gridDim.x * nwarps) {
    const uint2* wp = reinterpret_cast<const uint2*>(w_packed + (size_t)row * (size_t)kp);
    const uint8_t* we = w_e4m3 + (size_t)row * (size_t)nb;
    float acc[MR];
#pragma unroll
    for (int r = 0; r < MR; ++r) acc[r] = 0.0f;
    for (int b0 = lane; b0 < nb; b0 += 32 * kW4A4Unroll) {
      uint2 q[kW4A4Unroll];
      uint32_t e[kW4A4Unroll];
#pragma unroll
      for (int u = 0; u < kW4A4Unroll; ++u) {
        const int b = b0 + 32 * u;
        q[u] = b < nb ? __ldg(wp + b) : make_uint2(0u, 0u);
        e[u] = b < nb ? (uint32_t)__ldg(we + b) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kW4A4Unroll; ++u) {
        const int b = b0 + 32 * u;
        if (b >= nb) break;
        __half2 w2[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w2[i] = e2m1x2_to_half2((i < 4 ? q[u].x : q[u].y) >> (8 * (i & 3)));
        const float sw = e4m3_to_f32(e[u]);
#pragma unroll
        for (int r = 0; r < MR; ++r) {
          const uint2 av = *reinterpret_cast<const uint2*>(s_codes + (size_t)r * kp + (size_t)b * 8);
          const float sa = e4m3_to_f32(s_e4[(size_t)r * nb + b]);
          __half2 p2 = __float2half2_rn(0.0f);
#pragma unroll
          for (int i = 0; i < 8; ++i) p2 = __hfma2(e2m1x2_to_half2((i < 4 ? av.x : av.y) >> (8 * (i & 3))), w2[i], p2);
          const float p = __fadd_rn(__low2float(p2), __high2float(p2));  // exact
          acc[r] = __fmaf_rn(p, __fmul_rn(sa, sw), acc[r]);
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
        if (r < rows)
          out[(size_t)(m0 + r) * (size_t)n + row] = __float2bfloat16_rn(__fmul_rn(__fmul_rn(acc[r], s_s2[r]), scale2_w));
    }
  }
}

template <int MR>
cudaError_t launch_w4a4_t(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2_w,
                          uint16_t* out, int m, int n, int k, size_t smem_limit, cudaStream_t stream, int num_sms,
                          int dev) {
  auto kern = w4a4_decode_kernel<MR>;
  const size_t smem = decode_smem(MR, k).total;
  // the kernel's static shared memory (s_part) comes on top
  if (smem + sizeof(float) * MR * 32 > smem_limit) return cudaErrorInvalidValue;
  static size_t granted[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (smem > granted[dev] && smem > 48 * 1024 - sizeof(float) * MR * 32) {
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      granted[dev] = smem;
    }
  }
  // warps (= weight rows in flight) per CTA: spread the rows over all SMs
  int w = (int)((n + (long long)num_sms - 1) / num_sms);
  constexpr int kMaxW = w4a4_max_threads<MR>() / 32;
  w = w < 1 ? 1 : (w > kMaxW ? kMaxW : w);  // >= 32 threads: the MR row scales need MR <= 32
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
  cudaError_t e =
      cudaLaunchKernelEx(&cfg, kern, a, w_packed, w_e4m3, scale2_w, reinterpret_cast<__nv_bfloat16*>(out), m, n, k);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Rows per CTA of the decode kernel: the power of two >= M (at most 16)
// whose quantised rows fit in shared memory; 0 if even one row does not.
int w4a4_rows_per_cta(int m, int k, size_t smem_limit) {
  int mr = 1;
  while (mr < m && mr < kW4A4MaxMR) mr <<= 1;
  while (mr > 1 && decode_smem(mr, k).total + sizeof(float) * mr * 32 > smem_limit) mr >>= 1;
  return decode_smem(mr, k).total + sizeof(float) * mr * 32 > smem_limit ? 0 : mr;
}

// Per-device properties, queried once per device.
struct Dev {
  int num_sms = 0;
  size_t smem_optin = 0;
  int cc_major = 0;
};
Dev g_devs[64];
std::mutex g_devs_mu;

bsr_status query_device(Dev& out, int& dev) {
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return report(BSR_ENODEV, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return report(BSR_ENODEV, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_devs_mu);
  Dev& d = g_devs[dev];
  if (d.num_sms == 0) {
    int sms = 0, smem = 0, major = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return report(BSR_ENODEV, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    d.num_sms = sms;
    d.smem_optin = (size_t)smem;
    d.cc_major = major;
  }
  if (d.cc_major != 10)
    return report(BSR_ENODEV, "device %d has compute capability %d.x, need 10.x (sm_100a)", dev, d.cc_major);
  out = d;
  return BSR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bsr_status check_mk(int64_t m, int64_t k) {
  if (m < 0 || m > BSR_MAX_DIM || k < 0 || k > BSR_MAX_DIM)
    return report(BSR_EINVAL, "dimension out of range (m=%lld k=%lld)", (long long)m, (long long)k);
  if (k == 0 || k % 16 != 0) return report(BSR_ESHAPE, "K=%lld must be a positive multiple of 16", (long long)k);
  return BSR_OK;
}

bsr_status launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return report(BSR_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  return report(BSR_OK, "");
}

}  // namespace

// Row quantiser launch (8 rows per CTA, programmatic stream serialisation so
// a dependent kernel may start its prologue early).
cudaError_t launch_nvfp4_quant_rows(const uint16_t* a, uint8_t* a_packed, uint8_t* a_e4m3, float* a_scale2, int m,
                                    int k, cudaStream_t stream, int num_sms) {
  long long grid = (m + 7) / 8;  // 8 rows (warps) per CTA
  if (grid > 8LL * num_sms) grid = 8LL * num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, nvfp4_quant_rows_kernel, a, a_packed, a_e4m3, a_scale2, m, k);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e;
}

}  // namespace bsr

extern "C" {

bsr_status bsr_nvfp4_quant_rows(const uint16_t* a, uint8_t* a_packed, uint8_t* a_e4m3, float* a_scale2, int64_t m,
                                int64_t k, void* stream) {
  bsr_status st = bsr::check_mk(m, k);
  if (st != BSR_OK) return st;
  if (m == 0) return bsr::report(BSR_OK, "");
  if (!a || !a_packed || !a_e4m3 || !a_scale2) return bsr::report(BSR_EINVAL, "null pointer");
  if (!bsr::aligned16(a) || !bsr::aligned16(a_packed) || !bsr::aligned16(a_e4m3) || !bsr::aligned16(a_scale2))
    return bsr::report(BSR_EALIGN, "a, a_packed, a_e4m3, a_scale2 must be 16-byte aligned");
  bsr::Dev d;
  int dev = 0;
  if ((st = bsr::query_device(d, dev)) != BSR_OK) return st;
  const cudaError_t e = bsr::launch_nvfp4_quant_rows(a, a_packed, a_e4m3, a_scale2, (int)m, (int)k,
                                                     reinterpret_cast<cudaStream_t>(stream), d.num_sms);
  return bsr::launched(e, "nvfp4 row quantiser launch");
}

bsr_status bsr_w4a4_decode(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                           uint16_t* out, int64_t m, int64_t n, int64_t k, void* stream) {
  bsr_status st = bsr::check_mk(m, k);
  if (st != BSR_OK) return st;
  if (n < 0 || n > BSR_MAX_DIM) return bsr::report(BSR_EINVAL, "dimension out of range (n=%lld)", (long long)n);
  if (m == 0 || n == 0) return bsr::report(BSR_OK, "");
  if (!a || !w_packed || !w_e4m3 || !out) return bsr::report(BSR_EINVAL, "null pointer");
  if (!bsr::aligned16(a) || !bsr::aligned16(w_packed) || !bsr::aligned16(w_e4m3) ||
      (reinterpret_cast<uintptr_t>(out) & 1u))
    return bsr::report(BSR_EALIGN, "a, w_packed, w_e4m3 must be 16-byte aligned, out 2-byte aligned");
  if ((m + bsr::kW4A4MaxMR - 1) / bsr::kW4A4MaxMR > 65535)
    return bsr::report(BSR_EINVAL, "M=%lld too large for the decode grid", (long long)m);
  bsr::Dev d;
  int dev = 0;
  if ((st = bsr::query_device(d, dev)) != BSR_OK) return st;
  const int mr = bsr::w4a4_rows_per_cta((int)m, (int)k, d.smem_optin);
  if (mr == 0)
    return bsr::report(BSR_ESHAPE, "K=%lld too large for one quantised activation row in shared memory", (long long)k);
  cudaError_t e;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (mr) {
    case 1: e = bsr::launch_w4a4_t<1>(a, w_packed, w_e4m3, scale2, out, (int)m, (int)n, (int)k, d.smem_optin, s, d.num_sms, dev); break;
    case 2: e = bsr::launch_w4a4_t<2>(a, w_packed, w_e4m3, scale2, out, (int)m, (int)n, (int)k, d.smem_optin, s, d.num_sms, dev); break;
    case 4: e = bsr::launch_w4a4_t<4>(a, w_packed, w_e4m3, scale2, out, (int)m, (int)n, (int)k, d.smem_optin, s, d.num_sms, dev); break;
    case 8: e = bsr::launch_w4a4_t<8>(a, w_packed, w_e4m3, scale2, out, (int)m, (int)n, (int)k, d.smem_optin, s, d.num_sms, dev); break;
    default: e = bsr::launch_w4a4_t<16>(a, w_packed, w_e4m3, scale2, out, (int)m, (int)n, (int)k, d.smem_optin, s, d.num_sms, dev); break;
  }
  return bsr::launched(e, "w4a4 decode launch");
}

}  // extern "C"
