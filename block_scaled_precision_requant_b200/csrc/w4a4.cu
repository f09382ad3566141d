// NVFP4 W4A4 decode route (w4a4_proj/fixed.rs, `nvfp4_proj_mx`: a per-row
// NVFP4 quantiser of the BF16 input, then the "mx" GEMV against the NVFP4
// weight; a row's output bits do not depend on M or on the other rows).
//
// Here: the standalone row quantiser (the encoding of nvfp4_enc.cuh, F32
// scale2 per row, E4M3 scale per 16 elements, E2M1 codes; bit-exact with the
// CPU reference) and the C entry points of the decode GEMV, whose kernel
// (the quantiser fused in) is shared with W4A16 in nvfp4_gemv.cu.
#include <cstdint>
#include <mutex>

#include "bsr.h"
#include "kernels.h"
#include "nvfp4_enc.cuh"

namespace bsr {
// Records the message bsr_last_error() returns on this thread (api.cu).
bsr_status report(bsr_status st, const char* fmt, ...);
// Device address of the library's status word on the current device (api.cu).
bsr_status library_status_word(int** out);
}  // namespace bsr

namespace bsr {
namespace {

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

// Per-device properties, queried once per device.
struct Dev {
  int num_sms = 0;
  size_t smem_optin = 0;
  size_t smem_per_sm = 0;
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
    int sms = 0, smem = 0, smem_sm = 0, major = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return report(BSR_ENODEV, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    d.num_sms = sms;
    d.smem_optin = (size_t)smem;
    d.smem_per_sm = (size_t)smem_sm;
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

bsr_status bsr_w4a4_decode_ex(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                              uint16_t* out, int64_t m, int64_t n, int64_t k, unsigned flags, void* stream) {
  bsr_status st = bsr::check_mk(m, k);
  if (st != BSR_OK) return st;
  if (n < 0 || n > BSR_MAX_DIM) return bsr::report(BSR_EINVAL, "dimension out of range (n=%lld)", (long long)n);
  if (flags & ~BSR_DECODE_STATIC_WEIGHT) return bsr::report(BSR_EINVAL, "unknown flags 0x%x", flags);
  if (m == 0 || n == 0) return bsr::report(BSR_OK, "");
  if (!a || !w_packed || !w_e4m3 || !out) return bsr::report(BSR_EINVAL, "null pointer");
  if (!bsr::aligned16(a) || !bsr::aligned16(w_packed) || !bsr::aligned16(w_e4m3) ||
      (reinterpret_cast<uintptr_t>(out) & 1u))
    return bsr::report(BSR_EALIGN, "a, w_packed, w_e4m3 must be 16-byte aligned, out 2-byte aligned");
  bsr::Dev d;
  int dev = 0;
  if ((st = bsr::query_device(d, dev)) != BSR_OK) return st;
  int* status = nullptr;
  if ((st = bsr::library_status_word(&status)) != BSR_OK) return st;
  bsr::GemvPlan p;
  if (!bsr::nvfp4_gemv_plan((int)m, (int)n, (int)k, true, d.smem_optin, d.smem_per_sm, d.num_sms, p))
    return bsr::report(BSR_ESHAPE, "K=%lld, M=%lld outside the NVFP4 GEMV (K <= 65536 with one activation row and one weight stage in shared memory)",
                       (long long)k, (long long)m);
  const cudaError_t e = bsr::launch_nvfp4_gemv(p, true, a, w_packed, w_e4m3, scale2, out, (int)m, (int)n, (int)k,
                                               (flags & BSR_DECODE_STATIC_WEIGHT) ? 1 : 0, status,
                                               reinterpret_cast<cudaStream_t>(stream));
  return bsr::launched(e, "w4a4 decode launch");
}

bsr_status bsr_w4a4_decode(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                           uint16_t* out, int64_t m, int64_t n, int64_t k, void* stream) {
  return bsr_w4a4_decode_ex(a, w_packed, w_e4m3, scale2, out, m, n, k, 0u, stream);
}

}  // extern "C"
