// Decode path (few activation rows): out[M, N] = A[M, K] . W[N, K]^T with the
// activation requantisation fused in, on CUDA cores only (dp4a), split over K
// across the 32 lanes of a warp with a fixed-order shuffle reduction.
//
// Same arithmetic per 32-block as the tensor-core path: P = exact int32 dot
// product of the codes, u = RN(float(P) * w_scale), acc = fma(u, a_scale, acc);
// the blocks of one output are summed lane-cyclically (lane l takes blocks
// l, l+32, ...) and the 32 lane sums are added in a fixed xor tree, so an
// output's bits depend only on K, never on M, N or the launch grid.
//
// Each CTA re-quantises the activation rows it serves into shared memory (a
// few KB read from L2), after issuing its first weight loads so the HBM
// latency overlaps with that work.  The int8 codes and scales match the
// standalone requant_a kernel bit for bit (same rule, same quant.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace bsr {

constexpr int kDecodeWarps = 8;
constexpr int kDecodeUnroll = 4;  // 32-blocks per lane in flight

__device__ __forceinline__ void bf16x8_to_f32_d(const uint4& v, float (&x)[8]) {
  x[0] = __uint_as_float(v.x << 16);
  x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16);
  x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  x[4] = __uint_as_float(v.z << 16);
  x[5] = __uint_as_float(v.z & 0xFFFF0000u);
  x[6] = __uint_as_float(v.w << 16);
  x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

__device__ __forceinline__ int dot32(const uint4& w0, const uint4& w1, const uint4& a0, const uint4& a1) {
  int p = 0;
  p = __dp4a((int)w0.x, (int)a0.x, p);
  p = __dp4a((int)w0.y, (int)a0.y, p);
  p = __dp4a((int)w0.z, (int)a0.z, p);
  p = __dp4a((int)w0.w, (int)a0.w, p);
  p = __dp4a((int)w1.x, (int)a1.x, p);
  p = __dp4a((int)w1.y, (int)a1.y, p);
  p = __dp4a((int)w1.z, (int)a1.z, p);
  p = __dp4a((int)w1.w, (int)a1.w, p);
  return p;
}

// MR: activation rows per CTA (compile time, >= rows actually present).
// Shared memory: codes [MR][K] int8, then scales [MR][K/32] f32.
template <int MR>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_kernel(const uint16_t* __restrict__ a,
                                                                    const int8_t* __restrict__ w_i8,
                                                                    const float* __restrict__ w_scale,
                                                                    __nv_bfloat16* __restrict__ out, int m, int n,
                                                                    int k) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int nb = k >> 5;
  int8_t* s_codes = reinterpret_cast<int8_t*>(smem);
  float* s_scale = reinterpret_cast<float*>(smem + (size_t)MR * k);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * MR;
  const int rows = min(MR, m - m0);

  int row = blockIdx.x * kDecodeWarps + warp;
  const int row_step = gridDim.x * kDecodeWarps;

  // First weight tile of this warp's first row, issued before the activation pass.
  uint4 wv[kDecodeUnroll][2];
  float ws[kDecodeUnroll];
  auto load_tile = [&](int r, int it) {
#pragma unroll
    for (int u = 0; u < kDecodeUnroll; ++u) {
      const int b = (it * kDecodeUnroll + u) * 32 + lane;
      if (r < n && b < nb) {
        const uint4* src = reinterpret_cast<const uint4*>(w_i8 + (size_t)r * k + (size_t)b * 32);
        wv[u][0] = __ldg(src);
        wv[u][1] = __ldg(src + 1);
        ws[u] = __ldg(w_scale + (size_t)r * nb + b);
      } else {
        wv[u][0] = wv[u][1] = make_uint4(0, 0, 0, 0);
        ws[u] = 0.0f;
      }
    }
  };
  load_tile(row, 0);

  // Activation requantisation into shared memory: 4 lanes per 32-group.
  {
    const int groups = MR * nb;
    const int sub = lane & 3;
    for (int g0 = warp * 8; g0 < groups; g0 += kDecodeWarps * 8) {
      const int g = g0 + (lane >> 2);
      const int r = g / nb;
      const int b = g - r * nb;
      const bool valid = (g < groups) && (r < rows);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (valid) v = __ldg(reinterpret_cast<const uint4*>(a + (size_t)(m0 + r) * k + (size_t)b * 32 + sub * 8));
      float x[8];
      bf16x8_to_f32_d(v, x);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
      const GroupScale gs = group_scale(amax);
      int q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = (gs.scale == 0.0f) ? 0 : quant_code(x[i], gs);
      if (g < groups) {
        *reinterpret_cast<uint2*>(s_codes + (size_t)r * k + (size_t)b * 32 + sub * 8) =
            make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
        if (sub == 0) s_scale[r * nb + b] = gs.scale;
      }
    }
  }
  __syncthreads();

  // Lane l reads the two 16-byte halves of its block in the order h, 1-h with
  // h = (l >> 2) & 1, so that each 8-lane phase of a 16-byte shared load hits
  // eight distinct 16-byte bank groups.
  const int h = (lane >> 2) & 1;
  const int iters = (nb + 32 * kDecodeUnroll - 1) / (32 * kDecodeUnroll);

  for (; row < n; row += row_step) {
    float acc[MR];
#pragma unroll
    for (int r = 0; r < MR; ++r) acc[r] = 0.0f;
    for (int it = 0; it < iters; ++it) {
      if (it > 0) load_tile(row, it);
#pragma unroll
      for (int u = 0; u < kDecodeUnroll; ++u) {
        const int b = (it * kDecodeUnroll + u) * 32 + lane;
        if (b < nb) {
          const uint4 w0 = h ? wv[u][1] : wv[u][0];
          const uint4 w1 = h ? wv[u][0] : wv[u][1];
#pragma unroll
          for (int r = 0; r < MR; ++r) {
            const uint4* cs = reinterpret_cast<const uint4*>(s_codes + (size_t)r * k + (size_t)b * 32);
            const uint4 a0 = cs[h];
            const uint4 a1 = cs[1 - h];
            const int p = dot32(w0, w1, a0, a1);
            const float u_ = __fmul_rn((float)p, ws[u]);
            acc[r] = __fmaf_rn(u_, s_scale[r * nb + b], acc[r]);
          }
        }
      }
    }
    // fixed-order reduction over the 32 lanes
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
        if (r < rows) out[(size_t)(m0 + r) * n + row] = __float2bfloat16_rn(acc[r]);
    }
    const int next = row + row_step;
    if (next < n) load_tile(next, 0);
  }
}

static size_t decode_smem(int mr, int k) { return (size_t)mr * k + (size_t)mr * (k / 32) * 4; }

// Rows per CTA: the largest power of two <= 16 that covers M and fits the
// shared-memory budget.
int decode_rows_per_cta(int m, int k, size_t smem_limit) {
  int mr = 1;
  while (mr < m && mr < 16) mr <<= 1;
  while (mr > 1 && decode_smem(mr, k) > smem_limit) mr >>= 1;
  if (decode_smem(mr, k) > smem_limit) return 0;
  return mr;
}

template <int MR>
static cudaError_t launch_decode_t(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int m,
                                   int n, int k, cudaStream_t stream, int num_sms) {
  const size_t smem = decode_smem(MR, k);
  auto kern = decode_kernel<MR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeWarps * 32, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  long long gx = (n + kDecodeWarps - 1) / kDecodeWarps;
  const long long cap = (long long)num_sms * per_sm;
  const int gy = (m + MR - 1) / MR;
  if (gx * gy > cap) gx = (cap + gy - 1) / gy;
  if (gx < 1) gx = 1;
  dim3 grid((unsigned)gx, (unsigned)gy);
  kern<<<grid, kDecodeWarps * 32, smem, stream>>>(a, w_i8, w_scale, reinterpret_cast<__nv_bfloat16*>(out), m, n, k);
  return cudaGetLastError();
}

cudaError_t launch_decode(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int m, int n,
                          int k, int mr, cudaStream_t stream, int num_sms) {
  switch (mr) {
    case 1: return launch_decode_t<1>(a, w_i8, w_scale, out, m, n, k, stream, num_sms);
    case 2: return launch_decode_t<2>(a, w_i8, w_scale, out, m, n, k, stream, num_sms);
    case 4: return launch_decode_t<4>(a, w_i8, w_scale, out, m, n, k, stream, num_sms);
    case 8: return launch_decode_t<8>(a, w_i8, w_scale, out, m, n, k, stream, num_sms);
    case 16: return launch_decode_t<16>(a, w_i8, w_scale, out, m, n, k, stream, num_sms);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace bsr
