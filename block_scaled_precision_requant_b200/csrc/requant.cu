// Requantisation kernels (HBM-bound):
//
//  * requant_w: NVFP4 weight -> int8 codes + one F32 scale per 32 elements
//    (gemm_dense_int8.rs, `requant_w_nvfp4_int8`: reads W_packed[N, K/2] and
//    W_e4m3[N, K/16], folds the per-tensor scale2, writes W_i8[N, K] and
//    W_scale[N, K/32]).
//  * requant_a: BF16 activations -> int8 codes + one F32 scale per 32
//    elements (gemm_dense_int8.rs, `requant_a_kernel` inside
//    `int8_gemm_faith2_prefill`).  The scales are written block-major,
//    a_scale_t[K/32][ld], which is the layout the tensor-core GEMM stages.
#include "common.cuh"
#include "fp_cvt.cuh"
#include "kernels.h"
#include "occupancy.h"
#include "quant.cuh"

namespace bsr {

// ---------------------------------------------------------------------------
// requant_w
//
// One thread per 32-group: 16 packed bytes (32 E2M1 nibbles, element 2i in
// the low nibble of byte i), two E4M3 block scales, 32 output codes and one
// scale.  A 16-element block shares one E4M3 scale, so its dequantised values
// take at most 8 magnitudes: v_i = RN((e2m1_i * e4m3) * scale2), i = 0..7.
// The kernel quantises those 8 candidates once per block and maps every
// nibble to its code with byte permutes; codes of negative nibbles are the
// negated codes (rint half-even and the division are odd functions).
// ---------------------------------------------------------------------------

// E2M1 magnitude of index i (0..7): 0, .5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_mag(uint32_t i) {
  if (i == 0) return 0.0f;
  if (i == 1) return 0.5f;
  return __uint_as_float((((i >> 1) + 126u) << 23) | ((i & 1u) << 22));
}

// Largest nibble magnitude index (0..7) among the 16 nibbles of (x, y).
__device__ __forceinline__ uint32_t max_mag_index(uint32_t x, uint32_t y) {
  const uint32_t gx = (x & 0x77777777u) | 0x88888888u;
  const uint32_t gy = (y & 0x77777777u) | 0x88888888u;
  // nibble n >= t  <=>  ((8 + n) - t) keeps bit 3; no borrow crosses nibbles
  auto any_ge = [&](uint32_t t) {
    const uint32_t rep = t * 0x11111111u;
    return (((gx - rep) | (gy - rep)) & 0x88888888u) != 0u;
  };
  uint32_t lo = any_ge(4) ? 4u : 0u;
  lo += any_ge(lo + 2) ? 2u : 0u;
  lo += any_ge(lo + 1) ? 1u : 0u;
  return lo;
}

struct CodeTable {
  uint32_t pos_lo, pos_hi, neg_lo, neg_hi;  // codes of magnitude index 0..7 (bytes)
};

__device__ __forceinline__ CodeTable block_codes(float s_e4m3, float scale2, const GroupScale& g) {
  int q[8];
  q[0] = 0;
  if (g.rcp != 0.0f) {
#pragma unroll
    for (int i = 1; i < 8; ++i)
      q[i] = quant_code_rcp(__fmul_rn(e2m1_mag(i) * s_e4m3, scale2), g);  // e2m1 * e4m3 is exact
  } else {
#pragma unroll
    for (int i = 1; i < 8; ++i) {
      const float v = __fmul_rn(e2m1_mag(i) * s_e4m3, scale2);
      q[i] = (g.scale == 0.0f) ? 0 : quant_code(v, g);
    }
  }
  CodeTable t;
  t.pos_lo = pack4_cvt(q[0], q[1], q[2], q[3]);
  t.pos_hi = pack4_cvt(q[4], q[5], q[6], q[7]);
  t.neg_lo = pack4_cvt(-q[0], -q[1], -q[2], -q[3]);
  t.neg_hi = pack4_cvt(-q[4], -q[5], -q[6], -q[7]);
  return t;
}

// Byte permute in the PTX default mode: a selector nibble with bit 3 set
// replicates the sign (bit 7) of the selected byte into the whole byte.
__device__ __forceinline__ uint32_t prmt_sign(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Codes of the 8 nibbles of w (elements 0..7 of the word) -> two words.
__device__ __forceinline__ uint2 map_word(uint32_t w, const CodeTable& t) {
  const uint32_t sel0 = w & 0x7777u;
  const uint32_t sel1 = (w >> 16) & 0x7777u;
  // sign bits: odd nibbles' signs are the byte MSBs of w, even nibbles' are
  // the byte MSBs of w << 4; replicate them into byte masks
  const uint32_t ws = w << 4;
  const uint32_t m0 = prmt_sign(ws, w, 0xD9C8u);
  const uint32_t m1 = prmt_sign(ws, w, 0xFBEAu);
  const uint32_t p0 = __byte_perm(t.pos_lo, t.pos_hi, sel0);
  const uint32_t n0 = __byte_perm(t.neg_lo, t.neg_hi, sel0);
  const uint32_t p1 = __byte_perm(t.pos_lo, t.pos_hi, sel1);
  const uint32_t n1 = __byte_perm(t.neg_lo, t.neg_hi, sel1);
  return make_uint2((p0 & ~m0) | (n0 & m0), (p1 & ~m1) | (n1 & m1));
}


__global__ void __launch_bounds__(256) requant_w_kernel(const uint4* __restrict__ w_packed,
                                                        const uint16_t* __restrict__ w_e4m3, float scale2,
                                                        uint4* __restrict__ w_i8, float* __restrict__ w_scale,
                                                        long long groups) {
  for (long long gi = (long long)blockIdx.x * blockDim.x + threadIdx.x; gi < groups;
       gi += (long long)gridDim.x * blockDim.x) {
    const uint4 p = __ldg(w_packed + gi);
    // both E4M3 scales of the group by one hardware conversion (exact)
    const uint32_t e2 = e4m3x2_to_f16x2(__ldg(w_e4m3 + gi));
    const float s0 = f16_lo_to_f32(e2);
    const float s1 = f16_hi_to_f32(e2);
    const uint32_t i0 = max_mag_index(p.x, p.y);
    const uint32_t i1 = max_mag_index(p.z, p.w);
    const float a0 = fabsf(__fmul_rn(e2m1_mag(i0) * s0, scale2));
    const float a1 = fabsf(__fmul_rn(e2m1_mag(i1) * s1, scale2));
    const GroupScale g = group_scale(fmaxf(a0, a1));
    const CodeTable t0 = block_codes(s0, scale2, g);
    const CodeTable t1 = block_codes(s1, scale2, g);
    const uint2 c0 = map_word(p.x, t0), c1 = map_word(p.y, t0);
    const uint2 c2 = map_word(p.z, t1), c3 = map_word(p.w, t1);
    w_i8[2 * gi] = make_uint4(c0.x, c0.y, c1.x, c1.y);
    w_i8[2 * gi + 1] = make_uint4(c2.x, c2.y, c3.x, c3.y);
    w_scale[gi] = g.scale;
  }
}

// ---------------------------------------------------------------------------
// requant_a
//
// One thread per 32-group: four 16-byte loads (64 contiguous bytes), the
// amax by packed 16-bit max, the group scale once, 32 codes in two 16-byte
// stores.  A warp takes 8 consecutive rows x 4 consecutive blocks (lane L:
// row 8R + L%8, block 4B + L/8), so its loads are eight 256-byte row
// segments, its codes eight 128-byte segments, and its scales four 32-byte
// segments of the block-major scale array.  The next task's loads are issued
// before the current task's arithmetic.
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) requant_a_kernel(const uint16_t* __restrict__ a, int8_t* __restrict__ a_i8,
                                                        float* __restrict__ a_scale_t, int m, int k, int ld) {
  const int lane = threadIdx.x & 31;
  const int nb = k >> 5;
  const int nb4 = (nb + 3) >> 2;
  const long long tasks = (long long)((m + 7) >> 3) * nb4;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  auto locate = [&](long long t, int& row, int& blk) {
    const long long r8 = t / nb4;
    row = (int)(r8 * 8) + (lane & 7);
    blk = (int)(t - r8 * nb4) * 4 + (lane >> 3);
  };
  auto load = [&](int row, int blk, uint4 (&v)[4]) {
    if (row < m && blk < nb) {
      const uint4* src = reinterpret_cast<const uint4*>(a + (size_t)row * k + (size_t)blk * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = __ldg(src + i);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = make_uint4(0, 0, 0, 0);
    }
  };
  long long t = warp0;
  if (t >= tasks) return;
  int row, blk;
  locate(t, row, blk);
  uint4 v[4];
  load(row, blk, v);
  for (; t < tasks; t += nwarps) {
    int nrow = 0, nblk = 0;
    uint4 nv[4];
    if (t + nwarps < tasks) {
      locate(t + nwarps, nrow, nblk);
      load(nrow, nblk, nv);
    }
    uint4 lo, hi;
    float scale;
    quant_group32(v, lo, hi, scale);
    if (row < m && blk < nb) {
      uint4* dst = reinterpret_cast<uint4*>(a_i8 + (size_t)row * k + (size_t)blk * 32);
      dst[0] = lo;
      dst[1] = hi;
      a_scale_t[(size_t)blk * ld + row] = scale;
    }
    row = nrow;
    blk = nblk;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = nv[i];
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

static int grid_for(long long work_items, int per_block, int max_blocks) {
  long long g = (work_items + per_block - 1) / per_block;
  if (g < 1) g = 1;
  if (g > max_blocks) g = max_blocks;
  return (int)g;
}

cudaError_t launch_requant_w(const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2, int8_t* w_i8,
                             float* w_scale, long long n, long long k, cudaStream_t stream, int num_sms) {
  const long long groups = n * (k / 32);
  const int grid = grid_for(groups, 256, num_sms * resident_ctas_per_sm((const void*)requant_w_kernel, 256));
  requant_w_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(w_packed),
                                             reinterpret_cast<const uint16_t*>(w_e4m3), scale2,
                                             reinterpret_cast<uint4*>(w_i8), w_scale, groups);
  return cudaGetLastError();
}

cudaError_t launch_requant_a(const uint16_t* a, int8_t* a_i8, float* a_scale_t, int m, int k, int ld,
                             cudaStream_t stream, int num_sms) {
  // warp tasks of 8 rows x 4 blocks, 8 warps per CTA
  const long long tasks = (long long)((m + 7) / 8) * ((k / 32 + 3) / 4);
  const int grid = grid_for(tasks, 8, num_sms * resident_ctas_per_sm((const void*)requant_a_kernel, 256));
  requant_a_kernel<<<grid, 256, 0, stream>>>(a, a_i8, a_scale_t, m, k, ld);
  return cudaGetLastError();
}

}  // namespace bsr
