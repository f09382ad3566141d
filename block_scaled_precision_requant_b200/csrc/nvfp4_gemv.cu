// NVFP4 decode GEMVs on the weight as stored (w_packed [N, K/2] E2M1 pairs,
// element 2i in the low nibble of byte i; w_e4m3 [N, K/16]; one F32
// scale2), 0.5625 B per weight element:
//
//  * W4A16 (gemv_sw.rs: `w4a16_gemv` / `w4a16_gemv_sw`; the page fixes the
//    launch arguments, not the arithmetic).  Reading taken:
//      out[m, n] = bf16( scale2 * sum_b e4m3[n, b] * p[m, n, b] ),
//      p = sum_{i<16} A[m, 16b+i] * e2m1[n, 16b+i]
//    accumulated in float32: per 16-element block the 16 products are
//    summed in element order by FMAs, then acc = fma(p, e4m3, acc).
//  * W4A4 (w4a4_proj/fixed.rs, `nvfp4_proj_mx`: a per-row NVFP4 quantiser of
//    the BF16 input, then the "mx" GEMV).  Reading taken: each activation row
//    is encoded as the weight is stored (nvfp4_enc.cuh), and
//      out[m, n] = bf16( (sum_b s16a * s16w * sum_{i<16} ea * ew) * scale2a[m] * scale2w ),
//    the 16-element sums exact (half-precision FMAs on E2M1 values: each
//    product a multiple of 1/4 of magnitude <= 36, each half-sum of 8 in
//    steps of 1/4 below 2^11 steps), the sum over blocks in float32.
//
// Arithmetic per element: the weight nibbles are converted to f16 by the
// hardware E2M1 conversion (two per instruction).  W4A16: each activation
// 16-block is scaled by a power of two 2^s (its largest magnitude into
// [2^15, 2^16)) and stored as f16 -- exact for every element within 2^32 of
// the block's largest, BF16 having 8 significant bits and f16 11 -- and the
// products are accumulated by the mixed-precision FMA (f16 x f16 + float32,
// the product exact, one rounding), then acc = fma(p', e4m3 * 2^-s, acc):
// scaling by 2^s commutes with every float32 rounding, so this is the
// float32 evaluation above.  W4A4: the codes of the quantised rows are
// expanded to f16 once per CTA and the products summed by f16x2 FMAs.
//
// Work split: a CTA owns a contiguous range of weight rows, in stages of RS
// rows (4 for K <= 8192); warp w takes stages w, w + W, ...  The CTA first
// stores its MR activation rows in shared memory in the form above; then
// each warp reduces its stages, lane l taking the 16-blocks l, l + 32, ...
// of every row of the stage.  An output is, in this fixed order, the
// per-lane sum over the lane's blocks (increasing), then the xor tree over
// the 32 lanes (masks 16, 8, 4, 2, 1): its bits depend only on K and its
// own inputs, never on M, N or the grid.
//
// Weight stream: each warp's stages go through its own ring of slots (codes
// then scales, one bulk copy each, completing on the slot's mbarrier), all
// slots issued at kernel start -- before waiting for the previous kernel on
// the stream when the caller declares the weight static -- and refilled by
// the warp as it consumes them.  At the decode shape (N = K = 4096) a CTA
// holds its whole weight share (64.5 KB) in 7 warps and leaves room on the
// SM for the next launch's CTA, which streams its weight while this one
// computes.  K % 256 != 0 (row pitches not 16-byte multiples): the warps
// read the weight from global memory instead, same arithmetic.
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "fp_cvt.cuh"
#include "kernels.h"
#include "nvfp4_enc.cuh"

namespace bsr {

namespace {

constexpr int kGemvMaxWarps = 16;

__host__ __device__ inline uint32_t up16(uint32_t x) { return (x + 15u) & ~15u; }

// Shared-memory layout of one CTA (byte offsets).
struct GemvSmem {
  uint32_t act, fac, s2, amax, slots, bars, abort_flag, total;
  uint32_t codes_bytes, stage_bytes;  // per stage: codes [RS][K/2], then scales [RS][K/16]
};

__host__ __device__ inline GemvSmem gemv_smem(int k, int mr, int rs, int warps, int slots, bool bulk) {
  GemvSmem L;
  const uint32_t kp = (uint32_t)k / 2, nb = (uint32_t)k / 16;
  L.act = 0;                                          // [MR][K/16] blocks of 32 B (f16)
  L.fac = L.act + (uint32_t)mr * (uint32_t)k * 2u;   // [MR][K/16] float
  L.s2 = up16(L.fac + (uint32_t)mr * nb * 4u);       // [MR] float (W4A4)
  L.amax = up16(L.s2 + (uint32_t)mr * 4u);           // [MR][warps] float (W4A4)
  L.codes_bytes = (uint32_t)rs * kp;
  L.stage_bytes = up16(L.codes_bytes + (uint32_t)rs * nb);
  (void)bulk;
  L.slots = (L.amax + (uint32_t)(mr * warps) * 4u + 127u) & ~127u;
  L.bars = L.slots + (uint32_t)(warps * slots) * L.stage_bytes;
  L.abort_flag = L.bars + (uint32_t)(warps * slots) * 8u;
  L.total = L.abort_flag + 16u;
  return L;
}

// Byte offset of half h (0: elements 0..7, 1: elements 8..15) of block b in
// an activation row: the halves of blocks with bit 2 set are swapped, so
// that the 16-byte loads of a quarter warp (lanes 4i .. 4i+3 read half 0 of
// four consecutive blocks, the next four lanes of the next four) hit eight
// distinct 16-byte bank groups.
__host__ __device__ inline uint32_t act_half(uint32_t b, uint32_t h) { return 32u * b + 16u * (h ^ ((b >> 2) & 1u)); }

// Largest |x| over 16 BF16 values as BF16 bits (packed 16-bit max).
__device__ __forceinline__ uint32_t bf16x16_absmax_bits(const uint4& v0, const uint4& v1) {
  const uint32_t c = 0x7FFF7FFFu;
  uint32_t m = __vmaxu2(__vmaxu2(v0.x & c, v0.y & c), __vmaxu2(v0.z & c, v0.w & c));
  m = __vmaxu2(m, __vmaxu2(__vmaxu2(v1.x & c, v1.y & c), __vmaxu2(v1.z & c, v1.w & c)));
  return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ float bf16x16_amax_f32(const uint4& v0, const uint4& v1) {
  return __uint_as_float(bf16x16_absmax_bits(v0, v1) << 16);
}

// W4A16 activation block: 16 BF16 values -> 8 f16x2 words scaled by 2^s,
// s = min(142 - E, 126) for the BF16 exponent field E of the block's largest
// magnitude (which so lands in [2^15, 2^16)); returns 2^-s.
__device__ __forceinline__ float a16_block(const uint4& v0, const uint4& v1, uint4& h0, uint4& h1) {
  const int e = (int)(bf16x16_absmax_bits(v0, v1) >> 7);
  const int s = min(142 - e, 126);
  const float mul = __uint_as_float((uint32_t)(s + 127) << 23);
  auto cv = [&](uint32_t w) {
    return f32x2_to_f16x2(__fmul_rn(__uint_as_float(w << 16), mul), __fmul_rn(__uint_as_float(w & 0xFFFF0000u), mul));
  };
  h0 = make_uint4(cv(v0.x), cv(v0.y), cv(v0.z), cv(v0.w));
  h1 = make_uint4(cv(v1.x), cv(v1.y), cv(v1.z), cv(v1.w));
  return __uint_as_float((uint32_t)(127 - s) << 23);
}

__device__ __forceinline__ void bf16x16_to_f32(const uint4& v0, const uint4& v1, float (&x)[16]) {
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Sum over the 32 lanes of RS per-lane values, one per row: the rows are
// split on lane bit 4 (RS = 4: then bit 3) before the remaining masks, so
// that lane (32 / RS) * g ends with row g; every row still gets the xor
// tree of masks 16, 8, 4, 2, 1 (addition is commutative).
template <int RS>
__device__ __forceinline__ float lane_sum(const float (&v)[RS], int lane) {
  float x;
  if constexpr (RS == 4) {
    const bool hi4 = (lane & 16) != 0, hi3 = (lane & 8) != 0;
    const float s0 = __shfl_xor_sync(0xFFFFFFFFu, hi4 ? v[0] : v[2], 16);
    const float s1 = __shfl_xor_sync(0xFFFFFFFFu, hi4 ? v[1] : v[3], 16);
    const float k0 = __fadd_rn(hi4 ? v[2] : v[0], s0);
    const float k1 = __fadd_rn(hi4 ? v[3] : v[1], s1);
    x = __fadd_rn(hi3 ? k1 : k0, __shfl_xor_sync(0xFFFFFFFFu, hi3 ? k0 : k1, 8));
    x = __fadd_rn(x, __shfl_xor_sync(0xFFFFFFFFu, x, 4));
  } else if constexpr (RS == 2) {
    const bool hi4 = (lane & 16) != 0;
    x = __fadd_rn(hi4 ? v[1] : v[0], __shfl_xor_sync(0xFFFFFFFFu, hi4 ? v[0] : v[1], 16));
    x = __fadd_rn(x, __shfl_xor_sync(0xFFFFFFFFu, x, 8));
    x = __fadd_rn(x, __shfl_xor_sync(0xFFFFFFFFu, x, 4));
  } else {
    x = v[0];
#pragma unroll
    for (int off = 16; off >= 4; off >>= 1) x = __fadd_rn(x, __shfl_xor_sync(0xFFFFFFFFu, x, off));
  }
  x = __fadd_rn(x, __shfl_xor_sync(0xFFFFFFFFu, x, 2));
  return __fadd_rn(x, __shfl_xor_sync(0xFFFFFFFFu, x, 1));
}

template <int MR, int RS, bool A4>
__global__ void __launch_bounds__(kGemvMaxWarps * 32, 1)
    nvfp4_gemv_kernel(const uint16_t* __restrict__ a, const uint8_t* __restrict__ w_packed,
                      const uint8_t* __restrict__ w_e4m3, float scale2_w, __nv_bfloat16* __restrict__ out, int m,
                      int n, int k, int rows_per_cta, int slots, int bulk, int static_weight,
                      int* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int kp = k >> 1;
  const int nb = k >> 4;
  const GemvSmem L = gemv_smem(k, MR, RS, nwarps, slots, bulk != 0);
  float* s_fac = reinterpret_cast<float*>(smem + L.fac);
  float* s_s2 = reinterpret_cast<float*>(smem + L.s2);
  float* s_amax = reinterpret_cast<float*>(smem + L.amax);
  uint8_t* my_slots = smem + L.slots + (uint32_t)(warp * slots) * L.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * slots;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.abort_flag);

  const int m0 = blockIdx.y * MR;
  const int rows = min(MR, m - m0);
  const int r_begin = blockIdx.x * rows_per_cta;
  const int r_end = min(n, r_begin + rows_per_cta);
  const int n_st = (r_end - r_begin + RS - 1) / RS;                         // stages of the CTA
  const int my_st = warp < n_st ? (n_st - warp + nwarps - 1) / nwarps : 0;  // stages warp + j * W

  // lane 0: this warp's j-th stage into slot j % slots
  auto issue = [&](int j) {
    if (lane == 0 && j < my_st) {
      const int row0 = r_begin + (warp + j * nwarps) * RS;
      const int nr = min(RS, r_end - row0);
      uint8_t* dst = my_slots + (uint32_t)(j % slots) * L.stage_bytes;
      uint64_t* bar = &bars[j % slots];
      const uint32_t cb = (uint32_t)nr * (uint32_t)kp, sb = (uint32_t)nr * (uint32_t)nb;
      mbar_arrive_expect_tx(bar, cb + sb);
      bulk_load(dst, w_packed + (size_t)row0 * (size_t)kp, cb, bar);
      bulk_load(dst + L.codes_bytes, w_e4m3 + (size_t)row0 * (size_t)nb, sb, bar);
    }
  };

  if (threadIdx.x == 0) *abort_flag = 0;
  if (A4 && threadIdx.x < MR) s_amax[threadIdx.x] = 0.0f;  // row maxima of the one-pass quantiser
  if (bulk && lane == 0) {
    for (int s = 0; s < slots; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  if (A4)
    __syncthreads();
  else
    __syncwarp();
  const int first = min(slots, my_st);
  // Launched with programmatic stream serialisation: wait for the previous
  // kernel on the stream before reading what it may have written (the
  // activations; the weight too unless the caller declares it static).
  if (bulk && static_weight)
    for (int j = 0; j < first; ++j) issue(j);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (bulk && !static_weight)
    for (int j = 0; j < first; ++j) issue(j);

  // ---- the CTA's activation rows into shared memory ----
  // one 16-block: W4A16 scaled f16 and 2^-s, W4A4 the E2M1 values of its
  // NVFP4 codes (row scale s2) and its E4M3 scale
  auto store_block = [&](int i, const uint4& v0, const uint4& v1, float s2) {
    const int r = i / nb;
    const int b = i - r * nb;
    uint4 h0, h1;
    float f;
    if constexpr (A4) {
      float x[16];
      bf16x16_to_f32(v0, v1, x);
      const nvfp4::Block q = nvfp4::quant_block(x, s2);
      uint32_t w[8];
      e2m1x8_to_f16x2(q.lo, &w[0]);
      e2m1x8_to_f16x2(q.hi, &w[4]);
      h0 = make_uint4(w[0], w[1], w[2], w[3]);
      h1 = make_uint4(w[4], w[5], w[6], w[7]);
      f = e4m3_to_f32_hw(q.e4);
    } else {
      (void)s2;
      f = a16_block(v0, v1, h0, h1);
    }
    uint8_t* row_act = smem + L.act + (size_t)r * (size_t)k * 2;
    *reinterpret_cast<uint4*>(row_act + act_half((uint32_t)b, 0)) = h0;
    *reinterpret_cast<uint4*>(row_act + act_half((uint32_t)b, 1)) = h1;
    s_fac[i] = f;
  };
  auto load_block = [&](int i, uint4& v0, uint4& v1) {
    const int r = i / nb;
    const int b = i - r * nb;
    v0 = make_uint4(0, 0, 0, 0);
    v1 = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      const uint4* src = reinterpret_cast<const uint4*>(a + (size_t)(m0 + r) * (size_t)k + (size_t)b * 16);
      v0 = __ldg(src);
      v1 = __ldg(src + 1);
    }
  };
  if constexpr (A4) {
    if (MR * nb <= (int)blockDim.x) {
      // one block per thread, kept in registers across the row reduction
      // (row maxima by atomic max on the float bits, which order as
      // unsigned integers for non-negative values)
      const int i = threadIdx.x;
      const bool mine = i < MR * nb;
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
      if (mine) {
        load_block(i, v0, v1);
        const uint32_t bits = bf16x16_absmax_bits(v0, v1) << 16;
        if (bits) atomicMax(reinterpret_cast<unsigned int*>(s_amax) + i / nb, bits);
      }
      __syncthreads();
      if (threadIdx.x < MR) s_s2[threadIdx.x] = (int)threadIdx.x < rows ? nvfp4::row_scale2(s_amax[threadIdx.x]) : 0.0f;
      if (mine) store_block(i, v0, v1, i / nb < rows ? nvfp4::row_scale2(s_amax[i / nb]) : 0.0f);
    } else {
      // row maxima first (all threads), then the blocks
#pragma unroll
      for (int r = 0; r < MR; ++r) {
        float mx = 0.0f;
        if (r < rows) {
          const uint4* src = reinterpret_cast<const uint4*>(a + (size_t)(m0 + r) * (size_t)k);
          for (int i = threadIdx.x; i < nb; i += blockDim.x)
            mx = fmaxf(mx, bf16x16_amax_f32(__ldg(src + 2 * i), __ldg(src + 2 * i + 1)));
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        if (lane == 0) s_amax[r * nwarps + warp] = mx;
      }
      __syncthreads();
      if (threadIdx.x < MR) {
        const int r = threadIdx.x;
        float mx = 0.0f;
        for (int w = 0; w < nwarps; ++w) mx = fmaxf(mx, s_amax[r * nwarps + w]);
        s_s2[r] = r < rows ? nvfp4::row_scale2(mx) : 0.0f;
      }
      __syncthreads();
      for (int i = threadIdx.x; i < MR * nb; i += blockDim.x) {
        uint4 v0, v1;
        load_block(i, v0, v1);
        store_block(i, v0, v1, s_s2[i / nb]);
      }
    }
  } else {
    for (int i = threadIdx.x; i < MR * nb; i += blockDim.x) {
      uint4 v0, v1;
      load_block(i, v0, v1);
      store_block(i, v0, v1, 0.0f);
    }
  }
  __syncthreads();

  // ---- each warp reduces its stages ----
  // Per-lane 32-bit shared-memory offsets, advanced by 32 blocks per step:
  // activations 32 x 32 B (the other 16-byte half at offset ^ 16: rows of
  // 2K bytes and steps of 1 KB keep bit 4 clear), factors 32 x 4 B, codes
  // 32 x 8 B and scales 32 x 1 B of each row of the stage.
  const uint32_t act_lane = L.act + act_half((uint32_t)lane, 0);
  const uint32_t row_bytes = (uint32_t)k * 2u;
  bool aborted = false;
  int abort_j = 0;
  for (int j = 0; j < my_st; ++j) {
    const int row0 = r_begin + (warp + j * nwarps) * RS;
    const int nr = min(RS, r_end - row0);
    const uint32_t st = L.slots + (uint32_t)(warp * slots + j % slots) * L.stage_bytes;
    if (bulk) {
      const bool landed = mbar_wait(&bars[j % slots], (uint32_t)((j / slots) & 1), abort_flag, status,
                                    DEV_ERR_TIMEOUT_DECODE);
      if (__any_sync(0xFFFFFFFFu, !landed)) {
        aborted = true;
        abort_j = j;
        break;
      }
    } else {
      // row pitches not 16-byte multiples: the warp copies its stage itself
      for (int g = 0; g < nr; ++g) {
        const uint2* src = reinterpret_cast<const uint2*>(w_packed + (size_t)(row0 + g) * (size_t)kp);
        const uint8_t* src_e = w_e4m3 + (size_t)(row0 + g) * (size_t)nb;
        for (int b = lane; b < nb; b += 32) {
          *reinterpret_cast<uint2*>(smem + st + (uint32_t)g * (uint32_t)kp + 8u * (uint32_t)b) = __ldg(src + b);
          smem[st + L.codes_bytes + (uint32_t)(g * nb + b)] = __ldg(src_e + b);
        }
      }
      __syncwarp();
    }
    float acc[RS][MR];
#pragma unroll
    for (int g = 0; g < RS; ++g)
#pragma unroll
      for (int r = 0; r < MR; ++r) acc[g][r] = 0.0f;
    uint32_t o_act = act_lane, o_fac = L.fac + 4u * (uint32_t)lane;
    uint32_t o_w = st + 8u * (uint32_t)lane, o_e = st + L.codes_bytes + (uint32_t)lane;
    for (int b = lane; b < nb; b += 32, o_act += 1024u, o_fac += 128u, o_w += 256u, o_e += 32u) {
      uint4 ax[MR][2];
      float fa[MR];
#pragma unroll
      for (int r = 0; r < MR; ++r) {
        ax[r][0] = *reinterpret_cast<const uint4*>(smem + o_act + (uint32_t)r * row_bytes);
        ax[r][1] = *reinterpret_cast<const uint4*>(smem + ((o_act + (uint32_t)r * row_bytes) ^ 16u));
        fa[r] = *reinterpret_cast<const float*>(smem + o_fac + (uint32_t)(r * nb) * 4u);
      }
      // the stage's rows straight-line (their chains interleave); rows past
      // the CTA's range compute on what the slot holds and are never stored
#pragma unroll
      for (int g = 0; g < RS; ++g) {
        const uint2 qw = *reinterpret_cast<const uint2*>(smem + o_w + (uint32_t)g * (uint32_t)kp);
        const uint32_t e = smem[o_e + (uint32_t)(g * nb)];
        uint32_t w2[8];
        e2m1x8_to_f16x2(qw.x, &w2[0]);
        e2m1x8_to_f16x2(qw.y, &w2[4]);
        const float sw = e4m3_to_f32_hw(e);
#pragma unroll
        for (int r = 0; r < MR; ++r) {
          const uint32_t av[8] = {ax[r][0].x, ax[r][0].y, ax[r][0].z, ax[r][0].w,
                                  ax[r][1].x, ax[r][1].y, ax[r][1].z, ax[r][1].w};
          float p;
          if constexpr (A4) {
            uint32_t p2 = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) p2 = hfma2_u32(av[i], w2[i], p2);
            p = f16x2_sum_f32(p2);  // exact
          } else {
            p = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) p = fma2_f16_f32(av[i], w2[i], p);
          }
          acc[g][r] = __fmaf_rn(p, __fmul_rn(sw, fa[r]), acc[g][r]);
        }
      }
    }
    // every lane has read the slot: refill it (async proxy after generic reads)
    __syncwarp();
    if (bulk) {
      fence_proxy_async_smem();
      issue(j + slots);
    }
    constexpr int kPer = 32 / RS;  // lanes per row after the split
#pragma unroll
    for (int r = 0; r < MR; ++r) {
      float v[RS];
#pragma unroll
      for (int g = 0; g < RS; ++g) v[g] = acc[g][r];
      const float tot = lane_sum<RS>(v, lane);
      const int g = lane / kPer;
      if (lane % kPer == 0 && g < nr && r < rows) {
        const float y = A4 ? __fmul_rn(__fmul_rn(tot, s_s2[r]), scale2_w) : __fmul_rn(tot, scale2_w);
        out[(size_t)(m0 + r) * (size_t)n + (size_t)(row0 + g)] = __float2bfloat16_rn(y);
      }
    }
  }
  // A warp that gave up waiting may still have copies in flight (its stages
  // abort_j .. abort_j + slots - 1): wait for them once more, bounded, so
  // that the CTA does not exit under a bulk copy.
  if (aborted && lane == 0) {
    const unsigned long long t0 = globaltimer_ns();
    for (int j = abort_j; j < my_st && j < abort_j + slots; ++j)
      while (!mbar_try_wait(&bars[j % slots], (uint32_t)((j / slots) & 1)) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
  }
}

std::mutex g_gemv_optin_mu;

template <int MR, int RS, bool A4>
cudaError_t launch_t(const GemvPlan& p, const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3,
                     float scale2, uint16_t* out, int m, int n, int k, int static_weight, int* status,
                     cudaStream_t stream) {
  auto kern = nvfp4_gemv_kernel<MR, RS, A4>;
  static size_t granted[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lk(g_gemv_optin_mu);
    if (p.smem > granted[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
      if (e != cudaSuccess) return e;
      granted[dev] = p.smem;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.gx, (unsigned)p.gy);
  cfg.blockDim = dim3((unsigned)(p.warps * 32));
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a, w_packed, w_e4m3, scale2, reinterpret_cast<__nv_bfloat16*>(out), m, n, k,
                         p.rows_per_cta, p.slots, p.bulk ? 1 : 0, static_weight ? 1 : 0, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool A4>
cudaError_t launch_a(const GemvPlan& p, const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3,
                     float scale2, uint16_t* out, int m, int n, int k, int static_weight, int* status,
                     cudaStream_t stream) {
#define BSR_GEMV_CASE(MR_, RS_)                                                                                    \
  if (p.mr == MR_ && p.rs == RS_)                                                                                  \
    return launch_t<MR_, RS_, A4>(p, a, w_packed, w_e4m3, scale2, out, m, n, k, static_weight, status, stream);
  BSR_GEMV_CASE(1, 4)
  BSR_GEMV_CASE(1, 2)
  BSR_GEMV_CASE(1, 1)
  BSR_GEMV_CASE(2, 4)
  BSR_GEMV_CASE(2, 2)
  BSR_GEMV_CASE(2, 1)
  BSR_GEMV_CASE(4, 2)
  BSR_GEMV_CASE(4, 1)
  BSR_GEMV_CASE(8, 1)
  BSR_GEMV_CASE(16, 1)
#undef BSR_GEMV_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

bool nvfp4_gemv_plan(int m, int n, int k, bool a4, size_t smem_limit, size_t smem_per_sm, int num_sms,
                     GemvPlan& p) {
  if (m <= 0 || n <= 0 || k <= 0 || k % 16 != 0 || k > 65536 || num_sms <= 0) return false;
  const bool bulk = (k % 256) == 0;
  // activation rows per CTA: a power of two covering M (at most 16) whose
  // activations take at most half the shared memory
  int mr = 1;
  while (mr < m && mr < 16) mr <<= 1;
  auto act_bytes = [&](int r) { return (size_t)gemv_smem(k, r, 1, kGemvMaxWarps, 0, bulk).slots; };
  while (mr > 1 && act_bytes(mr) > smem_limit / 2) mr >>= 1;
  // rows per stage: 4 (2, 1) for short (longer) rows or more activation rows;
  // W4A4 takes half as many rows per warp (its CTA-wide quantiser prologue
  // runs faster on more warps)
  const int rs_k = k <= 8192 ? (a4 ? 2 : 4) : (k <= 16384 ? 2 : 1);
  const int rs_m = mr <= 2 ? 4 : (mr == 4 ? 2 : 1);
  const int rs = rs_k < rs_m ? rs_k : rs_m;
  const long long gy = ((long long)m + mr - 1) / mr;
  if (gy > 65535) return false;
  // rows per CTA: a multiple of the stage height, spread over the SMs
  long long gx_target = num_sms / gy;
  if (gx_target < 1) gx_target = 1;
  long long r = ((long long)n + gx_target - 1) / gx_target;
  r = (r + rs - 1) / rs * rs;
  const long long gx = ((long long)n + r - 1) / r;
  if (r > (1LL << 30) || gx > (1LL << 31) - 1) return false;
  const long long stages = r / rs;
  // warps and slots per warp: every stage in flight at once if it fits,
  // within half an SM's shared memory when possible (room for the next
  // launch's CTA), else the whole opt-in
  const int w = (int)(stages < kGemvMaxWarps ? stages : kGemvMaxWarps);
  const int slots_all = (int)((stages + w - 1) / w);
  auto total = [&](int ww, int s) { return (size_t)gemv_smem(k, mr, rs, ww, s, bulk).total; };
  auto fit = [&](size_t budget, int& ww, int& s) {
    ww = w;
    s = bulk ? slots_all : 1;
    while (s > 1 && total(ww, s) > budget) --s;
    while (ww > 1 && total(ww, s) > budget) --ww;
    return total(ww, s) <= budget;
  };
  const size_t half = smem_per_sm > 2048 ? smem_per_sm / 2 - 1024 : 0;
  int ww = 0, s = 0;
  const bool in_half = fit(half < smem_limit ? half : smem_limit, ww, s);
  // not all of the CTA's stages in flight within half an SM: take the whole
  // opt-in if that puts more stages in flight
  if (!in_half || ww < w || s < (bulk ? slots_all : 1)) {
    int w_full = 0, s_full = 0;
    if (fit(smem_limit, w_full, s_full) && (!in_half || w_full * s_full > ww * s)) {
      ww = w_full;
      s = s_full;
    } else if (!in_half) {
      return false;
    }
  }
  p.mr = mr;
  p.rs = rs;
  p.warps = ww;
  p.slots = s;
  p.rows_per_cta = (int)r;
  p.gx = (int)gx;
  p.gy = (int)gy;
  p.smem = total(ww, s);
  p.bulk = bulk;
  return true;
}

cudaError_t launch_nvfp4_gemv(const GemvPlan& p, bool a4, const uint16_t* a, const uint8_t* w_packed,
                              const uint8_t* w_e4m3, float scale2, uint16_t* out, int m, int n, int k,
                              int static_weight, int* status, cudaStream_t stream) {
  return a4 ? launch_a<true>(p, a, w_packed, w_e4m3, scale2, out, m, n, k, static_weight, status, stream)
            : launch_a<false>(p, a, w_packed, w_e4m3, scale2, out, m, n, k, static_weight, status, stream);
}

}  // namespace bsr
