// Block-scaled int8 GEMM on the sm_100a tensor cores (the `int8_gemm_faith2`
// step of gemm_dense_int8.rs, `int8_gemm_faith2_prefill`):
//
//   out[m, n] = bf16( sum_b  P[m, n, b] * a_scale[m, b] * w_scale[n, b] ),
//   P[m, n, b] = sum_{j<32} a_i8[m, 32b+j] * w_i8[n, 32b+j]   (exact int32)
//
// Tile: 128 weight rows (tensor-memory lanes, MMA M) x 128 activation rows
// (tensor-memory columns, MMA N).  Each 32-wide K block is ONE
// `tcgen05.mma.kind::i8` (128x128x32) into its own int32 tensor-memory
// buffer, because the scales change every 32 elements; a four-deep ring of
// such buffers lets the MMA of block b+1..b+3 run while the epilogue warps
// rescale block b into float32 register accumulators.
//
// Warp roles (384 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: per stage (4 K blocks = 128 bytes of K) the W
//               and A tiles (128x128 bytes, 128-byte swizzle) and their
//               scale tiles, into a 5-stage shared-memory ring.
//   warp 1      tensor-memory allocation and the MMA issuer (one thread).
//   warp 2      scale preparation: pre-multiplies the staged activation
//               scales by 2^49 and flags stages whose scales fall outside the
//               exponent window of the fast epilogue.
//   warps 4-11  epilogue: two warps per 32-lane quarter of tensor memory,
//               64 activation columns each.
//
// Epilogue arithmetic (per element and block, exact up to one rounding in
// each of two FMAs):
//   Tensor memory is preloaded with the integer 2^19 before every MMA, so the
//   accumulator holds P' = P + 2^19, which lies in [8160, 1040416] because
//   |P| <= 32*127*127 = 516128 < 2^19.  Read as a float32 bit pattern, P' is
//   the subnormal P' * 2^-149 exactly.  With W = w_scale * 2^100 and
//   c = -W * 2^-130 (both exact),
//       u = fma(P'*2^-149, W, c) = RN(P * w_scale * 2^-49)      (one rounding)
//       acc = fma(u, a_scale * 2^49, acc)
//   which is acc + RN(P * w_scale) * a_scale rounded once -- the same value
//   the decode path computes with an explicit int->float conversion.  It
//   needs W in [2^23, 2^128) and a_scale * 2^49 finite, i.e. nonzero
//   |w_scale| in [2^-77, 2^28) and a_scale < 2^79; a stage with any scale
//   outside that window (or NaN) takes the plain path (convert, multiply,
//   fma) for all its blocks.  Two FMAs per element run as packed f32x2 FMAs.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace bsr {

namespace gemm {

constexpr int BN = 128;           // weight rows per tile (MMA M, TMEM lanes)
constexpr int BM = 128;           // activation rows per tile (MMA N, TMEM columns)
constexpr int KBS = 4;            // 32-blocks per stage
constexpr int KS = 32 * KBS;      // bytes of K per stage
constexpr int STAGES = 5;
constexpr int TBUF = 4;           // tensor-memory ring depth (x BM columns)
constexpr int TMEM_COLS = TBUF * BM;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 384;
constexpr int EPI_WARP0 = 4;
// Register split: launched with 384 x 168 = 64512 registers; the control
// warpgroup (warps 0-3) drops to 40 and the two epilogue warpgroups rise to
// 224: 128 x 40 + 256 x 224 = 62464 <= 64512.
constexpr int CTRL_REGS = 56;
constexpr int EPI_REGS = 216;
static_assert(128 * CTRL_REGS + 256 * EPI_REGS <= THREADS * 168, "register split exceeds the launch allocation");

constexpr int W_TILE = BN * KS;             // 16384
constexpr int A_TILE = BM * KS;             // 16384
constexpr int WS_TILE = BN * KBS * 4;       // 2048
constexpr int AS_TILE = BM * KBS * 4;       // 2048
constexpr int STAGE_BYTES = W_TILE + A_TILE + WS_TILE + AS_TILE;  // 36864
constexpr int OFF_A = W_TILE;
constexpr int OFF_WS = W_TILE + A_TILE;
constexpr int OFF_AS = OFF_WS + WS_TILE;

constexpr uint32_t kBias = 1u << 19;
constexpr uint32_t kIdesc = idesc_i8(BN, BM);

struct Ctrl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t prep[STAGES];
  uint64_t tfull[TBUF];
  uint64_t tempty[TBUF];
  int exotic[STAGES];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Ctrl);

__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) { return make_float2(__uint_as_float(a), __uint_as_float(b)); }

template <bool DUMP>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
                const __grid_constant__ CUtensorMap tm_ws, const __grid_constant__ CUtensorMap tm_as,
                __nv_bfloat16* __restrict__ out, int32_t* __restrict__ partials, int* __restrict__ status, int m,
                int n, int k, int n_tiles, int m_tiles, int m_fastest) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + (size_t)STAGES * STAGE_BYTES);
  volatile int* abort_flag = &ctrl->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = n_tiles * m_tiles;
  const int kstages = k / KS;
  const int nb = k / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1 + EPI_WARPS);
      mbar_init(&ctrl->prep[s], 1);
      ctrl->exotic[s] = 0;
    }
    for (int b = 0; b < TBUF; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], EPI_WARPS);
    }
    ctrl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_ws);
    tma_prefetch_desc(&tm_as);
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctrl->tmem_base;

  auto tile_coords = [&](int tile, int& n0, int& m0) {
    int tn, tm;
    if (m_fastest) {
      tn = tile / m_tiles;
      tm = tile - tn * m_tiles;
    } else {
      tm = tile / n_tiles;
      tn = tile - tm * n_tiles;
    }
    n0 = tn * BN;
    m0 = tm * BM;
  };

  if (warp < EPI_WARP0) {
    setmaxnreg_dec<CTRL_REGS>();
    if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        int n0, m0;
        tile_coords(tile, n0, m0);
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t r = it / STAGES;
          if (!mbar_wait(&ctrl->empty[s], (r & 1) ^ 1, abort_flag, status, DEV_ERR_TIMEOUT_TMA)) goto tma_done;
          uint8_t* st = smem + (size_t)s * STAGE_BYTES;
          mbar_arrive_expect_tx(&ctrl->full[s], STAGE_BYTES);
          tma_load_2d(st, &tm_w, &ctrl->full[s], ks * KS, n0);
          tma_load_2d(st + OFF_A, &tm_a, &ctrl->full[s], ks * KS, m0);
          tma_load_2d(st + OFF_WS, &tm_ws, &ctrl->full[s], ks * KBS, n0);
          tma_load_2d(st + OFF_AS, &tm_as, &ctrl->full[s], m0, ks * KBS);
        }
      }
    tma_done:;
    }
    } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t it = 0, g = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t r = it / STAGES;
          if (!mbar_wait(&ctrl->full[s], r & 1, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + (size_t)s * STAGE_BYTES);
          const uint32_t b_base = a_base + OFF_A;
#pragma unroll
          for (int kb = 0; kb < KBS; ++kb, ++g) {
            const int buf = g % TBUF;
            if (!mbar_wait(&ctrl->tempty[buf], (g / TBUF) & 1, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
            tc_fence_after();
            mma_i8(tmem_base + buf * BM, smem_desc_k_sw128(a_base + kb * 32), smem_desc_k_sw128(b_base + kb * 32),
                   kIdesc, 1u);
            tc_commit(&ctrl->tfull[buf]);
          }
          tc_commit(&ctrl->empty[s]);
        }
      }
    mma_done:;
    }
    } else if (warp == 2) {
    // ---------------------------------------------------------------- scale prep
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      for (int ks = 0; ks < kstages; ++ks, ++it) {
        const int s = it % STAGES;
        const uint32_t r = it / STAGES;
        if (!mbar_wait(&ctrl->full[s], r & 1, abort_flag, status, DEV_ERR_TIMEOUT_PREP)) goto prep_done;
        uint8_t* st = smem + (size_t)s * STAGE_BYTES;
        float4* as4 = reinterpret_cast<float4*>(st + OFF_AS);
        const float4* ws4 = reinterpret_cast<const float4*>(st + OFF_WS);
        float4 av[4];
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          av[j] = as4[j * 32 + lane];
          bad |= !(av[j].x < 0x1p79f) | !(av[j].y < 0x1p79f) | !(av[j].z < 0x1p79f) | !(av[j].w < 0x1p79f);
          const float4 w = ws4[j * 32 + lane];
          const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float aw = fabsf(wv[t]);
            bad |= !((aw == 0.0f) | ((aw >= 0x1p-77f) & (aw < 0x1p28f)));
          }
        }
        const bool exotic = __any_sync(0xFFFFFFFFu, bad);
        if (!exotic) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float4 v = av[j];
            v.x *= 0x1p49f;
            v.y *= 0x1p49f;
            v.z *= 0x1p49f;
            v.w *= 0x1p49f;
            as4[j * 32 + lane] = v;
          }
        }
        if (lane == 0) ctrl->exotic[s] = exotic ? 1 : 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->prep[s]);
      }
    }
    prep_done:;
    }
  } else {
    setmaxnreg_inc<EPI_REGS>();
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                    // tensor-memory lane quarter
    const int hc = (warp - EPI_WARP0) >> 2;    // column half: 0 or 1
    const int n_local = q * 32 + lane;
    const uint32_t t_lane = (uint32_t)(q * 32) << 16;
    const uint32_t col0 = (uint32_t)(hc * 64);

    // preload the bias into every buffer slice this warp owns
#pragma unroll
    for (int b = 0; b < TBUF; ++b) tmem_st_x64_const(tmem_base + t_lane + b * BM + col0, kBias);
    tc_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int b = 0; b < TBUF; ++b) mbar_arrive(&ctrl->tempty[b]);

    uint32_t it = 0, g = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int n0, m0;
      tile_coords(tile, n0, m0);
      float2 acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = make_float2(0.0f, 0.0f);

      for (int ks = 0; ks < kstages; ++ks, ++it) {
        const int s = it % STAGES;
        const uint32_t r = it / STAGES;
        if (!mbar_wait(&ctrl->prep[s], r & 1, abort_flag, status, DEV_ERR_TIMEOUT_EPI)) goto epi_done;
        const uint8_t* st = smem + (size_t)s * STAGE_BYTES;
        const float* ws_row = reinterpret_cast<const float*>(st + OFF_WS) + n_local * KBS;
        const int exotic = ctrl->exotic[s];
        const float* as_stage = reinterpret_cast<const float*>(st + OFF_AS);
#pragma unroll 1
        for (int kb = 0; kb < KBS; ++kb, ++g) {
          const int buf = g % TBUF;
          if (!mbar_wait(&ctrl->tfull[buf], (g / TBUF) & 1, abort_flag, status, DEV_ERR_TIMEOUT_EPI)) goto epi_done;
          tc_fence_after();
          const uint32_t taddr = tmem_base + t_lane + buf * BM + col0;
          uint32_t p[64];
          tmem_ld_x64(taddr, p);
          tmem_st_x64_const(taddr, kBias);
          tc_wait_ld();
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctrl->tempty[buf]);

          const float* arow = as_stage + kb * BM + col0;
          const float wsb = ws_row[kb];
          if (!exotic) {
            const float W = wsb * 0x1p100f;
            const float c = -(W * 0x1p-130f);
            const float2 W2 = make_float2(W, W);
            const float2 c2 = make_float2(c, c);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float4 a4 = reinterpret_cast<const float4*>(arow)[j];
              const float2 u0 = __ffma2_rn(f2(p[4 * j], p[4 * j + 1]), W2, c2);
              const float2 u1 = __ffma2_rn(f2(p[4 * j + 2], p[4 * j + 3]), W2, c2);
              acc[2 * j] = __ffma2_rn(u0, make_float2(a4.x, a4.y), acc[2 * j]);
              acc[2 * j + 1] = __ffma2_rn(u1, make_float2(a4.z, a4.w), acc[2 * j + 1]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float4 a4 = reinterpret_cast<const float4*>(arow)[j];
              const float u0 = __fmul_rn(__int2float_rn((int)p[4 * j] - (int)kBias), wsb);
              const float u1 = __fmul_rn(__int2float_rn((int)p[4 * j + 1] - (int)kBias), wsb);
              const float u2 = __fmul_rn(__int2float_rn((int)p[4 * j + 2] - (int)kBias), wsb);
              const float u3 = __fmul_rn(__int2float_rn((int)p[4 * j + 3] - (int)kBias), wsb);
              acc[2 * j].x = __fmaf_rn(u0, a4.x, acc[2 * j].x);
              acc[2 * j].y = __fmaf_rn(u1, a4.y, acc[2 * j].y);
              acc[2 * j + 1].x = __fmaf_rn(u2, a4.z, acc[2 * j + 1].x);
              acc[2 * j + 1].y = __fmaf_rn(u3, a4.w, acc[2 * j + 1].y);
            }
          }
          if constexpr (DUMP) {
            const int nn = n0 + n_local;
            const int b = ks * KBS + kb;
            if (nn < n) {
#pragma unroll
              for (int c = 0; c < 64; ++c) {
                const int mm = m0 + (int)col0 + c;
                if (mm < m) partials[((size_t)mm * n + nn) * nb + b] = (int)p[c] - (int)kBias;
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->empty[s]);
      }
      // tile end: write BF16; a warp's 32 lanes write 64 contiguous bytes per row
      {
        const int nn = n0 + n_local;
        if (nn < n) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int mm = m0 + (int)col0 + 2 * j;
            if (mm < m) out[(size_t)mm * n + nn] = __float2bfloat16_rn(acc[j].x);
            if (mm + 1 < m) out[(size_t)(mm + 1) * n + nn] = __float2bfloat16_rn(acc[j].y);
          }
        }
      }
    }
  epi_done:;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace gemm

size_t gemm_smem_bytes() { return gemm::SMEM_BYTES; }

cudaError_t launch_gemm(const GemmMaps& maps, uint16_t* out, int32_t* partials, int* status, int m, int n, int k,
                        cudaStream_t stream, int num_sms) {
  using namespace gemm;
  const int n_tiles = (n + BN - 1) / BN;
  const int m_tiles = (m + BM - 1) / BM;
  const int tiles = n_tiles * m_tiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  // Sweep the smaller operand fastest so that it stays resident in L2 while
  // the larger one streams through once.
  const int m_fastest = ((long long)m <= (long long)n) ? 1 : 0;
  cudaError_t e;
  if (partials) {
    e = cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    gemm_kernel<true><<<grid, THREADS, SMEM_BYTES, stream>>>(maps.w, maps.a, maps.ws, maps.as,
                                                             reinterpret_cast<__nv_bfloat16*>(out), partials,
                                                             status, m, n, k, n_tiles, m_tiles, m_fastest);
  } else {
    e = cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    gemm_kernel<false><<<grid, THREADS, SMEM_BYTES, stream>>>(maps.w, maps.a, maps.ws, maps.as,
                                                              reinterpret_cast<__nv_bfloat16*>(out), nullptr,
                                                              status, m, n, k, n_tiles, m_tiles, m_fastest);
  }
  return cudaGetLastError();
}

}  // namespace bsr
