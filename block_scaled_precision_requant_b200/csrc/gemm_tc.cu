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
// Warp roles (640 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: per stage (4 K blocks = 128 bytes of K) the W
//               and A tiles (128x128 bytes, 128-byte swizzle) and their
//               scale tiles, into a 5-stage shared-memory ring.
//   warps 1, 3  MMA issuers (one thread each; K blocks 0,2 and 1,3 of a
//               stage); warp 1 also allocates the tensor memory.
//   warp 2      scale preparation: pre-multiplies the staged activation
//               scales by 2^49 and the weight scales by 2^100, or flags the
//               stage when a scale falls outside the exponent window of the
//               fast epilogue (the stage then keeps its scales as loaded).
//   warps 4-19  epilogue: four warps per 32-lane quarter of tensor memory,
//               32 activation columns each, read with 16x128b loads (4
//               weight rows x 8 activation columns per thread).
//
// Epilogue arithmetic (per element and block, exact up to one rounding in
// each of two FMAs):
//   Every K block is two MMAs into the same buffer: first a u8 x u8 MMA of
//   two constant tiles of 128s with accumulation off (32*128*128 = 2^19),
//   then the s8 x s8 MMA of the data with accumulation on, so the
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

#include <type_traits>

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
constexpr int EPI_WARPS = 16;
constexpr int THREADS = 640;
constexpr int EPI_WARP0 = 4;
// Register split: launched with 640 x 96 = 61440 registers (the most that
// 640 threads can hold); the control warpgroup (warps 0-3) drops to 64 and
// the four epilogue warpgroups rise to 104: 128 x 64 + 512 x 104 = 61440.
constexpr int LAUNCH_REGS = 96;
constexpr int CTRL_REGS = 64;
constexpr int EPI_REGS = 104;
static_assert(THREADS * LAUNCH_REGS <= 65536, "launch register budget");
static_assert(128 * CTRL_REGS + (THREADS - 128) * EPI_REGS <= THREADS * LAUNCH_REGS,
              "register split exceeds the launch allocation");

constexpr int W_TILE = BN * KS;             // 16384
constexpr int A_TILE = BM * KS;             // 16384
constexpr int WS_TILE = BN * KBS * 4;       // 2048
constexpr int AS_TILE = BM * KBS * 4;       // 2048
constexpr int STAGE_BYTES = W_TILE + A_TILE + WS_TILE + AS_TILE;  // 36864
constexpr int OFF_A = W_TILE;
constexpr int OFF_WS = W_TILE + A_TILE;
constexpr int OFF_AS = OFF_WS + WS_TILE;

constexpr uint32_t kBias = 1u << 19;  // = 32 * 128 * 128
constexpr uint32_t kIdesc = idesc_i8(BN, BM);
// u8 x u8 variant of the same shape, for the bias MMA
constexpr uint32_t kIdescBias = kIdesc & ~((7u << 7) | (7u << 10));
constexpr int CONST_TILE = BN * KS;  // 16 KB of 0x80 bytes: the bias MMA's operands
static_assert(TBUF == KBS, "tensor-memory buffer index equals the K block index within a stage");

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

constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + CONST_TILE + sizeof(Ctrl);

__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) { return make_float2(__uint_as_float(a), __uint_as_float(b)); }

template <bool DUMP>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
                const __grid_constant__ CUtensorMap tm_ws, const __grid_constant__ CUtensorMap tm_as,
                __nv_bfloat16* __restrict__ out, int32_t* __restrict__ partials, int* __restrict__ status, int m,
                int n, int k, int n_tiles, int m_tiles, int m_fastest, long long ldo) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles, keeping the pointer
  // derived from the shared array so accesses stay shared-space loads
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* const_tile = smem + (size_t)STAGES * STAGE_BYTES;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(const_tile + CONST_TILE);
  volatile int* abort_flag = &ctrl->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = n_tiles * m_tiles;
  const int kstages = k / KS;
  const int nb = k / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 2 + EPI_WARPS);  // two MMA commits + the epilogue warps
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
  for (int i = threadIdx.x; i < CONST_TILE / 16; i += THREADS)
    reinterpret_cast<uint4*>(const_tile)[i] = make_uint4(0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u);
  fence_proxy_async_smem();
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
    } else if (warp == 1 || warp == 3) {
    // ---------------------------------------------------------------- MMA
    // Two issuing threads: warp 1 takes K blocks 0 and 2 of every stage,
    // warp 3 blocks 1 and 3 (= tensor-memory buffers), so the per-block issue
    // cost (two MMAs and a commit) is paid on two warps.
    if (lane == 0) {
      const uint64_t c_desc = smem_desc_k_sw128(smem_u32(const_tile));
      const int kb0 = (warp == 1) ? 0 : 1;
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = it % STAGES;
          const uint32_t r = it / STAGES;
          if (!mbar_wait(&ctrl->full[s], r & 1, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + (size_t)s * STAGE_BYTES);
          const uint32_t b_base = a_base + OFF_A;
#pragma unroll
          for (int kb = kb0; kb < KBS; kb += 2) {
            if (!mbar_wait(&ctrl->tempty[kb], it & 1, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
            tc_fence_after();
            // D = 2^19 (constant u8 tiles of 128s, accumulate off), then D += A x B
            mma_i8(tmem_base + kb * BM, c_desc, c_desc, kIdescBias, 0u);
            mma_i8(tmem_base + kb * BM, smem_desc_k_sw128(a_base + kb * 32), smem_desc_k_sw128(b_base + kb * 32),
                   kIdesc, 1u);
            tc_commit(&ctrl->tfull[kb]);
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
        float4* ws4 = reinterpret_cast<float4*>(st + OFF_WS);
        float4 av[4], wv[4];
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          av[j] = as4[j * 32 + lane];
          bad |= !(av[j].x < 0x1p79f) | !(av[j].y < 0x1p79f) | !(av[j].z < 0x1p79f) | !(av[j].w < 0x1p79f);
          wv[j] = ws4[j * 32 + lane];
          const float w4[4] = {wv[j].x, wv[j].y, wv[j].z, wv[j].w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float aw = fabsf(w4[t]);
            bad |= !((aw == 0.0f) | ((aw >= 0x1p-77f) & (aw < 0x1p28f)));
          }
        }
        const bool exotic = __any_sync(0xFFFFFFFFu, bad);
        // a_scale * 2^49 and W = w_scale * 2^100 (exact inside the window;
        // an exotic stage keeps the scales as loaded)
        const float fa = exotic ? 1.0f : 0x1p49f;
        const float fw = exotic ? 1.0f : 0x1p100f;
        __syncwarp();
        // Rewrite both scale tiles in the order the epilogue reads them.
        // Activation scales [kb][m], m = 32h + r + 4k  ->  [kb][h][r][k]:
        // lane L holds m = 4L..4L+3 of every kb (h = L/8, k = L%8, r = e).
        // Weight scales [n][kb], n = 32q + l + 8i  ->  [kb][q][l][i]: lane L
        // holds row n = 32j + L (q = j, l = L%8, i = L/8) for all four kb.
        float* asf = reinterpret_cast<float*>(st + OFF_AS);
        float* wsf = reinterpret_cast<float*>(st + OFF_WS);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a4[4] = {av[j].x, av[j].y, av[j].z, av[j].w};
          const float w4[4] = {wv[j].x, wv[j].y, wv[j].z, wv[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            asf[j * BM + (lane >> 3) * 32 + e * 8 + (lane & 7)] = a4[e] * fa;
            wsf[e * BN + j * 32 + (lane & 7) * 4 + (lane >> 3)] = w4[e] * fw;
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
    // Warp (quarter q, column slice h) owns tensor-memory lanes 32q..32q+31
    // (weight rows) and columns 32h..32h+31 (activation rows), read per block
    // with two 16x128b.x8 loads (lanes 32q..+15 and 32q+16..+31): thread t
    // holds weight rows 32q + t/4 + 8i (i = 0..3) and activation columns
    // 32h + t%4 + 4k (k = 0..7).  Registers r[2k], r[2k+1] of one load are
    // rows (t/4, t/4 + 8) at the same column: the operand pair of one packed
    // FMA.  Per block a thread needs 4 weight scales (one 16-byte load) and
    // 8 activation scales (two), from the tiles the prep warp rewrote.
    // A warp hands its buffer back as soon as its loads have landed and then
    // rescales from registers; four warps per scheduler hide each other's
    // load latency.
    const int q = warp & 3;
    const int h = (warp - EPI_WARP0) >> 2;
    const int l8 = lane >> 2;
    const int c4 = lane & 3;
    const uint32_t tl = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 32);
    const int my_tiles = (num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t ws_off = OFF_WS + (uint32_t)(q * 32 + l8 * 4) * 4u;  // + kb*BN*4
    const uint32_t as_off = OFF_AS + (uint32_t)(h * 32 + c4 * 8) * 4u;  // + kb*BM*4

    // open the tensor-memory ring
    mbar_arrive_lane0(&ctrl->tempty[0], lane);
    mbar_arrive_lane0(&ctrl->tempty[1], lane);
    mbar_arrive_lane0(&ctrl->tempty[2], lane);
    mbar_arrive_lane0(&ctrl->tempty[3], lane);

    float2 acc[2][8];  // acc[j][k] = rows (2j, 2j+1) of this thread's four, column k
    uint32_t r0[16], r1[16];

    auto dump = [&](int n0, int m0, int b) {
      if constexpr (DUMP) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int nn = n0 + q * 32 + l8 + 8 * i;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int mm = m0 + h * 32 + c4 + 4 * k;
            const uint32_t v = (i < 2) ? r0[2 * k + (i & 1)] : r1[2 * k + (i & 1)];
            if (nn < n && mm < m) partials[((size_t)mm * n + nn) * nb + b] = (int)v - (int)kBias;
          }
        }
      }
    };

    // Stage sequence of this CTA: stage counter itg (tiles x K stages), ring
    // slot itg % STAGES; within a stage the four K blocks are unrolled, block
    // kb in tensor-memory buffer kb (phase itg & 1).
    const int total_st = my_tiles * kstages;
    int tile = blockIdx.x, n0 = 0, m0 = 0, kst = 0;
    tile_coords(tile, n0, m0);
    uint32_t st_addr = smem_base;
    uint32_t itg = 0;

    // One K block: scales, partials, buffer release, rescale.  The choice of
    // the exotic path is a template parameter, so a stage runs one of two
    // fully unrolled code paths with no branch inside.
    auto sub = [&](auto kbc, auto exc) -> bool {
      constexpr int kb = decltype(kbc)::value;
      constexpr bool EXO = decltype(exc)::value;
      const float4 W4 = lds_f32x4(st_addr + ws_off + (uint32_t)kb * (BN * 4u));
      const float4 A0 = lds_f32x4(st_addr + as_off + (uint32_t)kb * (BM * 4u));
      const float4 A1 = lds_f32x4(st_addr + as_off + (uint32_t)kb * (BM * 4u) + 16u);
      if (!mbar_wait(&ctrl->tfull[kb], itg & 1u, abort_flag, status, DEV_ERR_TIMEOUT_EPI)) return false;
      tc_fence_after();
      tmem_ld_16x128b_x8(tl + kb * BM, r0);
      tmem_ld_16x128b_x8(tl + kb * BM + (16u << 16), r1);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive_lane0(&ctrl->tempty[kb], lane);
      const float av[8] = {A0.x, A0.y, A0.z, A0.w, A1.x, A1.y, A1.z, A1.w};
      const float2 Wp[2] = {make_float2(W4.x, W4.y), make_float2(W4.z, W4.w)};
      if constexpr (!EXO) {
        const float2 Cp[2] = {make_float2(-(W4.x * 0x1p-130f), -(W4.y * 0x1p-130f)),
                              make_float2(-(W4.z * 0x1p-130f), -(W4.w * 0x1p-130f))};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float2 u0 = __ffma2_rn(f2(r0[2 * k], r0[2 * k + 1]), Wp[0], Cp[0]);
          const float2 u1 = __ffma2_rn(f2(r1[2 * k], r1[2 * k + 1]), Wp[1], Cp[1]);
          acc[0][k] = __ffma2_rn(u0, make_float2(av[k], av[k]), acc[0][k]);
          acc[1][k] = __ffma2_rn(u1, make_float2(av[k], av[k]), acc[1][k]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t* rr = j ? r1 : r0;
            const float ux = __fmul_rn(__int2float_rn((int)rr[2 * k] - (int)kBias), j ? W4.z : W4.x);
            const float uy = __fmul_rn(__int2float_rn((int)rr[2 * k + 1] - (int)kBias), j ? W4.w : W4.y);
            acc[j][k].x = __fmaf_rn(ux, av[k], acc[j][k].x);
            acc[j][k].y = __fmaf_rn(uy, av[k], acc[j][k].y);
          }
        }
      }
      dump(n0, m0, kst * KBS + kb);
      if (kb == KBS - 1) {
        mbar_arrive_lane0(&ctrl->empty[(int)(itg % STAGES)], lane);
        if (++kst == kstages) {
          // tile end: write BF16 out[m][n]; the tile origin passes through a
          // volatile move so the store addresses are formed here only
          int nr, mr;
          asm volatile("mov.b32 %0, %1;" : "=r"(nr) : "r"(n0 + q * 32 + l8));
          asm volatile("mov.b32 %0, %1;" : "=r"(mr) : "r"(m0 + h * 32 + c4));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int nn = nr + 8 * i;
            if (nn < n) {
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int mm = mr + 4 * k;
                const float v = (i & 1) ? acc[i >> 1][k].y : acc[i >> 1][k].x;
                if (mm < m) out[(size_t)mm * (size_t)ldo + nn] = __float2bfloat16_rn(v);
              }
            }
          }
          kst = 0;
          tile += gridDim.x;
          tile_coords(tile, n0, m0);
        }
      }
      return true;
    };

    bool ok = true;
    for (; ok && itg < (uint32_t)total_st; ++itg) {
      const int s = (int)(itg % STAGES);
      if (!mbar_wait(&ctrl->prep[s], (itg / STAGES) & 1u, abort_flag, status, DEV_ERR_TIMEOUT_EPI)) break;
      st_addr = smem_base + (uint32_t)s * STAGE_BYTES;
      const int exotic = ctrl->exotic[s];
      if (kst == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[j][k] = make_float2(0.0f, 0.0f);
      }
      using K0 = std::integral_constant<int, 0>;
      using K1 = std::integral_constant<int, 1>;
      using K2 = std::integral_constant<int, 2>;
      using K3 = std::integral_constant<int, 3>;
      if (!exotic) {
        const std::false_type fast;
        ok = sub(K0{}, fast) && sub(K1{}, fast) && sub(K2{}, fast) && sub(K3{}, fast);
      } else {
        const std::true_type slow;
        ok = sub(K0{}, slow) && sub(K1{}, slow) && sub(K2{}, slow) && sub(K3{}, slow);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace gemm

size_t gemm_smem_bytes() { return gemm::SMEM_BYTES; }

cudaError_t launch_gemm(const GemmMaps& maps, uint16_t* out, int32_t* partials, int* status, int m, int n, int k,
                        long long ldo, cudaStream_t stream, int num_sms, int max_ctas) {
  using namespace gemm;
  const int n_tiles = (n + BN - 1) / BN;
  const int m_tiles = (m + BM - 1) / BM;
  const int tiles = n_tiles * m_tiles;
  // persistent CTAs: one per SM, or fewer when the caller shares the GPU
  // between concurrent launches (max_ctas)
  const int cap = (max_ctas > 0 && max_ctas < num_sms) ? max_ctas : num_sms;
  const int grid = tiles < cap ? tiles : cap;
  // Sweep the smaller operand fastest so that it stays resident in L2 while
  // the larger one streams through once.
  const int m_fastest = ((long long)m <= (long long)n) ? 1 : 0;
  // the shared-memory opt-in is set once per device and kernel variant
  static bool granted[64][2] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (partials) {
    if (!granted[dev][1]) {
      e = cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
      if (e != cudaSuccess) return e;
      granted[dev][1] = true;
    }
    gemm_kernel<true><<<grid, THREADS, SMEM_BYTES, stream>>>(maps.w, maps.a, maps.ws, maps.as,
                                                             reinterpret_cast<__nv_bfloat16*>(out), partials,
                                                             status, m, n, k, n_tiles, m_tiles, m_fastest, ldo);
  } else {
    if (!granted[dev][0]) {
      e = cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
      if (e != cudaSuccess) return e;
      granted[dev][0] = true;
    }
    gemm_kernel<false><<<grid, THREADS, SMEM_BYTES, stream>>>(maps.w, maps.a, maps.ws, maps.as,
                                                              reinterpret_cast<__nv_bfloat16*>(out), nullptr,
                                                              status, m, n, k, n_tiles, m_tiles, m_fastest, ldo);
  }
  return cudaGetLastError();
}

}  // namespace bsr
