// Block-scaled int8 GEMM on the sm_100a tensor cores (the `int8_gemm_faith2`
// step of gemm_dense_int8.rs, `int8_gemm_faith2_prefill`):
//
//   out[m, n] = bf16( sum_b  P[m, n, b] * a_scale[m, b] * w_scale[n, b] ),
//   P[m, n, b] = sum_{j<32} a_i8[m, 32b+j] * w_i8[n, 32b+j]   (exact int32)
//
// Tile: 128 weight rows (tensor-memory lanes, MMA M) x BM activation rows
// (tensor-memory columns, MMA N), BM in {128, 192, 256}: 128 when M <= 128,
// else the width whose whole waves of tiles take the least estimated time.  Each
// 32-wide K block is ONE `tcgen05.mma.kind::i8` (128 x BM x 32) into its own
// int32 tensor-memory buffer, because the scales change every 32 elements;
// a ring of 512 / BM such buffers lets the MMA of the next block run while
// the epilogue warps rescale this one into float32 register accumulators.
//
// The rescale is two FP32 FMAs per element and block on the CUDA cores, so
// the kernel is bound by the FP32 pipe, not by the tensor pipe.  What decides
// how close it gets to that bound is the instruction overhead per block
// (barrier waits, tensor-memory loads, scale loads) against the FMAs it
// feeds: each epilogue thread owns 4 weight rows x BM/8 activation columns,
// so one wait, one buffer release and one weight-scale load serve BM/2 FMA
// pairs.
//
// Warp roles (384 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: per stage (4 K blocks = 128 bytes of K) the W
//               and A tiles (128-byte swizzle) and their scale tiles, into a
//               multi-stage shared-memory ring.
//   warp 1      MMA issuer (one thread); also owns the tensor memory.
//   warp 2      scale preparation: pre-multiplies the staged activation
//               scales by 2^49 and the weight scales by 2^100 and rewrites
//               both tiles into the epilogue's read order, or flags the stage
//               when a scale falls outside the exponent window of the fast
//               epilogue (the stage then keeps its scales as loaded).
//   warp 3      idle.
//   warps 4-11  epilogue: warp w reads tensor-memory lanes 32(w%4).. (the
//               quarter it may access) and the half (w-4)/4 of the columns,
//               in chunks of 16 columns with 16x128b loads, the next chunk's
//               load in flight while the current one is rescaled: a thread
//               holds weight rows 32q + t/4 + 8i (i = 0..3) x columns
//               c + t%4 + 4k.
//
// Epilogue arithmetic (per element and block, exact up to one rounding in
// each of two FMAs):
//   Every K block is two MMAs into the same buffer: first a u8 x u8 MMA of
//   two constant operands of 128s with accumulation off (32*128*128 = 2^19),
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
//   fma) for all its blocks.  Registers (l, l+8) of a 16x128b load are two
//   weight rows at one column: the operand pair of one packed f32x2 FMA.
//
// Failure handling: every wait is bounded.  A wait that runs out raises the
// CTA's abort flag and a bit in the status word; the TMA thread then waits
// (bounded) for the copies it issued, the MMA thread commits and waits for
// its issued MMAs, and only then does the CTA free its tensor memory.
#include <cuda_bf16.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace bsr {

namespace gemm {

constexpr int BN = 128;          // weight rows per tile (MMA M, TMEM lanes)
constexpr int KBS = 4;           // 32-blocks per stage
constexpr int KS = 32 * KBS;     // bytes of K per stage (one 128-byte swizzle row)
constexpr int EPI_WARP0 = 4;
constexpr uint32_t TMEM_COLS = 512;
// Constant operand of the bias MMA: 8 KB of 0x80 bytes read through an
// unswizzled K-major descriptor (core matrices 8 rows x 16 bytes; 128 bytes
// to the next one along K, 256 bytes to the next 8 rows: 256 rows x 32 bytes
// of K span exactly 8 KB).
constexpr int CONST_BYTES = 8192;
constexpr uint32_t kBias = 1u << 19;  // = 32 * 128 * 128
constexpr size_t kSmemPerCta = 232448;  // 227 KB opt-in limit of sm_100

// Epilogue shape: EW epilogue warps (8 or 12: two or three per scheduler)
// and CW-column tensor-memory chunks (16 or 32).  Register split: the CTA is
// launched with THREADS x LAUNCH_REGS registers; the control warpgroup
// (warps 0-3) drops to CTRL_REGS and the epilogue warpgroups rise to EPI_REGS.
template <int EW>
struct Warps {
  static constexpr int EPI_WARPS = EW;
  static constexpr int THREADS = 32 * (EPI_WARP0 + EW);
  static constexpr int LAUNCH_REGS = EW == 8 ? 168 : 128;
  static constexpr int CTRL_REGS = EW == 8 ? 56 : 32;
  static constexpr int EPI_REGS = EW == 8 ? 224 : 160;
  static_assert(EW == 8 || EW == 12, "two or three epilogue warps per scheduler");
  static_assert(THREADS * LAUNCH_REGS <= 65536, "launch register budget");
  static_assert(128 * CTRL_REGS + 32 * EW * EPI_REGS <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch allocation");
};

template <int BM>
struct Tile {
  static constexpr int W_TILE = BN * KS;
  static constexpr int A_TILE = BM * KS;
  static constexpr int WS_TILE = BN * KBS * 4;
  static constexpr int AS_TILE = BM * KBS * 4;
  static constexpr int STAGE_BYTES = W_TILE + A_TILE + WS_TILE + AS_TILE;
  static constexpr int OFF_A = W_TILE;
  static constexpr int OFF_WS = W_TILE + A_TILE;
  static constexpr int OFF_AS = OFF_WS + WS_TILE;
  static constexpr int TBUF = (int)TMEM_COLS / BM;  // tensor-memory ring depth
  static constexpr int STAGES_FIT = (int)((kSmemPerCta - 1024 - CONST_BYTES - 512) / STAGE_BYTES);
  static constexpr int STAGES = STAGES_FIT < 6 ? STAGES_FIT : 6;
  static constexpr uint32_t IDESC = idesc_i8(BN, BM);
  static constexpr uint32_t IDESC_BIAS = IDESC & ~((7u << 7) | (7u << 10));  // u8 x u8
  static_assert(KBS % TBUF == 0, "buffer index pattern");
  static_assert(BM % 32 == 0 && BM <= 256, "MMA N and the scale-prep lanes");
  static_assert(STAGES >= 3, "shared-memory ring");
};

template <int BM>
struct Ctrl {
  uint64_t full[Tile<BM>::STAGES];
  uint64_t empty[Tile<BM>::STAGES];
  uint64_t prep[Tile<BM>::STAGES];
  uint64_t tfull[Tile<BM>::TBUF];
  uint64_t tempty[Tile<BM>::TBUF];
  uint64_t drain;
  int exotic[Tile<BM>::STAGES];
  uint32_t tmem_base;
  int abort_flag;
};

template <int BM>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Tile<BM>::STAGES * Tile<BM>::STAGE_BYTES + CONST_BYTES + sizeof(Ctrl<BM>);
}
static_assert(smem_bytes<256>() <= kSmemPerCta && smem_bytes<192>() <= kSmemPerCta &&
                  smem_bytes<128>() <= kSmemPerCta,
              "shared memory");

__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) { return make_float2(__uint_as_float(a), __uint_as_float(b)); }

// Unswizzled K-major descriptor of the constant bias operand (see CONST_BYTES).
__device__ __forceinline__ uint64_t smem_desc_const(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)(128u >> 4) << 16;           // leading byte offset (next core matrix along K)
  d |= (uint64_t)(256u >> 4) << 32;           // stride byte offset (next 8 rows)
  d |= (uint64_t)1 << 46;                     // descriptor version (sm_100)
  return d;                                   // layout type 0: no swizzle
}

// Ties 16 registers written by a tensor-memory load to this point of the
// program: placed after tcgen05.wait::ld, it keeps the compiler from moving
// their uses above the wait.
template <int R>
__device__ __forceinline__ void regs_after_wait(uint32_t (&r)[R]) {
#pragma unroll
  for (int i = 0; i < R; i += 8)
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]),
                      "+r"(r[i + 6]), "+r"(r[i + 7]));
}

// 16 lanes x 128 bits, repeated 4 times along the columns (16 columns):
// thread t holds r[2k] = (lane t/4, column t%4 + 4k) and
// r[2k+1] = (lane t/4 + 8, same column), k = 0..3.
__device__ __forceinline__ void tmem_ld_16x128b_x4(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.16x128b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

// One CW-column chunk of 16 lanes: x4 (16 columns, 8 registers) or x8
// (32 columns, 16 registers).
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, uint32_t (&r)[8]) { tmem_ld_16x128b_x4(taddr, r); }
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, uint32_t (&r)[16]) { tmem_ld_16x128b_x8(taddr, r); }

// Bounded wait that ignores the abort flag (used while draining).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

template <int BM, int EW, int CW, bool DUMP>
__global__ void __launch_bounds__(Warps<EW>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
                const __grid_constant__ CUtensorMap tm_ws, const __grid_constant__ CUtensorMap tm_as,
                __nv_bfloat16* __restrict__ out, int32_t* __restrict__ partials, int* __restrict__ status, int m,
                int n, int k, int n_tiles, int m_tiles, int m_fastest, long long ldo) {
  using T = Tile<BM>;
  using WG = Warps<EW>;
  constexpr int STAGES = T::STAGES;
  constexpr int TBUF = T::TBUF;
  constexpr int EPI_WARPS = WG::EPI_WARPS;
  constexpr int HALVES = EW / 4;            // column groups of epilogue warps
  constexpr int COLS_W = BM / HALVES;       // columns per epilogue warp
  constexpr int CHUNKS = COLS_W / CW;
  constexpr int CR = CW / 2;                // registers of one 16-lane chunk load
  constexpr int KK = CW / 4;                // columns of a chunk per thread
  static_assert(COLS_W % CW == 0 && CHUNKS >= 2, "the epilogue pipelines its loads over >= 2 chunks");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles, keeping the pointer
  // derived from the shared array so accesses stay shared-space loads
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* const_tile = smem + (size_t)STAGES * T::STAGE_BYTES;
  Ctrl<BM>* ctrl = reinterpret_cast<Ctrl<BM>*>(const_tile + CONST_BYTES);
  volatile int* abort_flag = &ctrl->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = n_tiles * m_tiles;
  const int kstages = k / KS;
  const int nb = k / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1 + EPI_WARPS);  // the MMA commit + the epilogue warps
      mbar_init(&ctrl->prep[s], 1);
      ctrl->exotic[s] = 0;
    }
    for (int b = 0; b < TBUF; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], EPI_WARPS);
    }
    mbar_init(&ctrl->drain, 1);
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
  for (int i = threadIdx.x; i < CONST_BYTES / 16; i += WG::THREADS)
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
    setmaxnreg_dec<WG::CTRL_REGS>();
    if (warp == 0) {
      // -------------------------------------------------------------- TMA
      if (lane == 0) {
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
          int n0, m0;
          tile_coords(tile, n0, m0);
          for (int ks = 0; ks < kstages; ++ks, ++it) {
            const int s = (int)(it % STAGES);
            const uint32_t r = it / STAGES;
            if (!mbar_wait(&ctrl->empty[s], (r & 1) ^ 1, abort_flag, status, DEV_ERR_TIMEOUT_TMA)) goto tma_done;
            uint8_t* st = smem + (size_t)s * T::STAGE_BYTES;
            mbar_arrive_expect_tx(&ctrl->full[s], T::STAGE_BYTES);
            tma_load_2d(st, &tm_w, &ctrl->full[s], ks * KS, n0);
            tma_load_2d(st + T::OFF_A, &tm_a, &ctrl->full[s], ks * KS, m0);
            tma_load_2d(st + T::OFF_WS, &tm_ws, &ctrl->full[s], ks * KBS, n0);
            tma_load_2d(st + T::OFF_AS, &tm_as, &ctrl->full[s], m0, ks * KBS);
          }
        }
      tma_done:
        // the copies of the last min(it, STAGES) stages issued must have
        // landed before the CTA may exit (their phases complete on their own;
        // after a normal run they have all completed already)
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
        for (uint32_t j = first; j < it; ++j)
          if (!mbar_wait_drain(&ctrl->full[j % STAGES], (j / STAGES) & 1u)) break;
      }
    } else if (warp == 1) {
      // -------------------------------------------------------------- MMA
      if (lane == 0) {
        const uint64_t c_desc = smem_desc_const(smem_u32(const_tile));
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
          for (int ks = 0; ks < kstages; ++ks, ++it) {
            const int s = (int)(it % STAGES);
            const uint32_t r = it / STAGES;
            if (!mbar_wait(&ctrl->full[s], r & 1, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
            tc_fence_after();
            const uint32_t a_base = smem_u32(smem + (size_t)s * T::STAGE_BYTES);
            const uint32_t b_base = a_base + T::OFF_A;
#pragma unroll
            for (int kb = 0; kb < KBS; ++kb) {
              const uint32_t g = it * KBS + kb;
              const uint32_t buf = g % TBUF;
              const uint32_t use = g / TBUF;
              if (!mbar_wait(&ctrl->tempty[buf], use & 1u, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
              tc_fence_after();
              // D = 2^19 (constant u8 operands of 128s, accumulate off), then D += A x B
              mma_i8(tmem_base + buf * BM, c_desc, c_desc, T::IDESC_BIAS, 0u);
              mma_i8(tmem_base + buf * BM, smem_desc_k_sw128(a_base + kb * 32), smem_desc_k_sw128(b_base + kb * 32),
                     T::IDESC, 1u);
              tc_commit(&ctrl->tfull[buf]);
            }
            tc_commit(&ctrl->empty[s]);
          }
        }
      mma_done:
        // every MMA issued so far (and the arrivals of its commits) has
        // completed once this commit arrives
        tc_commit(&ctrl->drain);
        mbar_wait_drain(&ctrl->drain, 0u);
      }
    } else if (warp == 2) {
      // -------------------------------------------------------------- scale prep
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = (int)(it % STAGES);
          const uint32_t r = it / STAGES;
          if (!mbar_wait(&ctrl->full[s], r & 1, abort_flag, status, DEV_ERR_TIMEOUT_PREP)) goto prep_done;
          uint8_t* st = smem + (size_t)s * T::STAGE_BYTES;
          float* wsf = reinterpret_cast<float*>(st + T::OFF_WS);  // [n][kb] as loaded
          float* asf = reinterpret_cast<float*>(st + T::OFF_AS);  // [kb][m] as loaded
          // pass 1: is every scale of the stage inside the fast path's window?
          bool bad = false;
#pragma unroll
          for (int i = 0; i < (BN * KBS) / 32; ++i) {
            const float aw = fabsf(wsf[i * 32 + lane]);
            bad |= !((aw == 0.0f) | ((aw >= 0x1p-77f) & (aw < 0x1p28f)));
          }
#pragma unroll 4
          for (int i = 0; i < (BM * KBS) / 32; ++i) bad |= !(asf[i * 32 + lane] < 0x1p79f);
          const bool exotic = __any_sync(0xFFFFFFFFu, bad);
          const float fa = exotic ? 1.0f : 0x1p49f;
          const float fw = exotic ? 1.0f : 0x1p100f;
          // pass 2: rewrite both tiles in the order the epilogue reads them.
          // Weight scales [n][kb], n = 32q + 8i + l  ->  [kb][q][l][i]: lane L
          // holds the four kb of row 32q + L (l = L%8, i = L/8).
          float4 wv[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) wv[q] = reinterpret_cast<const float4*>(wsf)[q * 32 + lane];
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float w4[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
#pragma unroll
            for (int kb = 0; kb < KBS; ++kb) wsf[kb * BN + q * 32 + (lane & 7) * 4 + (lane >> 3)] = w4[kb] * fw;
          }
          // Activation scales [kb][m], m = CW*g + 4j + r  ->  [kb][g][r][j]
          // (g = CW-column chunk, r = t%4 of the epilogue thread, j = its
          // column index within the chunk): a permutation inside each chunk.
          // Lane L takes m = 32G + L: chunk offset (L/CW)*CW, j = (L%CW)/4.
#pragma unroll 1
          for (int kb = 0; kb < KBS; ++kb) {
            float av[BM / 32];
#pragma unroll
            for (int g = 0; g < BM / 32; ++g) av[g] = asf[kb * BM + g * 32 + lane];
            __syncwarp();
            const int dst = (lane / CW) * CW + (lane & 3) * (CW / 4) + (lane % CW) / 4;
#pragma unroll
            for (int g = 0; g < BM / 32; ++g) asf[kb * BM + g * 32 + dst] = av[g] * fa;
          }
          // the rewritten bytes are overwritten later by TMA (async proxy)
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            ctrl->exotic[s] = exotic ? 1 : 0;
            mbar_arrive(&ctrl->prep[s]);
          }
        }
      }
    prep_done:;
    }
  } else {
    setmaxnreg_inc<WG::EPI_REGS>();
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int h = (warp - EPI_WARP0) >> 2;
    const int l8 = lane >> 2;
    const int c4 = lane & 3;
    const uint32_t tl = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * COLS_W);
    const int my_tiles = (num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t ws_off = T::OFF_WS + (uint32_t)(q * 32 + l8 * 4) * 4u;                // + kb*BN*4
    const uint32_t as_off = T::OFF_AS + (uint32_t)(h * COLS_W + c4 * KK) * 4u;           // + kb*BM*4 + c*CW*4

    // open the tensor-memory ring
#pragma unroll
    for (int b = 0; b < TBUF; ++b) mbar_arrive_lane0(&ctrl->tempty[b], lane);

    float2 acc[CHUNKS][2][KK];  // acc[c][j][k]: rows (l8 + 16j, l8 + 16j + 8), column CW*c + c4 + 4k
    uint32_t ra[2][CR], rb[2][CR];

    const int total_st = my_tiles * kstages;
    int tile = blockIdx.x, n0 = 0, m0 = 0, kst = 0;
    tile_coords(tile, n0, m0);
    uint32_t st_addr = smem_base;
    uint32_t itg = 0;

    auto dump = [&](int c, int b, const uint32_t (&x)[CR], const uint32_t (&y)[CR]) {
      if constexpr (DUMP) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int nn = n0 + q * 32 + l8 + 8 * i;
#pragma unroll
          for (int kk = 0; kk < KK; ++kk) {
            const int mm = m0 + h * COLS_W + c * CW + c4 + 4 * kk;
            const uint32_t v = (i < 2) ? x[2 * kk + (i & 1)] : y[2 * kk + (i & 1)];
            if (nn < n && mm < m) partials[((size_t)mm * n + nn) * nb + b] = (int)v - (int)kBias;
          }
        }
      }
    };

    // One K block: weight scales, pipelined chunk loads, buffer release,
    // rescale.  kb and the exotic choice are template parameters, so a stage
    // runs one of two fully unrolled code paths with no branch inside.
    auto block = [&](auto kbc, auto exc) -> bool {
      constexpr int kb = decltype(kbc)::value;
      constexpr bool EXO = decltype(exc)::value;
      const uint32_t g = itg * KBS + kb;
      const uint32_t buf = (uint32_t)(kb % TBUF);  // TBUF divides KBS*itg
      const uint32_t par = (g / TBUF) & 1u;
      const float4 W4 = lds_f32x4(st_addr + ws_off + (uint32_t)kb * (BN * 4u));
      const float2 Wp0 = make_float2(W4.x, W4.y), Wp1 = make_float2(W4.z, W4.w);
      float2 Cp0, Cp1;
      if constexpr (!EXO) {
        Cp0 = __fmul2_rn(Wp0, make_float2(-0x1p-130f, -0x1p-130f));
        Cp1 = __fmul2_rn(Wp1, make_float2(-0x1p-130f, -0x1p-130f));
      }
      if (!mbar_wait(&ctrl->tfull[buf], par, abort_flag, status, DEV_ERR_TIMEOUT_EPI)) return false;
      tc_fence_after();
      const uint32_t tb = tl + buf * BM;
      tmem_ld_chunk(tb, ra[0]);
      tmem_ld_chunk(tb + (16u << 16), rb[0]);
      tc_wait_ld();
      regs_after_wait(ra[0]);
      regs_after_wait(rb[0]);
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c) {
        const int cur = c & 1;
        // the fast path loads the next chunk while it rescales this one; the
        // exotic path (rare) loads it afterwards and keeps one buffer live
        if (!EXO && c + 1 < CHUNKS) {
          tmem_ld_chunk(tb + (uint32_t)CW * (c + 1), ra[cur ^ 1]);
          tmem_ld_chunk(tb + (uint32_t)CW * (c + 1) + (16u << 16), rb[cur ^ 1]);
        }
        float av[KK];
#pragma unroll
        for (int v = 0; v < KK / 4; ++v) {
          const float4 A = lds_f32x4(st_addr + as_off + (uint32_t)kb * (BM * 4u) + (uint32_t)c * (CW * 4u) + 16u * v);
          av[4 * v] = A.x;
          av[4 * v + 1] = A.y;
          av[4 * v + 2] = A.z;
          av[4 * v + 3] = A.w;
        }
        dump(c, (kst * KBS) + kb, ra[cur], rb[cur]);
        if constexpr (!EXO) {
#pragma unroll
          for (int kk = 0; kk < KK; ++kk) {
            const float2 u0 = __ffma2_rn(f2(ra[cur][2 * kk], ra[cur][2 * kk + 1]), Wp0, Cp0);
            const float2 u1 = __ffma2_rn(f2(rb[cur][2 * kk], rb[cur][2 * kk + 1]), Wp1, Cp1);
            const float2 ap = make_float2(av[kk], av[kk]);
            acc[c][0][kk] = __ffma2_rn(u0, ap, acc[c][0][kk]);
            acc[c][1][kk] = __ffma2_rn(u1, ap, acc[c][1][kk]);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint32_t* rr = j ? rb[cur] : ra[cur];
              const float ux = __fmul_rn(__int2float_rn((int)rr[2 * kk] - (int)kBias), j ? W4.z : W4.x);
              const float uy = __fmul_rn(__int2float_rn((int)rr[2 * kk + 1] - (int)kBias), j ? W4.w : W4.y);
              acc[c][j][kk].x = __fmaf_rn(ux, av[kk], acc[c][j][kk].x);
              acc[c][j][kk].y = __fmaf_rn(uy, av[kk], acc[c][j][kk].y);
            }
          }
        }
        if (c + 1 < CHUNKS) {
          if (EXO) {
            tmem_ld_chunk(tb + (uint32_t)CW * (c + 1), ra[cur ^ 1]);
            tmem_ld_chunk(tb + (uint32_t)CW * (c + 1) + (16u << 16), rb[cur ^ 1]);
          }
          tc_wait_ld();
          regs_after_wait(ra[cur ^ 1]);
          regs_after_wait(rb[cur ^ 1]);
          if (c + 2 == CHUNKS) {
            // the last chunk is in registers: hand the buffer back to the MMA
            tc_fence_before();
            mbar_arrive_lane0(&ctrl->tempty[buf], lane);
          }
        }
      }
      return true;
    };

    bool ok = true;
    for (; ok && itg < (uint32_t)total_st; ++itg) {
      const int s = (int)(itg % STAGES);
      if (!mbar_wait(&ctrl->prep[s], (itg / STAGES) & 1u, abort_flag, status, DEV_ERR_TIMEOUT_EPI)) break;
      st_addr = smem_base + (uint32_t)s * T::STAGE_BYTES;
      const int exotic = ctrl->exotic[s];
      if (kst == 0) {
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c)
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) acc[c][j][kk] = make_float2(0.0f, 0.0f);
      }
      using K0 = std::integral_constant<int, 0>;
      using K1 = std::integral_constant<int, 1>;
      using K2 = std::integral_constant<int, 2>;
      using K3 = std::integral_constant<int, 3>;
      if (!exotic) {
        const std::false_type fast;
        ok = block(K0{}, fast) && block(K1{}, fast) && block(K2{}, fast) && block(K3{}, fast);
      } else {
        const std::true_type slow;
        ok = block(K0{}, slow) && block(K1{}, slow) && block(K2{}, slow) && block(K3{}, slow);
      }
      if (!ok) break;
      // this stage's scales are no longer read
      mbar_arrive_lane0(&ctrl->empty[s], lane);
      if (++kst == kstages) {
        // tile end: write BF16 out[m][n], one activation row (4 weight rows
        // of it) at a time; the row pointer advances by a volatile add so the
        // compiler does not form all the store addresses at once
        const int nr = n0 + q * 32 + l8;
        const int mr = m0 + h * COLS_W + c4;
        __nv_bfloat16* p = out + (size_t)mr * (size_t)ldo + nr;
        const long long step = 4 * ldo;
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
#pragma unroll
          for (int kk = 0; kk < KK; ++kk) {
            const int mm = mr + CW * c + 4 * kk;
            if (mm < m) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float v = (i & 1) ? acc[c][i >> 1][kk].y : acc[c][i >> 1][kk].x;
                if (nr + 8 * i < n) p[8 * i] = __float2bfloat16_rn(v);
              }
            }
            asm volatile("add.s64 %0, %0, %1;" : "+l"(p) : "l"(step * 2));
          }
        }
        kst = 0;
        tile += gridDim.x;
        tile_coords(tile, n0, m0);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// Epilogue configuration per tile width: (epilogue warps, chunk columns).
template <int BM>
struct Epi;
template <>
struct Epi<128> {
  static constexpr int EW = 8, CW = 32;
};
template <>
struct Epi<192> {
  static constexpr int EW = 8, CW = 32;
};
template <>
struct Epi<256> {
  static constexpr int EW = 8, CW = 16;
};

// Shared-memory opt-in per device and kernel variant, made once under a lock.
std::mutex g_optin_mu;
bool g_optin[64][6] = {};

template <int BM, bool DUMP>
cudaError_t optin_variant(int dev) {
  constexpr int EW = Epi<BM>::EW, CW = Epi<BM>::CW;
  const int slot = (BM == 128 ? 0 : BM == 192 ? 2 : 4) + (DUMP ? 1 : 0);
  if (g_optin[dev][slot]) return cudaSuccess;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, gemm_kernel<BM, EW, CW, DUMP>);
  if (e != cudaSuccess) return e;
  // the register split assumes every thread starts with LAUNCH_REGS registers
  if (fa.numRegs < Warps<EW>::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(gemm_kernel<BM, EW, CW, DUMP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_bytes<BM>());
  if (e != cudaSuccess) return e;
  g_optin[dev][slot] = true;
  return cudaSuccess;
}

template <int BM>
cudaError_t optin(int dev, bool partials) {
  return partials ? optin_variant<BM, true>(dev) : optin_variant<BM, false>(dev);
}

template <int BM>
void launch_bm(const GemmMaps& maps, __nv_bfloat16* out, int32_t* partials, int* status, int m, int n, int k,
               long long ldo, cudaStream_t stream, int grid, int n_tiles, int m_tiles, int m_fastest) {
  constexpr int EW = Epi<BM>::EW, CW = Epi<BM>::CW;
  constexpr int threads = Warps<EW>::THREADS;
  if (partials)
    gemm_kernel<BM, EW, CW, true><<<grid, threads, smem_bytes<BM>(), stream>>>(
        maps.w, maps.a, maps.ws, maps.as, out, partials, status, m, n, k, n_tiles, m_tiles, m_fastest, ldo);
  else
    gemm_kernel<BM, EW, CW, false><<<grid, threads, smem_bytes<BM>(), stream>>>(
        maps.w, maps.a, maps.ws, maps.as, out, nullptr, status, m, n, k, n_tiles, m_tiles, m_fastest, ldo);
}

// Relative epilogue throughput per element of the tile widths, measured on
// B200 from whole-kernel times of the three widths on the 2048 x 14336 x
// 4096, 8192 x 4096 x 14336 and 4095 x 8192 x 8192 projections (they agree
// within 2%): 192 rows give each thread 96 columns in three 32-column chunks
// with no register spills; 256 rows need more registers than the epilogue
// warps hold.
constexpr double kRate128 = 1.0, kRate192 = 1.145, kRate256 = 0.945;

}  // namespace gemm

int gemm_block_m(long long m, long long n, int num_sms) {
  // M <= 128: one activation tile.  Otherwise the width with the least
  // estimated time: whole waves of persistent tiles x tile width / rate.
  if (m <= 128) return 128;
  const long long nt = (n + gemm::BN - 1) / gemm::BN;
  const int widths[3] = {256, 192, 128};
  const double rates[3] = {gemm::kRate256, gemm::kRate192, gemm::kRate128};
  int best = 256;
  double best_t = 0.0;
  for (int i = 0; i < 3; ++i) {
    const long long tiles = nt * ((m + widths[i] - 1) / widths[i]);
    const long long waves = (tiles + num_sms - 1) / num_sms;
    const double t = (double)waves * widths[i] / rates[i];
    if (i == 0 || t < best_t * (1.0 - 1e-9)) {
      best = widths[i];
      best_t = t;
    }
  }
  return best;
}

long long gemm_tiles(long long m, long long n, int num_sms) {
  const long long bm = gemm_block_m(m, n, num_sms);
  return ((n + gemm::BN - 1) / gemm::BN) * ((m + bm - 1) / bm);
}

size_t gemm_smem_bytes() { return gemm::smem_bytes<256>(); }

cudaError_t gemm_prepare_device(bool partials, int bm) {
  using namespace gemm;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_optin_mu);
  switch (bm) {
    case 128: return optin<128>(dev, partials);
    case 192: return optin<192>(dev, partials);
    case 256: return optin<256>(dev, partials);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(const GemmMaps& maps, uint16_t* out, int32_t* partials, int* status, int m, int n, int k,
                        int bm, long long ldo, cudaStream_t stream, int num_sms, int max_ctas) {
  using namespace gemm;
  const int n_tiles = (n + BN - 1) / BN;
  const int m_tiles = (m + bm - 1) / bm;
  const int tiles = n_tiles * m_tiles;
  // persistent CTAs: one per SM, or fewer when the caller shares the GPU
  // between concurrent launches (max_ctas)
  const int cap = (max_ctas > 0 && max_ctas < num_sms) ? max_ctas : num_sms;
  const int grid = tiles < cap ? tiles : cap;
  // Sweep the smaller operand fastest so that it stays resident in L2 while
  // the larger one streams through once.
  const int m_fastest = ((long long)m <= (long long)n) ? 1 : 0;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  switch (bm) {
    case 128: launch_bm<128>(maps, o, partials, status, m, n, k, ldo, stream, grid, n_tiles, m_tiles, m_fastest); break;
    case 192: launch_bm<192>(maps, o, partials, status, m, n, k, ldo, stream, grid, n_tiles, m_tiles, m_fastest); break;
    case 256: launch_bm<256>(maps, o, partials, status, m, n, k, ldo, stream, grid, n_tiles, m_tiles, m_fastest); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace bsr
