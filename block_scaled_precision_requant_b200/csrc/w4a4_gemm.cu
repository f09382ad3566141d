// NVFP4 W4A4 GEMM on the 5th-generation tensor cores (w4a4_proj/fixed.rs,
// `nvfp4_proj_mx`: NVFP4 activations against the NVFP4 weight; the product
// is this library's reading):
//
//   out[m, n] = bf16( scale2_a[m] * scale2_w
//                     * sum_b s16a[m, b] * s16w[n, b] * sum_{i<16} ea[m,16b+i] * ew[n,16b+i] ),
//
// which is exactly what a block-scaled FP4 MMA (`tcgen05.mma kind::mxf4nvf4`,
// E2M1 operands, one UE4M3 scale per 16 elements of K) accumulates in FP32,
// with the two F32 scales applied in the epilogue.
//
// Tiles: 128 activation rows (MMA M, tensor-memory lanes) x 128 weight rows
// (MMA N, columns) x 256 elements of K per stage (128 bytes of packed E2M1
// per row, four MMAs of K = 64).  Operands come by TMA into 128-byte-swizzled
// K-major tiles, exactly as the int8 GEMM stages its int8 codes; the scale
// bytes come by bulk copy in the blocked layout below and are moved into
// tensor memory by `tcgen05.cp` before the stage's MMAs (the copies and the
// MMAs of one thread execute in issue order, so one scale region serves every
// stage).  Accumulators are double-buffered in tensor memory so the epilogue
// of one tile overlaps the MMAs of the next.
//
// Blocked scale layout (built by bsr_nvfp4_sf_blocked from the row-major
// E4M3 bytes): for 128-row tile t and K group g (64 elements = 4 scales) a
// 512-byte atom at offset (t * K/64 + g) * 512; inside it, the 32-bit word
// 4*r0 + r1 holds the four scales of row 128t + r0 + 32*r1 (r0 < 32, r1 < 4),
// scale 4g + j in byte j.  Copied by `tcgen05.cp.32x128b.warpx4`, lane r0 of
// every 32-lane quarter receives the four words of rows r0, r0+32, r0+64,
// r0+96 in four consecutive columns, the arrangement the block-scaled MMA
// reads.  Rows past the matrix are zero.
//
// Roles (6 warps): warp 0 issues the loads, warp 1 the scale copies and the
// MMAs (and owns the tensor-memory allocation), warps 2-5 the epilogue
// (warp w reads lanes 32*(w%4).., the quarter it may access).  Every wait is
// bounded: a wait that runs out sets a status bit and the CTA drains its
// in-flight copies and MMAs (with bounded waits), frees its tensor memory
// and returns.
#include <cuda_bf16.h>

#include <cstdint>
#include <mutex>

#include "bsr.h"
#include "common.cuh"
#include "w4a4_desc.cuh"

namespace bsr {
// Records the message bsr_last_error() returns on this thread (api.cu).
bsr_status report(bsr_status st, const char* fmt, ...);
// Device address of the library's status word on the current device (api.cu).
bsr_status library_status_word(int** out);
// The NVFP4 row quantiser's launch (w4a4.cu).
cudaError_t launch_nvfp4_quant_rows(const uint16_t* a, uint8_t* a_packed, uint8_t* a_e4m3, float* a_scale2, int m,
                                    int k, cudaStream_t stream, int num_sms);
}  // namespace bsr

namespace bsr {
namespace w4gemm {

constexpr int BM = 128;                  // activation rows per tile
constexpr int BN = 128;                  // weight rows per tile
constexpr int KB = 128;                  // bytes of packed E2M1 per row and stage (256 elements)
constexpr int KE = 2 * KB;               // elements of K per stage
constexpr int MMAS = KE / 64;            // MMAs per stage (K = 64 each)
constexpr int STAGES = 5;
constexpr int A_TILE = BM * KB;          // 16384
constexpr int B_TILE = BN * KB;          // 16384
constexpr int SF_STAGE = MMAS * 512;     // scale atoms of one operand per stage: 2048
constexpr int OFF_B = A_TILE;
constexpr int OFF_SFA = A_TILE + B_TILE;
constexpr int OFF_SFB = OFF_SFA + SF_STAGE;
constexpr int STAGE_BYTES = OFF_SFB + SF_STAGE;  // 36864
constexpr int THREADS = 192;  // warp 0 loads, warp 1 MMAs, warps 2-5 epilogue
constexpr int ACC_BUFS = 2;
constexpr uint32_t TMEM_COLS = 512;      // 2 x 128 accumulator columns + 2 x 16 scale columns, rounded up
constexpr uint32_t COL_SFA = ACC_BUFS * BN;        // 256
constexpr uint32_t COL_SFB = COL_SFA + 4 * MMAS;   // 272
static_assert(COL_SFB + 4 * MMAS <= TMEM_COLS, "tensor-memory plan");

constexpr uint32_t kIdesc = idesc_mxf4(BM, BN);

struct Ctrl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[ACC_BUFS];
  uint64_t tempty[ACC_BUFS];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Ctrl);

__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 bits, 32 columns: thread t holds lane t, columns c..c+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Bounded wait that ignores the abort flag: used while draining after an
// abort.  Returns false when the limit runs out.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t l = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

__global__ void __launch_bounds__(THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                     const uint8_t* __restrict__ a_sf, const uint8_t* __restrict__ w_sf,
                     const float* __restrict__ a_scale2, float scale2_w, __nv_bfloat16* __restrict__ out,
                     int* __restrict__ status, int m, int n, int k, int m_tiles, int n_tiles, int m_fastest,
                     int vec_store) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + (size_t)STAGES * STAGE_BYTES);
  volatile int* abort_flag = &ctrl->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = m_tiles * n_tiles;
  const int kstages = k / KE;
  const int kgroups = k / 64;  // scale atoms per 128-row tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int b = 0; b < ACC_BUFS; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], 4);  // the four epilogue warps
    }
    mbar_init(&ctrl->drain, 1);
    ctrl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctrl->tmem_base;

  auto tile_coords = [&](int tile, int& m0, int& n0) {
    int tm, tn;
    if (m_fastest) {
      tn = tile / m_tiles;
      tm = tile - tn * m_tiles;
    } else {
      tm = tile / n_tiles;
      tn = tile - tm * n_tiles;
    }
    m0 = tm * BM;
    n0 = tn * BN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        int m0, n0;
        tile_coords(tile, m0, n0);
        const uint8_t* sfa = a_sf + ((size_t)(m0 / BM) * kgroups) * 512;
        const uint8_t* sfb = w_sf + ((size_t)(n0 / BN) * kgroups) * 512;
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = (int)(it % STAGES);
          const uint32_t r = it / STAGES;
          if (!mbar_wait(&ctrl->empty[s], (r & 1) ^ 1, abort_flag, status, DEV_ERR_TIMEOUT_TMA)) goto loads_done;
          uint8_t* st = smem + (size_t)s * STAGE_BYTES;
          mbar_arrive_expect_tx(&ctrl->full[s], STAGE_BYTES);
          tma_load_2d(st, &tm_a, &ctrl->full[s], ks * KB, m0);
          tma_load_2d(st + OFF_B, &tm_w, &ctrl->full[s], ks * KB, n0);
          bulk_load(st + OFF_SFA, sfa + (size_t)ks * SF_STAGE, SF_STAGE, &ctrl->full[s]);
          bulk_load(st + OFF_SFB, sfb + (size_t)ks * SF_STAGE, SF_STAGE, &ctrl->full[s]);
        }
      }
    loads_done:
      // drain: the last min(it, STAGES) stages issued must have landed
      // before the CTA may exit (their phases complete on their own)
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
      for (uint32_t j = first; j < it; ++j)
        if (!mbar_wait_drain(&ctrl->full[j % STAGES], (j / STAGES) & 1u, kWaitLimitNs)) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMAs
    if (lane == 0) {
      uint32_t it = 0;
      uint32_t tcount = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1u;
        const uint32_t use = tcount >> 1;
        if (!mbar_wait(&ctrl->tempty[buf], (use & 1u) ^ 1u, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = (int)(it % STAGES);
          if (!mbar_wait(&ctrl->full[s], (it / STAGES) & 1u, abort_flag, status, DEV_ERR_TIMEOUT_MMA)) goto mma_done;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + (size_t)s * STAGE_BYTES);
#pragma unroll
          for (int j = 0; j < MMAS; ++j) {
            tmem_cp_32x128b_x4(tmem_base + COL_SFA + 4 * j, smem_desc_k_plain(st + OFF_SFA + 512 * j));
            tmem_cp_32x128b_x4(tmem_base + COL_SFB + 4 * j, smem_desc_k_plain(st + OFF_SFB + 512 * j));
          }
#pragma unroll
          for (int j = 0; j < MMAS; ++j)
            mma_mxf4(d_tmem, smem_desc_k_sw128(st + 32 * j), smem_desc_k_sw128(st + OFF_B + 32 * j), kIdesc,
                     tmem_base + COL_SFA + 4 * j, tmem_base + COL_SFB + 4 * j, (ks | j) != 0 ? 1u : 0u);
          tc_commit(&ctrl->empty[s]);
        }
        tc_commit(&ctrl->tfull[buf]);
      }
    mma_done:
      // drain: every MMA and copy issued so far has completed once this
      // commit arrives
      tc_commit(&ctrl->drain);
      mbar_wait_drain(&ctrl->drain, 0u, kWaitLimitNs);
    }
  } else {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;  // tensor-memory lane quarter this warp may read
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
      int m0, n0;
      tile_coords(tile, m0, n0);
      const uint32_t buf = tcount & 1u;
      const uint32_t use = tcount >> 1;
      const int row = m0 + q * 32 + lane;
      const float s2a = row < m ? __ldg(a_scale2 + row) : 0.0f;
      if (!mbar_wait(&ctrl->tfull[buf], use & 1u, abort_flag, status, DEV_ERR_TIMEOUT_EPI)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + lane_addr + buf * BN + 32 * c, r);
        tc_wait_ld();
        uint32_t p[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          p[j] = pack_bf16x2(__fmul_rn(__fmul_rn(__uint_as_float(r[2 * j]), s2a), scale2_w),
                             __fmul_rn(__fmul_rn(__uint_as_float(r[2 * j + 1]), s2a), scale2_w));
        const int col0 = n0 + 32 * c;
        if (row < m) {
          __nv_bfloat16* dst = out + (size_t)row * (size_t)n + col0;
          if (vec_store && col0 + 32 <= n) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<uint4*>(dst)[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < n)
                dst[j] = __ushort_as_bfloat16((unsigned short)((j & 1) ? (p[j >> 1] >> 16) : (p[j >> 1] & 0xFFFFu)));
          }
        }
      }
      tc_fence_before();
      mbar_arrive_lane0(&ctrl->tempty[buf], lane);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// Row-major E4M3 scales [rows, K/16] -> the blocked atoms described above;
// one thread per 32-bit word of the output, rows past `rows` zero.
__global__ void __launch_bounds__(256) sf_blocked_kernel(const uint8_t* __restrict__ src, uint32_t* __restrict__ dst,
                                                         int rows, int k, long long words) {
  const int kgroups = k / 64;
  const int ld = k / 16;  // bytes per source row
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < words; w += stride) {
    const long long atom = w >> 7;
    const int wi = (int)(w & 127);
    const long long t = atom / kgroups;
    const int g = (int)(atom - t * kgroups);
    const long long row = t * 128 + (wi >> 2) + 32 * (wi & 3);
    dst[w] = row < rows ? __ldg(reinterpret_cast<const uint32_t*>(src + row * ld + 4 * g)) : 0u;
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows, K/2] packed E2M1 bytes, box 128 B x 128 rows, 128-byte swizzle;
// rows past the matrix read as zero.
bsr_status encode_fp4_map(CUtensorMap* map, const void* base, long long rows, long long k, const char* what) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return report(BSR_ECUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)KB, (cuuint32_t)BM};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return report(BSR_ECUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
  return BSR_OK;
}

// Per-device properties and the status word's device address.
struct Dev {
  int num_sms = 0;
  size_t smem_optin = 0;
  int cc_major = 0;
  bool granted = false;
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
  if (!d.granted) {
    if (SMEM_BYTES > d.smem_optin) return report(BSR_ENODEV, "device %d: too little shared memory per CTA", dev);
    e = cudaFuncSetAttribute(w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return report(BSR_ECUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    d.granted = true;
  }
  out = d;
  return BSR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

long long sf_blocked_bytes(long long rows, long long k) { return (rows + 127) / 128 * (k / 64) * 512; }

cudaError_t launch_sf_blocked(const uint8_t* e4m3, uint8_t* blocked, long long rows, long long k, cudaStream_t stream,
                              int num_sms) {
  const long long words = sf_blocked_bytes(rows, k) / 4;
  long long grid = (words + 255) / 256;
  if (grid > 8LL * num_sms) grid = 8LL * num_sms;
  sf_blocked_kernel<<<(unsigned)grid, 256, 0, stream>>>(e4m3, reinterpret_cast<uint32_t*>(blocked), (int)rows,
                                                        (int)k, words);
  return cudaGetLastError();
}

// Everything a GEMM launch needs, prepared (and every check done) before
// anything is queued.
struct GemmLaunch {
  CUtensorMap tm_a, tm_w;
  int grid, m_tiles, n_tiles, m_fastest, vec_store;
};

bsr_status prepare_gemm(GemmLaunch& g, const uint8_t* a_packed, const uint8_t* w_packed, long long m, long long n,
                        long long k, int num_sms) {
  bsr_status st;
  if ((st = encode_fp4_map(&g.tm_a, a_packed, m, k, "a_packed")) != BSR_OK) return st;
  if ((st = encode_fp4_map(&g.tm_w, w_packed, n, k, "w_packed")) != BSR_OK) return st;
  g.m_tiles = (int)((m + BM - 1) / BM);
  g.n_tiles = (int)((n + BN - 1) / BN);
  const long long tiles = (long long)g.m_tiles * g.n_tiles;
  if (tiles > 0x7FFFFFFFLL) return report(BSR_EINVAL, "too many tiles");
  g.grid = (int)(tiles < num_sms ? tiles : num_sms);
  // sweep the smaller operand fastest so it stays in L2 while the larger one
  // streams through once
  g.m_fastest = m <= n ? 1 : 0;
  g.vec_store = n % 8 == 0 ? 1 : 0;
  return BSR_OK;
}

cudaError_t launch_prepared(const GemmLaunch& g, const uint8_t* a_sf, const uint8_t* w_sf, const float* a_scale2,
                            float scale2, uint16_t* out, int* status, long long m, long long n, long long k,
                            cudaStream_t stream) {
  w4a4_gemm_kernel<<<g.grid, THREADS, SMEM_BYTES, stream>>>(
      g.tm_a, g.tm_w, a_sf, w_sf, a_scale2, scale2, reinterpret_cast<__nv_bfloat16*>(out), status, (int)m, (int)n,
      (int)k, g.m_tiles, g.n_tiles, g.m_fastest, g.vec_store);
  return cudaGetLastError();
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch of the composite entry: packed codes, E4M3 bytes, blocked scales,
// row scales, each 256-byte aligned.
struct ProjScratch {
  size_t packed, e4m3, blocked, scale2, total;
};

ProjScratch proj_scratch(long long m, long long k) {
  ProjScratch p;
  p.packed = 0;
  p.e4m3 = align256((size_t)m * (size_t)(k / 2));
  p.blocked = p.e4m3 + align256((size_t)m * (size_t)(k / 16));
  p.scale2 = p.blocked + align256((size_t)sf_blocked_bytes(m, k));
  p.total = p.scale2 + align256((size_t)m * 4);
  return p;
}

}  // namespace w4gemm
}  // namespace bsr

extern "C" {

size_t bsr_nvfp4_sf_blocked_bytes(int64_t rows, int64_t k) {
  if (rows <= 0 || rows > BSR_MAX_DIM || k <= 0 || k > BSR_MAX_DIM || k % 64 != 0) return 0;
  return (size_t)bsr::w4gemm::sf_blocked_bytes(rows, k);
}

bsr_status bsr_nvfp4_sf_blocked(const uint8_t* e4m3, uint8_t* blocked, int64_t rows, int64_t k, void* stream) {
  using namespace bsr::w4gemm;
  if (rows < 0 || rows > BSR_MAX_DIM || k < 0 || k > BSR_MAX_DIM)
    return bsr::report(BSR_EINVAL, "dimension out of range (rows=%lld k=%lld)", (long long)rows, (long long)k);
  if (k == 0 || k % 64 != 0) return bsr::report(BSR_ESHAPE, "K=%lld must be a positive multiple of 64", (long long)k);
  if (rows == 0) return bsr::report(BSR_OK, "");
  if (!e4m3 || !blocked) return bsr::report(BSR_EINVAL, "null pointer");
  if (!aligned16(e4m3) || !aligned16(blocked))
    return bsr::report(BSR_EALIGN, "e4m3 and blocked must be 16-byte aligned");
  Dev d;
  int dev = 0;
  bsr_status st = query_device(d, dev);
  if (st != BSR_OK) return st;
  const cudaError_t e = launch_sf_blocked(e4m3, blocked, rows, k, reinterpret_cast<cudaStream_t>(stream), d.num_sms);
  if (e != cudaSuccess) return bsr::report(BSR_ECUDA, "scale relayout launch: %s", cudaGetErrorString(e));
  return bsr::report(BSR_OK, "");
}

bsr_status bsr_w4a4_gemm(const uint8_t* a_packed, const uint8_t* a_sf_blocked, const float* a_scale2,
                         const uint8_t* w_packed, const uint8_t* w_sf_blocked, float scale2, uint16_t* out, int64_t m,
                         int64_t n, int64_t k, int* status_dev, void* stream) {
  using namespace bsr::w4gemm;
  if (m < 0 || m > BSR_MAX_DIM || n < 0 || n > BSR_MAX_DIM || k < 0 || k > BSR_MAX_DIM)
    return bsr::report(BSR_EINVAL, "dimension out of range (m=%lld n=%lld k=%lld)", (long long)m, (long long)n,
                       (long long)k);
  if (k == 0 || k % KE != 0) return bsr::report(BSR_ESHAPE, "K=%lld must be a positive multiple of 256", (long long)k);
  if (m == 0 || n == 0) return bsr::report(BSR_OK, "");
  if (!a_packed || !a_sf_blocked || !a_scale2 || !w_packed || !w_sf_blocked || !out || !status_dev)
    return bsr::report(BSR_EINVAL, "null pointer");
  if (!aligned16(a_packed) || !aligned16(a_sf_blocked) || !aligned16(a_scale2) || !aligned16(w_packed) ||
      !aligned16(w_sf_blocked) || !aligned16(out))
    return bsr::report(BSR_EALIGN, "all arrays must be 16-byte aligned");
  Dev d;
  int dev = 0;
  bsr_status st = query_device(d, dev);
  if (st != BSR_OK) return st;
  GemmLaunch g;
  if ((st = prepare_gemm(g, a_packed, w_packed, m, n, k, d.num_sms)) != BSR_OK) return st;
  const cudaError_t e = launch_prepared(g, a_sf_blocked, w_sf_blocked, a_scale2, scale2, out, status_dev, m, n, k,
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return bsr::report(BSR_ECUDA, "w4a4 GEMM launch: %s", cudaGetErrorString(e));
  return bsr::report(BSR_OK, "");
}

size_t bsr_w4a4_proj_scratch_bytes(int64_t m, int64_t k) {
  using namespace bsr::w4gemm;
  if (m <= 0 || m > BSR_MAX_DIM || k <= 0 || k > BSR_MAX_DIM || k % KE != 0) return 0;
  return proj_scratch(m, k).total;
}

bsr_status bsr_w4a4_proj(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_sf_blocked, float scale2,
                         uint16_t* out, int64_t m, int64_t n, int64_t k, void* scratch, size_t scratch_bytes,
                         void* stream) {
  using namespace bsr::w4gemm;
  if (m < 0 || m > BSR_MAX_DIM || n < 0 || n > BSR_MAX_DIM || k < 0 || k > BSR_MAX_DIM)
    return bsr::report(BSR_EINVAL, "dimension out of range (m=%lld n=%lld k=%lld)", (long long)m, (long long)n,
                       (long long)k);
  if (k == 0 || k % KE != 0) return bsr::report(BSR_ESHAPE, "K=%lld must be a positive multiple of 256", (long long)k);
  if (m == 0 || n == 0) return bsr::report(BSR_OK, "");
  if (!a || !w_packed || !w_sf_blocked || !out) return bsr::report(BSR_EINVAL, "null pointer");
  if (!aligned16(a) || !aligned16(w_packed) || !aligned16(w_sf_blocked) || !aligned16(out))
    return bsr::report(BSR_EALIGN, "a, w_packed, w_sf_blocked and out must be 16-byte aligned");
  const ProjScratch ps = proj_scratch(m, k);
  if (!scratch || scratch_bytes < ps.total)
    return bsr::report(BSR_ESCRATCH, "scratch of %zu bytes needed, %zu given", ps.total,
                       scratch ? scratch_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0)
    return bsr::report(BSR_EALIGN, "scratch must be 256-byte aligned");
  Dev d;
  int dev = 0;
  bsr_status st = query_device(d, dev);
  if (st != BSR_OK) return st;
  int* status = nullptr;
  if ((st = bsr::library_status_word(&status)) != BSR_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint8_t* a_packed = base + ps.packed;
  uint8_t* a_e4m3 = base + ps.e4m3;
  uint8_t* a_sf = base + ps.blocked;
  float* a_scale2 = reinterpret_cast<float*>(base + ps.scale2);
  // every tensor map is encoded before the first launch, so a failure
  // leaves nothing queued
  GemmLaunch g;
  if ((st = prepare_gemm(g, a_packed, w_packed, m, n, k, d.num_sms)) != BSR_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = bsr::launch_nvfp4_quant_rows(a, a_packed, a_e4m3, a_scale2, (int)m, (int)k, s, d.num_sms);
  if (e == cudaSuccess) e = launch_sf_blocked(a_e4m3, a_sf, m, k, s, d.num_sms);
  if (e == cudaSuccess) e = launch_prepared(g, a_sf, w_sf_blocked, a_scale2, scale2, out, status, m, n, k, s);
  if (e != cudaSuccess) return bsr::report(BSR_ECUDA, "w4a4 projection launch: %s", cudaGetErrorString(e));
  return bsr::report(BSR_OK, "");
}

}  // extern "C"
