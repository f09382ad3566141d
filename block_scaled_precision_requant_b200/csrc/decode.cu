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
// Memory: one warp per weight row.  Lane 0 of each warp streams its row
// (and, when the row pitch allows, the row's scales) into the warp's own
// shared-memory slot as bulk copies of up to 16 KB, all issued at kernel
// start: the whole weight is in flight at once without holding registers.
// The slot is read in 1 KB chunks, one 32-block per lane, each chunk with
// its own mbarrier.  Meanwhile the CTA requantises the activation rows
// into shared memory (same rule and code as requant_a, so the codes match it
// bit for bit).  Launched with programmatic dependent launch: activations
// are read after waiting for the previous kernel on the stream; with the
// static-weight option an eighth of the warps send their first row's copies
// before that wait.  The
// weight is one [N, K] tensor or a table of stacked segments.
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace bsr {

// Warps (= weight rows in flight) per CTA at most: 32 for one or two
// activation rows, 8 for more (their per-row register arrays grow).
template <int MR>
constexpr int decode_max_warps() { return MR <= 2 ? 32 : 8; }

// 1 KB chunks per bulk copy of a weight row: a weight-sized stream of
// 1 KB copies measured at well under half the HBM rate of 16 KB copies
// (each CTA issuing its share before the grid-dependency wait).
constexpr uint32_t kChunksPerCopy = 16;

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

// Shared-memory layout of one CTA (byte offsets).
struct DecodeSmem {
  uint32_t codes, ascale, wrow, wscale, bars, abort_flag, total;
  uint32_t wrow_bytes, wscale_bytes;  // per warp
  uint32_t chunks;                    // 1 KB weight chunks per row (one 32-block per lane)
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline DecodeSmem decode_smem_layout(int mr, int k, int nwarps, bool scale_bulk) {
  DecodeSmem L;
  const uint32_t nb = (uint32_t)k / 32;
  L.codes = 0;
  L.ascale = align_up((uint32_t)mr * (uint32_t)k, 16);
  L.wrow_bytes = (uint32_t)k;
  L.wscale_bytes = scale_bulk ? nb * 4 : 0;
  L.wrow = align_up(L.ascale + (uint32_t)mr * nb * 4, 128);
  L.wscale = L.wrow + (uint32_t)nwarps * L.wrow_bytes;
  L.chunks = (nb + 31) / 32;
  L.bars = align_up(L.wscale + (uint32_t)nwarps * L.wscale_bytes, 8);
  L.abort_flag = L.bars + (uint32_t)nwarps * L.chunks * 8;
  L.total = L.abort_flag + 16;
  return L;
}

// Where a weight row comes from: one weight (compact kernel parameters: they
// are read on the kernel's critical path before its first copy, and a larger
// parameter block measured ~0.5 us slower per launch), or a table of up to
// kMaxDecodeSegs segments (stacked weight).
struct DecodeSingle {
  const int8_t* w;
  const float* ws;
  int n;
};
__device__ __forceinline__ int src_rows(const DecodeSingle& s) { return s.n; }
__device__ __forceinline__ int src_rows(const DecodeSegs& s) { return s.off[s.count]; }
__device__ __forceinline__ void src_row(const DecodeSingle& s, int r, int k, int nb, const int8_t*& w,
                                        const float*& ws) {
  w = s.w + (size_t)r * (size_t)k;
  ws = s.ws + (size_t)r * (size_t)nb;
}
// output column r of a stacked weight: row r - off[s] of the segment s with
// off[s] <= r < off[s + 1]
__device__ __forceinline__ void src_row(const DecodeSegs& s, int r, int k, int nb, const int8_t*& w,
                                        const float*& ws) {
  int i = 0;
#pragma unroll
  for (int j = 1; j < kMaxDecodeSegs; ++j) i += (j < s.count && r >= s.off[j]) ? 1 : 0;
  const size_t local = (size_t)(r - s.off[i]);
  w = s.w[i] + local * (size_t)k;
  ws = s.ws[i] + local * (size_t)nb;
}

// MR: activation rows per CTA (compile time, >= rows actually present).
template <int MR, class Src>
__global__ void __launch_bounds__(decode_max_warps<MR>() * 32, 1)
    decode_kernel(const uint16_t* __restrict__ a, const Src src, __nv_bfloat16* __restrict__ out, int m, int k,
                  int scale_bulk, int static_weight, int* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int nb = k >> 5;
  const int n = src_rows(src);  // output columns = weight rows
  auto seg_row = [&](int r, const int8_t*& wr, const float*& wsr) { src_row(src, r, k, nb, wr, wsr); };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const DecodeSmem L = decode_smem_layout(MR, k, nwarps, scale_bulk != 0);
  int8_t* s_codes = reinterpret_cast<int8_t*>(smem + L.codes);
  float* s_scale = reinterpret_cast<float*>(smem + L.ascale);
  int8_t* s_w = reinterpret_cast<int8_t*>(smem + L.wrow + (uint32_t)warp * L.wrow_bytes);
  float* s_ws = reinterpret_cast<float*>(smem + L.wscale + (uint32_t)warp * L.wscale_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + (size_t)warp * L.chunks;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.abort_flag);

  const int m0 = blockIdx.y * MR;
  const int rows = min(MR, m - m0);
  int row = blockIdx.x * nwarps + warp;
  const int row_step = gridDim.x * nwarps;

  if (threadIdx.x == 0) *abort_flag = 0;
  if (lane == 0) {
    for (uint32_t c = 0; c < L.chunks; ++c) mbar_init(&bars[c], 1);
    fence_mbar_init();
  }
  __syncwarp();
  // A row goes out as bulk copies of up to kChunksPerCopy 1 KB chunks (one
  // 32-block per lane per chunk); a row longer than one copy is consumed
  // copy by copy while its tail still streams.
  auto issue_row = [&](int r) {
    if (lane == 0 && r < n) {
      const int8_t* wr;
      const float* wsr;
      seg_row(r, wr, wsr);
      // up to kChunksPerCopy chunks (and their scales) per bulk copy, on the
      // group's first barrier; the group's other barriers complete at once,
      // so the consumer's per-chunk waits are unchanged
      for (uint32_t c0 = 0; c0 < L.chunks; c0 += kChunksPerCopy) {
        const uint32_t cn = min(kChunksPerCopy, L.chunks - c0);
        const uint32_t blocks = min(32u * cn, (uint32_t)nb - 32u * c0);
        const uint32_t wb = blocks * 32u, sb = L.wscale_bytes ? blocks * 4u : 0u;
        mbar_arrive_expect_tx(&bars[c0], wb + sb);
        bulk_load(s_w + (size_t)c0 * 1024, wr + (size_t)c0 * 1024, wb, &bars[c0]);
        if (sb) bulk_load(s_ws + (size_t)c0 * 32, wsr + (size_t)c0 * 32, sb, &bars[c0]);
        for (uint32_t c = c0 + 1; c < c0 + cn; ++c) mbar_arrive(&bars[c]);
      }
    }
  };

  // Activation requantisation into shared memory: 4 lanes per 32-group,
  // 8 groups per warp per pass.  The first pass's activation loads go out
  // before the weight copies so they are not queued behind the weight stream.
  {
    const int groups = MR * nb;
    const int sub = lane & 3;
    auto load_act = [&](int g0) {
      const int g = g0 + (lane >> 2);
      const int r = g / nb;
      const int b = g - r * nb;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (g < groups && r < rows)
        v = __ldg(reinterpret_cast<const uint4*>(a + (size_t)(m0 + r) * k + (size_t)b * 32 + sub * 8));
      return v;
    };
    // Launched with programmatic stream serialisation: the grid may be
    // scheduled while the previous kernel on the stream drains.  Wait for
    // that kernel to complete (and its writes to be visible) before reading
    // what it may have written, and let the next kernel be scheduled early in
    // turn.  With static_weight the caller guarantees that no kernel ahead
    // on the stream writes the weight, so the first eighth of the warps (at
    // least one) send their first row's copies before the wait, overlapping
    // the previous kernel's tail; the rest send theirs once the activation
    // loads are out.  Issuing every warp's row before the wait queues the
    // activation loads behind the whole first wave of the weight stream and
    // delays the requantisation that every row needs (slower at M=1,
    // N=K=4096 by about 15%); issuing none leaves the tail unused.
    const bool early = static_weight && warp < (nwarps + 7) / 8;
    if (early) issue_row(row);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    uint4 av = load_act(warp * 8);
    if (!early) issue_row(row);
    for (int g0 = warp * 8; g0 < groups; g0 += nwarps * 8) {
      const int g = g0 + (lane >> 2);
      const int r = g / nb;
      const int b = g - r * nb;
      const uint4 v = av;
      if (g0 + nwarps * 8 < groups) av = load_act(g0 + nwarps * 8);
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

  // Lane l reads the two 16-byte halves of its 32-byte block in the order h,
  // 1-h with h = (l >> 2) & 1, so each 8-lane phase of a 16-byte shared load
  // hits eight distinct 16-byte bank groups.
  const int h = (lane >> 2) & 1;
  uint32_t phase = 0;
  bool aborted = false;
  for (; row < n; row += row_step) {
    const int8_t* wrow;
    const float* wsrow;
    seg_row(row, wrow, wsrow);
    (void)wrow;
    float acc[MR];
#pragma unroll
    for (int r = 0; r < MR; ++r) acc[r] = 0.0f;
    for (int b = lane, c = 0; c < (int)L.chunks; b += 32, ++c) {
      // warp-uniform decision: a lane whose wait ran out takes the whole warp
      // out (the warp synchronises after the row)
      const bool landed = mbar_wait(&bars[c], phase, abort_flag, status, DEV_ERR_TIMEOUT_DECODE);
      if (__any_sync(0xFFFFFFFFu, !landed)) {
        aborted = true;
        break;
      }
      if (b >= nb) continue;
      const uint4* wsrc = reinterpret_cast<const uint4*>(s_w + (size_t)b * 32);
      const uint4 w0 = wsrc[h];
      const uint4 w1 = wsrc[1 - h];
      const float wsb = L.wscale_bytes ? s_ws[b] : __ldg(wsrow + b);
#pragma unroll
      for (int r = 0; r < MR; ++r) {
        const uint4* cs = reinterpret_cast<const uint4*>(s_codes + (size_t)r * k + (size_t)b * 32);
        const int p = dot32(w0, w1, cs[h], cs[1 - h]);
        const float u = __fmul_rn(__int2float_rn(p), wsb);
        acc[r] = __fmaf_rn(u, s_scale[r * nb + b], acc[r]);
      }
    }
    if (aborted) break;
    phase ^= 1u;
    // every lane has read the row slot: it may be refilled (async proxy)
    __syncwarp();
    fence_proxy_async_smem();
    issue_row(row + row_step);
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
  }
  // A warp that gave up waiting may still have its copy in flight: wait for it
  // once more, again bounded, so the CTA does not exit under a bulk copy.
  if (aborted && lane == 0) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t c = 0; c < L.chunks; ++c)
      while (!mbar_try_wait(&bars[c], phase) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
  }
}

static bool decode_scale_bulk(int k) { return (k % 128) == 0; }

static std::mutex g_decode_optin_mu;

// Rows per CTA: the largest power of two <= 16 that covers M and fits the
// shared-memory budget together with at least one weight-row slot.
int decode_rows_per_cta(int m, int k, size_t smem_limit) {
  int mr = 1;
  while (mr < m && mr < 16) mr <<= 1;
  auto fits = [&](int r) { return decode_smem_layout(r, k, 1, decode_scale_bulk(k)).total <= smem_limit; };
  while (mr > 1 && !fits(mr)) mr >>= 1;
  return fits(mr) ? mr : 0;
}

// Warps per CTA and dynamic shared memory of a launch over n weight rows,
// with the kernel's shared-memory opt-in (raised once per device and
// variant, under a lock shared by all variants).
template <int MR, class Src>
static cudaError_t decode_config(int n, int k, size_t smem_limit, int num_sms, int& w, size_t& smem) {
  const bool sb = decode_scale_bulk(k);
  // Warps (= weight rows in flight) per CTA: spread the rows over all SMs,
  // at most decode_max_warps<MR>() per CTA and as many row slots as fit in
  // shared memory; beyond one CTA per SM the warps loop over rows.
  constexpr int kMaxW = decode_max_warps<MR>();
  w = (int)((n + (long long)num_sms - 1) / num_sms);
  w = w < 1 ? 1 : (w > kMaxW ? kMaxW : w);
  while (w > 1 && decode_smem_layout(MR, k, w, sb).total > smem_limit) --w;
  smem = decode_smem_layout(MR, k, w, sb).total;
  static size_t granted[64] = {};  // per device, per <MR, Src>
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_decode_optin_mu);
  if (smem > granted[dev]) {
    e = cudaFuncSetAttribute(decode_kernel<MR, Src>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    granted[dev] = smem;
  }
  return cudaSuccess;
}

template <int MR, class Src>
static cudaError_t launch_decode_t(const uint16_t* a, const Src& src, int n, uint16_t* out, int m, int k,
                                   int static_weight, int* status, size_t smem_limit, cudaStream_t stream,
                                   int num_sms) {
  auto kern = decode_kernel<MR, Src>;
  const bool sb = decode_scale_bulk(k);
  int w = 1;
  size_t smem = 0;
  cudaError_t e = decode_config<MR, Src>(n, k, smem_limit, num_sms, w, smem);
  if (e != cudaSuccess) return e;
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
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  e = cudaLaunchKernelEx(&cfg, kern, a, src, o, m, k, sb ? 1 : 0, static_weight ? 1 : 0, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <class Src>
static cudaError_t launch_decode_src(const uint16_t* a, const Src& src, int n, uint16_t* out, int m, int k, int mr,
                                     int sw, int* status, size_t smem_limit, cudaStream_t stream, int num_sms) {
  switch (mr) {
    case 1: return launch_decode_t<1, Src>(a, src, n, out, m, k, sw, status, smem_limit, stream, num_sms);
    case 2: return launch_decode_t<2, Src>(a, src, n, out, m, k, sw, status, smem_limit, stream, num_sms);
    case 4: return launch_decode_t<4, Src>(a, src, n, out, m, k, sw, status, smem_limit, stream, num_sms);
    case 8: return launch_decode_t<8, Src>(a, src, n, out, m, k, sw, status, smem_limit, stream, num_sms);
    case 16: return launch_decode_t<16, Src>(a, src, n, out, m, k, sw, status, smem_limit, stream, num_sms);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t prepare_decode(int n, int k, int mr, size_t smem_limit, int num_sms) {
  int w = 1;
  size_t smem = 0;
  switch (mr) {
    case 1: return decode_config<1, DecodeSingle>(n, k, smem_limit, num_sms, w, smem);
    case 2: return decode_config<2, DecodeSingle>(n, k, smem_limit, num_sms, w, smem);
    case 4: return decode_config<4, DecodeSingle>(n, k, smem_limit, num_sms, w, smem);
    case 8: return decode_config<8, DecodeSingle>(n, k, smem_limit, num_sms, w, smem);
    case 16: return decode_config<16, DecodeSingle>(n, k, smem_limit, num_sms, w, smem);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int m, int n,
                          int k, int mr, int static_weight, int* status, size_t smem_limit, cudaStream_t stream,
                          int num_sms) {
  const DecodeSingle src = {w_i8, w_scale, n};
  return launch_decode_src(a, src, n, out, m, k, mr, static_weight, status, smem_limit, stream, num_sms);
}

cudaError_t launch_decode_stacked(const uint16_t* a, const DecodeSegs& segs, uint16_t* out, int m, int k, int mr,
                                  int static_weight, int* status, size_t smem_limit, cudaStream_t stream,
                                  int num_sms) {
  return launch_decode_src(a, segs, segs.off[segs.count], out, m, k, mr, static_weight, status, smem_limit, stream,
                           num_sms);
}

}  // namespace bsr
