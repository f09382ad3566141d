// C ABI of libbsr.so: argument validation, tensor-map encoding, launches.
// Declarations and the contract of every entry point are in include/bsr.h.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "bsr.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// Device status word (one per device that loads the library); kernels get
// its address as an argument.
__device__ int g_dev_status = 0;

thread_local char g_err[512] = {0};

bsr_status fail(bsr_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

bsr_status ok() {
  g_err[0] = 0;
  return BSR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device properties, queried once per device.
struct DevInfo {
  int num_sms = 0;
  size_t smem_optin = 0;
  size_t smem_per_sm = 0;
  int cc_major = 0;
  int* status = nullptr;  // device address of g_dev_status
};

DevInfo g_dev[64];
std::mutex g_dev_mu;

bsr_status device_info(DevInfo& out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(BSR_ENODEV, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(BSR_ENODEV, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (d.num_sms == 0) {
    int sms = 0, smem = 0, smem_sm = 0, major = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return fail(BSR_ENODEV, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    void* st = nullptr;
    if ((e = cudaGetSymbolAddress(&st, g_dev_status)) != cudaSuccess)
      return fail(BSR_ENODEV, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    d.num_sms = sms;
    d.smem_optin = (size_t)smem;
    d.smem_per_sm = (size_t)smem_sm;
    d.cc_major = major;
    d.status = static_cast<int*>(st);
  }
  if (d.cc_major != 10) return fail(BSR_ENODEV, "device %d has compute capability %d.x, need 10.x (sm_100a)", dev, d.cc_major);
  out = d;
  return BSR_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
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

bsr_status encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw,
                     const char* what) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(BSR_ECUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSR_ECUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
  return BSR_OK;
}

bsr_status check_dims(int64_t m, int64_t n, int64_t k, bool need_m, bool need_n) {
  if ((need_m && (m < 0 || m > BSR_MAX_DIM)) || (need_n && (n < 0 || n > BSR_MAX_DIM)) || k < 0 ||
      k > BSR_MAX_DIM)
    return fail(BSR_EINVAL, "dimension out of range (m=%lld n=%lld k=%lld)", (long long)m, (long long)n,
                (long long)k);
  if (k == 0 || k % 32 != 0) return fail(BSR_ESHAPE, "K=%lld must be a positive multiple of 32", (long long)k);
  return BSR_OK;
}

bsr_status cuda_status(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(BSR_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  return ok();
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int64_t a_scale_ld(int64_t m) { return (m + 3) / 4 * 4; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Everything one GEMM launch needs, prepared -- and every check that can
// fail done -- before anything is queued.
struct GemmPlan {
  bsr::GemmMaps maps;
  DevInfo d;
  int m = 0, n = 0, k = 0, bm = 0;
  long long ldo = 0;
  int max_ctas = 0;
};

bsr_status gemm_plan(GemmPlan& p, const int8_t* a_i8, const float* a_scale_t, const int8_t* w_i8,
                     const float* w_scale, uint16_t* out, bool partials, int64_t m, int64_t n, int64_t k,
                     int64_t ldo = -1, int max_ctas = 0) {
  if (ldo < 0) ldo = n;
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (k % 128 != 0) return fail(BSR_ESHAPE, "bsr_gemm needs K %% 128 == 0 (K=%lld)", (long long)k);
  if (!a_i8 || !a_scale_t || !w_i8 || !w_scale || !out) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(a_i8) || !aligned16(a_scale_t) || !aligned16(w_i8) || !aligned16(w_scale) ||
      (reinterpret_cast<uintptr_t>(out) & 1u))
    return fail(BSR_EALIGN, "bsr_gemm: pointers must be 16-byte aligned (out: 2-byte)");
  if ((st = device_info(p.d)) != BSR_OK) return st;
  if (bsr::gemm_smem_bytes() > p.d.smem_optin)
    return fail(BSR_ENODEV, "device shared memory %zu < %zu", p.d.smem_optin, bsr::gemm_smem_bytes());
  const uint32_t bm = (uint32_t)bsr::gemm_block_m(m, n, p.d.num_sms);
  cudaError_t e = bsr::gemm_prepare_device(partials, (int)bm);
  if (e != cudaSuccess) return fail(BSR_ECUDA, "gemm shared-memory opt-in: %s", cudaGetErrorString(e));
  const int64_t nb = k / 32;
  if ((st = encode_2d(&p.maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_i8, k, n, k, bsr::kGemmBoxK, bsr::kGemmBoxW,
                      CU_TENSOR_MAP_SWIZZLE_128B, "w_i8")) != BSR_OK ||
      (st = encode_2d(&p.maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_i8, k, m, k, bsr::kGemmBoxK, bm,
                      CU_TENSOR_MAP_SWIZZLE_128B, "a_i8")) != BSR_OK ||
      (st = encode_2d(&p.maps.ws, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w_scale, nb, n, nb * 4, bsr::kGemmBoxKB,
                      bsr::kGemmBoxW, CU_TENSOR_MAP_SWIZZLE_NONE, "w_scale")) != BSR_OK ||
      (st = encode_2d(&p.maps.as, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a_scale_t, m, nb, a_scale_ld(m) * 4,
                      bm, bsr::kGemmBoxKB, CU_TENSOR_MAP_SWIZZLE_NONE, "a_scale_t")) != BSR_OK)
    return st;
  p.m = (int)m;
  p.n = (int)n;
  p.k = (int)k;
  p.bm = (int)bm;
  p.ldo = (long long)ldo;
  p.max_ctas = max_ctas;
  return BSR_OK;
}

bsr_status gemm_run(const GemmPlan& p, uint16_t* out, int32_t* partials, void* stream) {
  return cuda_status(bsr::launch_gemm(p.maps, out, partials, p.d.status, p.m, p.n, p.k, p.bm, p.ldo,
                                      as_stream(stream), p.d.num_sms, p.max_ctas),
                     "gemm launch");
}

bsr_status gemm_impl(const int8_t* a_i8, const float* a_scale_t, const int8_t* w_i8, const float* w_scale,
                     uint16_t* out, int32_t* partials, int64_t m, int64_t n, int64_t k, void* stream) {
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (k % 128 != 0) return fail(BSR_ESHAPE, "bsr_gemm needs K %% 128 == 0 (K=%lld)", (long long)k);
  if (m == 0 || n == 0) return ok();
  GemmPlan p;
  if ((st = gemm_plan(p, a_i8, a_scale_t, w_i8, w_scale, out, partials != nullptr, m, n, k)) != BSR_OK) return st;
  return gemm_run(p, out, partials, stream);
}

bsr_status decode_mr(int64_t m, int64_t k, DevInfo& d, int& mr) {
  bsr_status st;
  if ((st = device_info(d)) != BSR_OK) return st;
  mr = bsr::decode_rows_per_cta((int)m, (int)k, d.smem_optin);
  if (mr == 0) return fail(BSR_ESHAPE, "K=%lld too large for the decode kernel's shared memory", (long long)k);
  return BSR_OK;
}

bsr_status decode_segs_impl(const uint16_t* a, const bsr::DecodeSegs& segs, uint16_t* out, int64_t m, int64_t k,
                            void* stream, int static_weight) {
  DevInfo d;
  int mr = 0;
  bsr_status st = decode_mr(m, k, d, mr);
  if (st != BSR_OK) return st;
  return cuda_status(bsr::launch_decode_stacked(a, segs, out, (int)m, (int)k, mr, static_weight, d.status,
                                                d.smem_optin, as_stream(stream), d.num_sms),
                     "decode launch");
}

bsr_status decode_impl(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m,
                       int64_t n, int64_t k, void* stream, int static_weight = 0) {
  DevInfo d;
  int mr = 0;
  bsr_status st = decode_mr(m, k, d, mr);
  if (st != BSR_OK) return st;
  return cuda_status(bsr::launch_decode(a, w_i8, w_scale, out, (int)m, (int)n, (int)k, mr, static_weight, d.status,
                                        d.smem_optin, as_stream(stream), d.num_sms),
                     "decode launch");
}

static_assert(BSR_MAX_SEGMENTS == bsr::kMaxDecodeSegs, "segment table size");

// Side streams and events of the stacked tensor-core route, created once per
// device; the enqueue sequence that uses them runs under a lock.
struct StackedStreams {
  bool ready = false;
  cudaStream_t side[BSR_MAX_SEGMENTS] = {};
  cudaEvent_t fork = nullptr;
  cudaEvent_t join[BSR_MAX_SEGMENTS] = {};
};
StackedStreams g_stacked[64];
std::mutex g_stacked_mu;

bsr_status stacked_streams(int dev, StackedStreams*& out) {
  if (dev < 0 || dev >= 64) return fail(BSR_ENODEV, "device index %d out of range", dev);
  StackedStreams& ss = g_stacked[dev];
  if (!ss.ready) {
    cudaError_t e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
    for (int i = 0; e == cudaSuccess && i < BSR_MAX_SEGMENTS; ++i) {
      e = cudaStreamCreateWithFlags(&ss.side[i], cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.join[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return fail(BSR_ECUDA, "stacked side streams: %s", cudaGetErrorString(e));
    ss.ready = true;
  }
  out = &ss;
  return BSR_OK;
}

// Validates a stacked weight (host arrays of num_segs device pointers and
// row counts) and fills the decode segment table; total rows into n_total.
bsr_status stacked_segs(const int8_t* const* w_i8, const float* const* w_scale, const int64_t* n_segs,
                        int num_segs, bsr::DecodeSegs& segs, int64_t& n_total) {
  if (num_segs < 1 || num_segs > BSR_MAX_SEGMENTS)
    return fail(BSR_EINVAL, "num_segs %d not in [1, %d]", num_segs, BSR_MAX_SEGMENTS);
  if (!w_i8 || !w_scale || !n_segs) return fail(BSR_EINVAL, "null segment array");
  segs = {};
  segs.count = num_segs;
  n_total = 0;
  for (int s = 0; s < num_segs; ++s) {
    if (n_segs[s] < 0) return fail(BSR_EINVAL, "segment %d: negative row count", s);
    if (n_segs[s] > 0 && (!w_i8[s] || !w_scale[s])) return fail(BSR_EINVAL, "segment %d: null pointer", s);
    if (!aligned16(w_i8[s]) || !aligned16(w_scale[s]))
      return fail(BSR_EALIGN, "segment %d: pointers must be 16-byte aligned", s);
    segs.off[s] = (int)n_total;
    segs.w[s] = w_i8[s];
    segs.ws[s] = w_scale[s];
    n_total += n_segs[s];
    if (n_total > 2147483647LL) return fail(BSR_EINVAL, "stacked rows exceed 2^31 - 1");
  }
  segs.off[num_segs] = (int)n_total;
  return BSR_OK;
}

bsr_status check_proj_args(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out) {
  if (!a || !w_i8 || !w_scale || !out) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(a) || !aligned16(w_i8) || !aligned16(w_scale) || (reinterpret_cast<uintptr_t>(out) & 1u))
    return fail(BSR_EALIGN, "a, w_i8, w_scale must be 16-byte aligned, out 2-byte aligned");
  return BSR_OK;
}

}  // namespace

namespace bsr {
// Device address of the library's status word on the current device (the
// word bsr_device_status() reads and clears).
bsr_status library_status_word(int** out) {
  DevInfo d;
  const bsr_status st = device_info(d);
  if (st != BSR_OK) return st;
  *out = d.status;
  return BSR_OK;
}

bsr_status report(bsr_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}
}  // namespace bsr

extern "C" {

int bsr_abi_version(void) { return BSR_ABI_VERSION; }

const char* bsr_last_error(void) { return g_err; }

int bsr_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(int)) != cudaSuccess) return -1;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_dev_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

bsr_status bsr_requant_w(const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2, int8_t* w_i8,
                         float* w_scale, int64_t n, int64_t k, void* stream) {
  bsr_status st = check_dims(0, n, k, false, true);
  if (st != BSR_OK) return st;
  if (n == 0) return ok();
  if (!w_packed || !w_e4m3 || !w_i8 || !w_scale) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(w_packed) || !aligned16(w_e4m3) || !aligned16(w_i8) || !aligned16(w_scale))
    return fail(BSR_EALIGN, "bsr_requant_w: pointers must be 16-byte aligned");
  DevInfo d;
  if ((st = device_info(d)) != BSR_OK) return st;
  return cuda_status(bsr::launch_requant_w(w_packed, w_e4m3, scale2, w_i8, w_scale, n, k, as_stream(stream),
                                           d.num_sms),
                     "requant_w launch");
}

int64_t bsr_a_scale_ld(int64_t m) { return m < 0 ? 0 : a_scale_ld(m); }

bsr_status bsr_requant_a(const uint16_t* a, int8_t* a_i8, float* a_scale_t, int64_t m, int64_t k, void* stream) {
  bsr_status st = check_dims(m, 0, k, true, false);
  if (st != BSR_OK) return st;
  if (m == 0) return ok();
  if (!a || !a_i8 || !a_scale_t) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(a) || !aligned16(a_i8) || !aligned16(a_scale_t))
    return fail(BSR_EALIGN, "bsr_requant_a: pointers must be 16-byte aligned");
  DevInfo d;
  if ((st = device_info(d)) != BSR_OK) return st;
  return cuda_status(bsr::launch_requant_a(a, a_i8, a_scale_t, (int)m, (int)k, (int)a_scale_ld(m),
                                           as_stream(stream), d.num_sms),
                     "requant_a launch");
}

bsr_status bsr_gemm(const int8_t* a_i8, const float* a_scale_t, const int8_t* w_i8, const float* w_scale,
                    uint16_t* out, int64_t m, int64_t n, int64_t k, void* stream) {
  return gemm_impl(a_i8, a_scale_t, w_i8, w_scale, out, nullptr, m, n, k, stream);
}

bsr_status bsr_gemm_partials(const int8_t* a_i8, const float* a_scale_t, const int8_t* w_i8, const float* w_scale,
                             uint16_t* out, int32_t* partials, int64_t m, int64_t n, int64_t k, void* stream) {
  if (!partials) return fail(BSR_EINVAL, "null partials");
  return gemm_impl(a_i8, a_scale_t, w_i8, w_scale, out, partials, m, n, k, stream);
}

int bsr_gemm_block_m(int64_t m, int64_t n) {
  if (m < 1 || n < 1 || m > BSR_MAX_DIM || n > BSR_MAX_DIM) return 0;
  DevInfo d;
  if (device_info(d) != BSR_OK) return 0;
  return bsr::gemm_block_m(m, n, d.num_sms);
}

size_t bsr_proj_scratch_bytes(int64_t m, int64_t k) {
  if (m <= BSR_DECODE_MAX_M || k <= 0 || k % 128 != 0) return 0;
  return align256((size_t)m * (size_t)k) + (size_t)(k / 32) * (size_t)a_scale_ld(m) * 4;
}

bsr_status bsr_debug_wait_timeout(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000) return fail(BSR_EINVAL, "bsr_debug_wait_timeout: limit_ms %d not in [1, 2000]", limit_ms);
  DevInfo d;
  bsr_status st = device_info(d);
  if (st != BSR_OK) return st;
  return cuda_status(bsr::launch_debug_wait(d.status, (unsigned long long)limit_ms * 1000000ull, as_stream(stream)),
                     "debug wait launch");
}

bsr_status bsr_decode(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m,
                      int64_t n, int64_t k, void* stream) {
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (m == 0 || n == 0) return ok();
  if ((st = check_proj_args(a, w_i8, w_scale, out)) != BSR_OK) return st;
  return decode_impl(a, w_i8, w_scale, out, m, n, k, stream);
}

bsr_status bsr_decode_ex(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m,
                         int64_t n, int64_t k, unsigned flags, void* stream) {
  if (flags & ~(unsigned)BSR_DECODE_STATIC_WEIGHT) return fail(BSR_EINVAL, "bsr_decode_ex: unknown flags 0x%x", flags);
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (m == 0 || n == 0) return ok();
  if ((st = check_proj_args(a, w_i8, w_scale, out)) != BSR_OK) return st;
  return decode_impl(a, w_i8, w_scale, out, m, n, k, stream, (flags & BSR_DECODE_STATIC_WEIGHT) ? 1 : 0);
}

// The device address of a page-locked host buffer mapped into the current
// device's address space; nullptr when `p` is not one.
static const void* mapped_host(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr) return nullptr;
  return at.devicePointer;
}

bsr_status bsr_decode_host(const uint16_t* a_host, const int8_t* w_i8, const float* w_scale, uint16_t* out_host,
                           int64_t m, int64_t n, int64_t k, uint16_t* a_dev, uint16_t* out_dev, unsigned flags,
                           void* stream) {
  if (flags & ~(unsigned)BSR_DECODE_STATIC_WEIGHT)
    return fail(BSR_EINVAL, "bsr_decode_host: unknown flags 0x%x", flags);
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (m == 0 || n == 0) return ok();
  if (!a_host || !out_host) return fail(BSR_EINVAL, "null pointer");
  if ((st = check_proj_args(a_dev, w_i8, w_scale, out_dev)) != BSR_OK) return st;
  if (!aligned16(a_host) || !aligned16(out_host) || !aligned16(out_dev))
    return fail(BSR_EALIGN, "bsr_decode_host: a_host, out_host, a_dev, out_dev must be 16-byte aligned");
  DevInfo d;
  int mr = 0;
  if ((st = decode_mr(m, k, d, mr)) != BSR_OK) return st;
  const void* a_map = mapped_host(a_host);
  void* out_map = const_cast<void*>(mapped_host(out_host));
  if (!a_map || !out_map)
    return fail(BSR_EINVAL, "bsr_decode_host: a_host and out_host must be page-locked host memory mapped into "
                            "the device's address space");
  // the decode launch's configuration before anything is queued
  if ((st = cuda_status(bsr::prepare_decode((int)n, (int)k, mr, d.smem_optin, d.num_sms), "decode setup")) != BSR_OK)
    return st;
  cudaStream_t cs = as_stream(stream);
  if ((st = cuda_status(bsr::launch_host_copy(a_map, a_dev, (size_t)m * (size_t)k * 2, cs, d.num_sms),
                        "input copy launch")) != BSR_OK)
    return st;
  if ((st = cuda_status(bsr::launch_decode(a_dev, w_i8, w_scale, out_dev, (int)m, (int)n, (int)k, mr,
                                           (flags & BSR_DECODE_STATIC_WEIGHT) ? 1 : 0, d.status, d.smem_optin, cs,
                                           d.num_sms),
                        "decode launch")) != BSR_OK)
    return st;
  return cuda_status(bsr::launch_host_copy(out_dev, out_map, (size_t)m * (size_t)n * 2, cs, d.num_sms),
                     "output copy launch");
}

// Copy streams and events of the host-buffer projection, created once per
// device; the enqueue sequence that uses them runs under a lock.
static constexpr int kMaxHostChunks = 64;
struct HostPipe {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaEvent_t in[kMaxHostChunks] = {}, done[kMaxHostChunks] = {};
};
static HostPipe g_host_pipe[64];
static std::mutex g_host_pipe_mu;

static bsr_status host_pipe(int dev, HostPipe*& out) {
  if (dev < 0 || dev >= 64) return fail(BSR_ENODEV, "device index %d out of range", dev);
  HostPipe& hp = g_host_pipe[dev];
  if (!hp.ready) {
    cudaError_t e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.join, cudaEventDisableTiming);
    for (int i = 0; e == cudaSuccess && i < kMaxHostChunks; ++i) {
      e = cudaEventCreateWithFlags(&hp.in[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.done[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return fail(BSR_ECUDA, "host-buffer projection streams: %s", cudaGetErrorString(e));
    hp.ready = true;
  }
  out = &hp;
  return BSR_OK;
}

static bool is_pinned_host(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeHost;
}

static int64_t host_chunk_rows(int64_t m, int64_t chunk_rows) {
  if (chunk_rows <= 0) {
    // about four chunks, whole 128-row tiles, at least 512 rows
    chunk_rows = (m + 3) / 4;
    chunk_rows = (chunk_rows + 127) / 128 * 128;
    if (chunk_rows < 512) chunk_rows = 512;
  }
  const int64_t min_rows = (m + kMaxHostChunks - 1) / kMaxHostChunks;
  if (chunk_rows < min_rows) chunk_rows = min_rows;
  return chunk_rows > m ? m : chunk_rows;
}

bsr_status bsr_proj(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m, int64_t n,
                    int64_t k, void* scratch, size_t scratch_bytes, void* stream) {
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (m == 0 || n == 0) return ok();
  if ((st = check_proj_args(a, w_i8, w_scale, out)) != BSR_OK) return st;
  if (m <= BSR_DECODE_MAX_M || k % 128 != 0) return decode_impl(a, w_i8, w_scale, out, m, n, k, stream);
  const size_t need = bsr_proj_scratch_bytes(m, k);
  if (!scratch || scratch_bytes < need)
    return fail(BSR_ESCRATCH, "scratch of %zu bytes needed, %zu given", need, scratch ? scratch_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return fail(BSR_EALIGN, "scratch must be 256-byte aligned");
  int8_t* a_i8 = static_cast<int8_t*>(scratch);
  float* a_scale_t = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + align256((size_t)m * (size_t)k));
  // plan the GEMM (tensor maps, shared-memory opt-in) before the first launch
  GemmPlan p;
  if ((st = gemm_plan(p, a_i8, a_scale_t, w_i8, w_scale, out, false, m, n, k)) != BSR_OK) return st;
  if ((st = cuda_status(bsr::launch_requant_a(a, a_i8, a_scale_t, (int)m, (int)k, (int)a_scale_ld(m),
                                              as_stream(stream), p.d.num_sms),
                        "requant_a launch")) != BSR_OK)
    return st;
  return gemm_run(p, out, nullptr, stream);
}

int64_t bsr_proj_host_scratch_bytes(int64_t m, int64_t k, int64_t chunk_rows) {
  if (m <= 0 || k <= 0) return 0;
  return (int64_t)bsr_proj_scratch_bytes(host_chunk_rows(m, chunk_rows), k);
}

bsr_status bsr_proj_host(const uint16_t* a_host, const int8_t* w_i8, const float* w_scale, uint16_t* out_host,
                         int64_t m, int64_t n, int64_t k, uint16_t* a_dev, uint16_t* out_dev, void* scratch,
                         size_t scratch_bytes, int64_t chunk_rows, void* stream) {
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (chunk_rows < 0) return fail(BSR_EINVAL, "bsr_proj_host: chunk_rows %lld < 0", (long long)chunk_rows);
  if (m == 0 || n == 0) return ok();
  if (!a_host || !out_host) return fail(BSR_EINVAL, "null pointer");
  if ((st = check_proj_args(a_dev, w_i8, w_scale, out_dev)) != BSR_OK) return st;
  const int64_t rows = host_chunk_rows(m, chunk_rows);
  const int chunks = (int)((m + rows - 1) / rows);
  const size_t need = bsr_proj_scratch_bytes(rows, k);
  if (need && (!scratch || scratch_bytes < need))
    return fail(BSR_ESCRATCH, "scratch of %zu bytes needed, %zu given", need, scratch ? scratch_bytes : (size_t)0);
  if (need && (reinterpret_cast<uintptr_t>(scratch) & 255u) != 0)
    return fail(BSR_EALIGN, "scratch must be 256-byte aligned");
  if (!is_pinned_host(a_host) || !is_pinned_host(out_host))
    return fail(BSR_EINVAL, "bsr_proj_host: a_host and out_host must be page-locked host memory");
  DevInfo d;
  if ((st = device_info(d)) != BSR_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(BSR_ENODEV, "cudaGetDevice failed");
  // every chunk's launch prepared before anything is queued: the GEMM plan
  // (tensor maps, opt-in) of a tensor-core chunk, the decode setup of a
  // chunk the decode kernel serves (at most 16 rows, or K % 128 != 0)
  std::vector<GemmPlan> plans((size_t)chunks);
  std::vector<int> dec_mr((size_t)chunks, 0);
  int8_t* a_i8 = static_cast<int8_t*>(scratch);
  for (int c = 0; c < chunks; ++c) {
    const int64_t r0 = (int64_t)c * rows, mc = (m - r0 < rows) ? m - r0 : rows;
    if (mc <= BSR_DECODE_MAX_M || k % 128 != 0) {
      DevInfo dd;
      if ((st = decode_mr(mc, k, dd, dec_mr[c])) != BSR_OK) return st;
      if ((st = cuda_status(bsr::prepare_decode((int)n, (int)k, dec_mr[c], dd.smem_optin, dd.num_sms),
                            "decode setup")) != BSR_OK)
        return st;
    } else {
      float* a_st = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + align256((size_t)mc * (size_t)k));
      if ((st = gemm_plan(plans[c], a_i8, a_st, w_i8, w_scale, out_dev + r0 * n, false, mc, n, k)) != BSR_OK)
        return st;
    }
  }
  std::lock_guard<std::mutex> lk(g_host_pipe_mu);
  HostPipe* hp = nullptr;
  if ((st = host_pipe(dev, hp)) != BSR_OK) return st;
  cudaStream_t cs = as_stream(stream);
  // the copy streams start after the work already queued on `stream`
  if (cudaEventRecord(hp->fork, cs) != cudaSuccess || cudaStreamWaitEvent(hp->h2d, hp->fork, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->d2h, hp->fork, 0) != cudaSuccess)
    return fail(BSR_ECUDA, "host-buffer projection fork failed");
  for (int c = 0; c < chunks; ++c) {
    const int64_t r0 = (int64_t)c * rows, mc = (m - r0 < rows) ? m - r0 : rows;
    if (cudaMemcpyAsync(a_dev + r0 * k, a_host + r0 * k, (size_t)(mc * k) * 2, cudaMemcpyHostToDevice, hp->h2d) !=
            cudaSuccess ||
        cudaEventRecord(hp->in[c], hp->h2d) != cudaSuccess || cudaStreamWaitEvent(cs, hp->in[c], 0) != cudaSuccess)
      return fail(BSR_ECUDA, "host-buffer projection: input copy of chunk %d failed", c);
    if (dec_mr[c]) {
      if ((st = cuda_status(bsr::launch_decode(a_dev + r0 * k, w_i8, w_scale, out_dev + r0 * n, (int)mc, (int)n,
                                               (int)k, dec_mr[c], 0, d.status, d.smem_optin, cs, d.num_sms),
                            "decode launch")) != BSR_OK)
        return st;
    } else {
      float* a_st = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + align256((size_t)mc * (size_t)k));
      if ((st = cuda_status(bsr::launch_requant_a(a_dev + r0 * k, a_i8, a_st, (int)mc, (int)k, (int)a_scale_ld(mc),
                                                  cs, d.num_sms),
                            "requant_a launch")) != BSR_OK ||
          (st = gemm_run(plans[c], out_dev + r0 * n, nullptr, cs)) != BSR_OK)
        return st;
    }
    if (cudaEventRecord(hp->done[c], cs) != cudaSuccess || cudaStreamWaitEvent(hp->d2h, hp->done[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(out_host + r0 * n, out_dev + r0 * n, (size_t)(mc * n) * 2, cudaMemcpyDeviceToHost,
                        hp->d2h) != cudaSuccess)
      return fail(BSR_ECUDA, "host-buffer projection: output copy of chunk %d failed", c);
  }
  // `stream` passes this call once the last output copy has landed
  if (cudaEventRecord(hp->join, hp->d2h) != cudaSuccess || cudaStreamWaitEvent(cs, hp->join, 0) != cudaSuccess)
    return fail(BSR_ECUDA, "host-buffer projection join failed");
  return ok();
}

bsr_status bsr_silu_mul(const uint16_t* gate, const uint16_t* up, uint16_t* x, int64_t m, int64_t k, void* stream) {
  bsr_status st = check_dims(m, 0, k, true, false);
  if (st != BSR_OK) return st;
  if (m == 0) return ok();
  if (!gate || !up || !x) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(gate) || !aligned16(up) || !aligned16(x))
    return fail(BSR_EALIGN, "bsr_silu_mul: pointers must be 16-byte aligned");
  DevInfo d;
  if ((st = device_info(d)) != BSR_OK) return st;
  return cuda_status(bsr::launch_silu_mul(gate, up, x, (int)m, (int)k, as_stream(stream), d.num_sms),
                     "silu_mul launch");
}

bsr_status bsr_requant_silu_a(const uint16_t* gate, const uint16_t* up, int8_t* a_i8, float* a_scale_t, int64_t m,
                              int64_t k, void* stream) {
  bsr_status st = check_dims(m, 0, k, true, false);
  if (st != BSR_OK) return st;
  if (m == 0) return ok();
  if (!gate || !up || !a_i8 || !a_scale_t) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(gate) || !aligned16(up) || !aligned16(a_i8) || !aligned16(a_scale_t))
    return fail(BSR_EALIGN, "bsr_requant_silu_a: pointers must be 16-byte aligned");
  DevInfo d;
  if ((st = device_info(d)) != BSR_OK) return st;
  return cuda_status(bsr::launch_requant_silu_a(gate, up, a_i8, a_scale_t, (int)m, (int)k, (int)a_scale_ld(m),
                                                as_stream(stream), d.num_sms),
                     "requant_silu_a launch");
}

size_t bsr_proj_silu_scratch_bytes(int64_t m, int64_t k) {
  if (m <= 0 || k <= 0 || k % 32 != 0) return 0;
  if (m <= BSR_DECODE_MAX_M || k % 128 != 0) return align256((size_t)m * (size_t)k * 2);  // BF16 product
  return bsr_proj_scratch_bytes(m, k);
}

bsr_status bsr_proj_silu(const uint16_t* gate, const uint16_t* up, const int8_t* w_i8, const float* w_scale,
                         uint16_t* out, int64_t m, int64_t n, int64_t k, void* scratch, size_t scratch_bytes,
                         void* stream) {
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (m == 0 || n == 0) return ok();
  if ((st = check_proj_args(gate, w_i8, w_scale, out)) != BSR_OK) return st;
  if (!up) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(up)) return fail(BSR_EALIGN, "bsr_proj_silu: pointers must be 16-byte aligned");
  const size_t need = bsr_proj_silu_scratch_bytes(m, k);
  if (!scratch || scratch_bytes < need)
    return fail(BSR_ESCRATCH, "scratch of %zu bytes needed, %zu given", need, scratch ? scratch_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return fail(BSR_EALIGN, "scratch must be 256-byte aligned");
  if (m <= BSR_DECODE_MAX_M || k % 128 != 0) {
    // decode route: the BF16 product into scratch, then the decode kernel
    // (its shared-memory fit is checked before the first launch)
    uint16_t* x = static_cast<uint16_t*>(scratch);
    DevInfo d;
    int mr = 0;
    if ((st = decode_mr(m, k, d, mr)) != BSR_OK) return st;
    if ((st = cuda_status(bsr::launch_silu_mul(gate, up, x, (int)m, (int)k, as_stream(stream), d.num_sms),
                          "silu_mul launch")) != BSR_OK)
      return st;
    return decode_impl(x, w_i8, w_scale, out, m, n, k, stream);
  }
  int8_t* a_i8 = static_cast<int8_t*>(scratch);
  float* a_scale_t = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + align256((size_t)m * (size_t)k));
  GemmPlan p;
  if ((st = gemm_plan(p, a_i8, a_scale_t, w_i8, w_scale, out, false, m, n, k)) != BSR_OK) return st;
  if ((st = cuda_status(bsr::launch_requant_silu_a(gate, up, a_i8, a_scale_t, (int)m, (int)k, (int)a_scale_ld(m),
                                                   as_stream(stream), p.d.num_sms),
                        "requant_silu_a launch")) != BSR_OK)
    return st;
  return gemm_run(p, out, nullptr, stream);
}

bsr_status bsr_decode_stacked(const uint16_t* a, const int8_t* const* w_i8, const float* const* w_scale,
                              const int64_t* n_segs, int num_segs, uint16_t* out, int64_t m, int64_t k, unsigned flags,
                              void* stream) {
  if (flags & ~(unsigned)BSR_DECODE_STATIC_WEIGHT)
    return fail(BSR_EINVAL, "bsr_decode_stacked: unknown flags 0x%x", flags);
  bsr::DecodeSegs segs;
  int64_t n = 0;
  bsr_status st = stacked_segs(w_i8, w_scale, n_segs, num_segs, segs, n);
  if (st != BSR_OK) return st;
  if ((st = check_dims(m, n, k, true, true)) != BSR_OK) return st;
  if (m == 0 || n == 0) return ok();
  if (!a || !out) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(a) || (reinterpret_cast<uintptr_t>(out) & 1u))
    return fail(BSR_EALIGN, "a must be 16-byte aligned, out 2-byte aligned");
  return decode_segs_impl(a, segs, out, m, k, stream, (flags & BSR_DECODE_STATIC_WEIGHT) ? 1 : 0);
}

bsr_status bsr_proj_stacked(const uint16_t* a, const int8_t* const* w_i8, const float* const* w_scale,
                            const int64_t* n_segs, int num_segs, uint16_t* out, int64_t m, int64_t k, void* scratch,
                            size_t scratch_bytes, void* stream) {
  bsr::DecodeSegs segs;
  int64_t n = 0;
  bsr_status st = stacked_segs(w_i8, w_scale, n_segs, num_segs, segs, n);
  if (st != BSR_OK) return st;
  if ((st = check_dims(m, n, k, true, true)) != BSR_OK) return st;
  if (m == 0 || n == 0) return ok();
  if (!a || !out) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(a) || (reinterpret_cast<uintptr_t>(out) & 1u))
    return fail(BSR_EALIGN, "a must be 16-byte aligned, out 2-byte aligned");
  if (m <= BSR_DECODE_MAX_M || k % 128 != 0) return decode_segs_impl(a, segs, out, m, k, stream, 0);
  const size_t need = bsr_proj_scratch_bytes(m, k);
  if (!scratch || scratch_bytes < need)
    return fail(BSR_ESCRATCH, "scratch of %zu bytes needed, %zu given", need, scratch ? scratch_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return fail(BSR_EALIGN, "scratch must be 256-byte aligned");
  int8_t* a_i8 = static_cast<int8_t*>(scratch);
  float* a_scale_t = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + align256((size_t)m * (size_t)k));
  // One GEMM per segment into its column slice of out (row stride = all
  // rows).  The segments run concurrently, each on a side stream forked from
  // and joined back into the caller's stream, with persistent grids sized in
  // proportion to their tile counts so that together they fill the SMs once
  // (a small segment alone would leave most SMs idle).  Every segment's plan
  // and the side streams are made before the first launch.
  DevInfo d;
  if ((st = device_info(d)) != BSR_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(BSR_ENODEV, "cudaGetDevice failed");
  long long tiles[BSR_MAX_SEGMENTS] = {}, total_tiles = 0;
  for (int s = 0; s < num_segs; ++s) {
    const int64_t ns = segs.off[s + 1] - segs.off[s];
    tiles[s] = bsr::gemm_tiles(m, ns, d.num_sms);
    total_tiles += tiles[s];
  }
  GemmPlan plans[BSR_MAX_SEGMENTS];
  for (int s = 0; s < num_segs; ++s) {
    if (tiles[s] == 0) continue;
    int ctas = (int)((long long)d.num_sms * tiles[s] / total_tiles);
    ctas = ctas < 1 ? 1 : ctas;
    const int64_t ns = segs.off[s + 1] - segs.off[s];
    if ((st = gemm_plan(plans[s], a_i8, a_scale_t, w_i8[s], w_scale[s], out + segs.off[s], false, m, ns, k, n,
                        ctas)) != BSR_OK)
      return st;
  }
  std::lock_guard<std::mutex> lk(g_stacked_mu);
  StackedStreams* ss = nullptr;
  if ((st = stacked_streams(dev, ss)) != BSR_OK) return st;
  cudaStream_t cs = as_stream(stream);
  if ((st = cuda_status(bsr::launch_requant_a(a, a_i8, a_scale_t, (int)m, (int)k, (int)a_scale_ld(m), cs,
                                              d.num_sms),
                        "requant_a launch")) != BSR_OK)
    return st;
  if (cudaEventRecord(ss->fork, cs) != cudaSuccess) return fail(BSR_ECUDA, "stacked fork record failed");
  for (int s = 0; s < num_segs; ++s) {
    if (tiles[s] == 0) continue;
    if (cudaStreamWaitEvent(ss->side[s], ss->fork, 0) != cudaSuccess) return fail(BSR_ECUDA, "stacked fork wait failed");
    if ((st = gemm_run(plans[s], out + segs.off[s], nullptr, ss->side[s])) != BSR_OK) return st;
    if (cudaEventRecord(ss->join[s], ss->side[s]) != cudaSuccess) return fail(BSR_ECUDA, "stacked join record failed");
    if (cudaStreamWaitEvent(cs, ss->join[s], 0) != cudaSuccess) return fail(BSR_ECUDA, "stacked join wait failed");
  }
  return ok();
}

bsr_status bsr_w4a16_decode_ex(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                               uint16_t* out, int64_t m, int64_t n, int64_t k, unsigned flags, void* stream) {
  bsr_status st = check_dims(m, n, k, true, true);
  if (st != BSR_OK) return st;
  if (flags & ~BSR_DECODE_STATIC_WEIGHT) return fail(BSR_EINVAL, "unknown flags 0x%x", flags);
  if (m == 0 || n == 0) return ok();
  if (!a || !w_packed || !w_e4m3 || !out) return fail(BSR_EINVAL, "null pointer");
  if (!aligned16(a) || !aligned16(w_packed) || !aligned16(w_e4m3) || (reinterpret_cast<uintptr_t>(out) & 1u))
    return fail(BSR_EALIGN, "a, w_packed, w_e4m3 must be 16-byte aligned, out 2-byte aligned");
  DevInfo d;
  if ((st = device_info(d)) != BSR_OK) return st;
  bsr::GemvPlan p;
  if (!bsr::nvfp4_gemv_plan((int)m, (int)n, (int)k, false, d.smem_optin, d.smem_per_sm, d.num_sms, p))
    return fail(BSR_ESHAPE, "K=%lld, M=%lld outside the NVFP4 GEMV (K <= 65536 with one activation row and one weight stage in shared memory)",
                (long long)k, (long long)m);
  return cuda_status(bsr::launch_nvfp4_gemv(p, false, a, w_packed, w_e4m3, scale2, out, (int)m, (int)n, (int)k,
                                            (flags & BSR_DECODE_STATIC_WEIGHT) ? 1 : 0, d.status, as_stream(stream)),
                     "w4a16 decode launch");
}

bsr_status bsr_w4a16_decode(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                            uint16_t* out, int64_t m, int64_t n, int64_t k, void* stream) {
  return bsr_w4a16_decode_ex(a, w_packed, w_e4m3, scale2, out, m, n, k, 0u, stream);
}

}  // extern "C"
