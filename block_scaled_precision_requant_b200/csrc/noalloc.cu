// bsr_proj_noalloc: bsr_proj with its scratch built into the library.
//
// Some callers cannot allocate device memory when they run the projection:
// an inference runtime that plans all of its device memory up front and
// hands kernels only their inputs and outputs, or code running where
// cudaMalloc is not allowed (it synchronises the device, which a serving hot
// path cannot afford).  For them the activation codes and block scales that
// bsr_proj keeps in caller scratch live in one fixed array in this file.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds BSR_NOALLOC_SCRATCH_BYTES of device memory for it until the
// process exits.  Host code cannot use the array's name as a device address
// (it names a host-side stand-in), so the device address is looked up once
// per device with cudaGetSymbolAddress, with that device current, on the
// first call made on it; that first call should happen before any stream
// capture begins.  All calls share the one array and each call overwrites
// it: calls whose kernels may overlap on the GPU (different streams, or
// several host threads) race on it and must be serialised by the caller.
// Nothing in the array needs to start at zero: every byte the GEMM reads is
// written by the same call's activation requantisation first.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "bsr.h"

namespace bsr {
// Records the message bsr_last_error() returns on this thread (api.cu).
bsr_status report(bsr_status st, const char* fmt, ...);
}  // namespace bsr

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[BSR_NOALLOC_SCRATCH_BYTES];

void* g_scratch_addr[64] = {nullptr};
std::mutex g_scratch_mu;

}  // namespace

extern "C" bsr_status bsr_proj_noalloc(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out,
                                       int64_t m, int64_t n, int64_t k, void* stream) {
  const size_t need = bsr_proj_scratch_bytes(m, k);
  if (need == 0) {
    // decode path (or K % 128 != 0): bsr_proj needs no scratch at all
    return bsr_proj(a, w_i8, w_scale, out, m, n, k, nullptr, 0, stream);
  }
  if (need > (size_t)BSR_NOALLOC_SCRATCH_BYTES)
    return bsr::report(BSR_ESCRATCH,
                       "bsr_proj_noalloc: M=%lld K=%lld needs %zu bytes of activation scratch; the built-in array "
                       "holds %zu (BSR_NOALLOC_SCRATCH_BYTES): use bsr_proj with caller scratch",
                       (long long)m, (long long)k, need, (size_t)BSR_NOALLOC_SCRATCH_BYTES);
  int dev = 0;
  const cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) return bsr::report(BSR_ENODEV, "cudaGetDevice: %s", cudaGetErrorString(de));
  if (dev < 0 || dev >= 64) return bsr::report(BSR_ENODEV, "device index %d out of range", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr)
        return bsr::report(BSR_ECUDA, "cudaGetSymbolAddress(scratch array): %s", cudaGetErrorString(e));
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return bsr_proj(a, w_i8, w_scale, out, m, n, k, scratch, (size_t)BSR_NOALLOC_SCRATCH_BYTES, stream);
}
