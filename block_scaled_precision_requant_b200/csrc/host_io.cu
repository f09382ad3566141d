// Transfers between page-locked host memory (mapped into the device's address
// space) and device memory for the host-buffer decode entry: a kernel per
// direction instead of a DMA copy, launched with programmatic dependent
// launch so that it chains with the decode kernel the way consecutive decode
// steps chain with each other.  For the few KB a decode step moves, a DMA
// copy costs several microseconds of engine latency and ends the
// dependent-launch chain (the next kernel can no longer start its weight
// copies early); a one-CTA kernel costs one round trip over the host link.
#include <cstdint>

#include <cuda_runtime.h>

#include "kernels.h"

namespace bsr {

namespace {

// 16-byte vectors in a grid-stride loop, then the 2-byte tail (fewer than 8
// elements).  Plain loads: the source may be host memory, which the
// read-only data path is not used for here.
__global__ void __launch_bounds__(512) host_copy_kernel(const uint4* src, uint4* dst, long long n16,
                                                        const uint16_t* src_tail, uint16_t* dst_tail, int tail) {
  // Wait for the previous kernel on the stream (it may read dst or write
  // src), then let the next kernel be scheduled: it waits for this grid to
  // complete before it reads what this one writes.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) dst[i] = src[i];
  if (blockIdx.x == 0 && (int)threadIdx.x < tail) dst_tail[threadIdx.x] = src_tail[threadIdx.x];
}

}  // namespace

cudaError_t launch_host_copy(const void* src, void* dst, size_t bytes, cudaStream_t stream, int num_sms) {
  const long long n16 = (long long)(bytes / 16);
  const int tail = (int)((bytes % 16) / 2);
  long long grid = (n16 + 511) / 512;
  if (grid < 1) grid = 1;
  if (grid > num_sms) grid = num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(512);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint8_t* s = static_cast<const uint8_t*>(src);
  uint8_t* d = static_cast<uint8_t*>(dst);
  cudaError_t e = cudaLaunchKernelEx(&cfg, host_copy_kernel, reinterpret_cast<const uint4*>(s),
                                     reinterpret_cast<uint4*>(d), n16,
                                     reinterpret_cast<const uint16_t*>(s + (size_t)n16 * 16),
                                     reinterpret_cast<uint16_t*>(d + (size_t)n16 * 16), tail);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bsr
