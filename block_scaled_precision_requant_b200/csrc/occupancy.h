// Host-side launch helper of the grid-stride kernels (requant, SiLU).
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace bsr {

// CTAs of `kernel` (launched with `threads` threads, no dynamic shared
// memory) that one SM holds at once, from the occupancy calculator, cached
// per kernel and device; 1 if the query fails.  Grid-stride kernels size
// their grids to SMs x this, so that all their CTAs run in one wave.
inline int resident_ctas_per_sm(const void* kernel, int threads) {
  struct Entry {
    const void* k;
    int dev, blocks;
  };
  static Entry cache[64];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].k == kernel && cache[i].dev == dev) return cache[i].blocks;
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, 0) != cudaSuccess || b < 1) b = 1;
  if (used < 64) cache[used++] = Entry{kernel, dev, b};
  return b;
}

}  // namespace bsr
