// Descriptors of the W4A4 tensor-core GEMM (block-scaled FP4 MMA,
// `tcgen05.mma kind::mxf4nvf4`), host- and device-callable so that a host
// test can compare them with the values CUTLASS/CuTe derive for the same
// configuration.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define BSR_DESC_HD __host__ __device__ __forceinline__
#else
#define BSR_DESC_HD inline
#endif

namespace bsr {
namespace w4gemm {

// Instruction descriptor of the block-scaled FP4 MMA: A and B E2M1 (format 1
// of the FP4 kind), UE4M3 scales, both K-major, dense K = 64, scale ids 0.
BSR_DESC_HD constexpr uint32_t idesc_mxf4(int m, int n) {
  return (1u << 7)                        // A format: E2M1
         | (1u << 10)                     // B format: E2M1
         | ((uint32_t)(n >> 3) << 17)     // N / 8
         | (0u << 23)                     // scale format: UE4M3
         | ((uint32_t)(m >> 4) << 24);    // M / 16
}

// Shared-memory descriptor of a K-major, unswizzled source: 16-byte rows,
// 8-row core matrices 128 bytes apart (the tcgen05.cp source of one 512-byte
// scale atom); leading byte offset 16 (one core matrix along K).
BSR_DESC_HD uint64_t smem_desc_k_plain(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)(16u >> 4) << 16;            // leading byte offset
  d |= (uint64_t)(128u >> 4) << 32;           // stride byte offset: 8 rows x 16 B
  d |= (uint64_t)1 << 46;                     // descriptor version (sm_100)
  return d;                                   // layout type 0: no swizzle
}

}  // namespace w4gemm
}  // namespace bsr
