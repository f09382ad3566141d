// Internal launch interface between the C-ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace bsr {

// Tensor maps of one GEMM launch.  BM = gemm_block_m(M, N, SMs) activation
// rows per tile (128, 192 or 256), 128 weight rows, 4 K blocks per stage.
struct GemmMaps {
  CUtensorMap w;   // W_i8 [N, K] int8, box 128 rows x 128 B, 128-byte swizzle
  CUtensorMap a;   // a_i8 [M, K] int8, box BM rows x 128 B, 128-byte swizzle
  CUtensorMap ws;  // W_scale [N, K/32] f32, box 128 rows x 4
  CUtensorMap as;  // a_scale_t [K/32, ld] f32 (dims K/32 x M), box 4 rows x BM
};
constexpr int kGemmBoxK = 128;  // bytes of K per stage
constexpr int kGemmBoxW = 128;  // weight rows per tile
constexpr int kGemmBoxKB = 4;   // 32-blocks per stage
int gemm_block_m(long long m, long long n, int num_sms);
long long gemm_tiles(long long m, long long n, int num_sms);

cudaError_t launch_requant_w(const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2, int8_t* w_i8,
                             float* w_scale, long long n, long long k, cudaStream_t stream, int num_sms);
cudaError_t launch_requant_a(const uint16_t* a, int8_t* a_i8, float* a_scale_t, int m, int k, int ld,
                             cudaStream_t stream, int num_sms);
// Weight segments of one decode launch: output column r (global row of the
// stacked weight) belongs to the segment s with off[s] <= r < off[s + 1] and
// reads row r - off[s] of that segment's own codes and scales.
constexpr int kMaxDecodeSegs = 8;
struct DecodeSegs {
  int count;
  int off[kMaxDecodeSegs + 1];
  const int8_t* w[kMaxDecodeSegs];
  const float* ws[kMaxDecodeSegs];
};

int decode_rows_per_cta(int m, int k, size_t smem_limit);
// The decode launch's configuration and shared-memory opt-in for a single
// weight, made ahead of any launch (the launch itself repeats it, cached).
cudaError_t prepare_decode(int n, int k, int mr, size_t smem_limit, int num_sms);
// Copy of `bytes` (even) from src to dst by one or more CTAs, launched with
// programmatic dependent launch; either side may be device-mapped host
// memory.  Both pointers 16-byte aligned.
cudaError_t launch_host_copy(const void* src, void* dst, size_t bytes, cudaStream_t stream, int num_sms);
cudaError_t launch_decode(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int m, int n,
                          int k, int mr, int static_weight, int* status, size_t smem_limit, cudaStream_t stream,
                          int num_sms);
cudaError_t launch_decode_stacked(const uint16_t* a, const DecodeSegs& segs, uint16_t* out, int m, int k, int mr,
                                  int static_weight, int* status, size_t smem_limit, cudaStream_t stream,
                                  int num_sms);
size_t gemm_smem_bytes();
// Shared-memory opt-in of the kernel variant with tile width bm (with or
// without the partials dump), once per device, thread-safe.  Fails if the
// kernel was not built with the register count its register split assumes.
cudaError_t gemm_prepare_device(bool partials, int bm);
// out row stride ldo (elements) >= n: the output may be a column slice of a
// wider matrix.  max_ctas > 0 caps the persistent grid (to share the GPU
// between concurrent launches).
cudaError_t launch_gemm(const GemmMaps& maps, uint16_t* out, int32_t* partials, int* status, int m, int n, int k,
                        int bm, long long ldo, cudaStream_t stream, int num_sms, int max_ctas = 0);

// SiLU.mul: x = bf16(silu(g) * u) (x, g, u [M, K] BF16), and the fused
// quantiser requant_a(bf16(silu(g) * u)) into the requant_a layout.
cudaError_t launch_silu_mul(const uint16_t* g, const uint16_t* u, uint16_t* x, int m, int k, cudaStream_t stream,
                            int num_sms);
cudaError_t launch_requant_silu_a(const uint16_t* g, const uint16_t* u, int8_t* a_i8, float* a_scale_t, int m, int k,
                                  int ld, cudaStream_t stream, int num_sms);

// NVFP4 decode GEMVs on the weight as stored (W4A16: BF16 activations; W4A4:
// activation rows quantised to NVFP4 inside the kernel).  The plan fixes the
// launch: MR activation rows per CTA (gy = ceil(M / MR) CTA rows),
// rows_per_cta weight rows per CTA (gx CTAs) in stages of RS rows, `warps`
// warps taking alternate stages through `slots` slots each (bulk copies when
// K % 256 == 0).  False if K > 65536, if even one slot per warp does not fit
// in smem_limit, or if M needs more than 65535 CTA rows.
struct GemvPlan {
  int mr, rs, warps, slots, rows_per_cta, gx, gy;
  size_t smem;
  bool bulk;
};
bool nvfp4_gemv_plan(int m, int n, int k, bool a4, size_t smem_limit, size_t smem_per_sm, int num_sms,
                     GemvPlan& p);
cudaError_t launch_nvfp4_gemv(const GemvPlan& p, bool a4, const uint16_t* a, const uint8_t* w_packed,
                              const uint8_t* w_e4m3, float scale2, uint16_t* out, int m, int n, int k,
                              int static_weight, int* status, cudaStream_t stream);

// Test entry: one CTA waits on an mbarrier nothing arrives on, through the
// bounded wait of the pipelined kernels, for at most limit_ns.
cudaError_t launch_debug_wait(int* status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace bsr
