/*
 * bsr.h -- C ABI of the block-scaled int8 projection library (libbsr.so) for
 * NVIDIA B200 (sm_100a).
 *
 * The library computes the quantised projection out[M, N] = A[M, K] . W[N, K]^T
 * described by the launcher page gemm_dense_int8.rs of the metrale
 * model-layers ops crate:
 *
 *   1. `requant_w_nvfp4_int8` (doc comment): an NVFP4 weight -- packed E2M1
 *      nibbles W_packed[N, K/2], one E4M3 scale per 16 elements W_e4m3[N, K/16],
 *      one per-tensor F32 scale2 -- is requantised once to signed int8
 *      W_i8[N, K] with one F32 scale per 32 elements W_scale[N, K/32]; the
 *      caller keeps the result and reuses it ("ensure_int8_weight").
 *   2. `int8_gemm_faith2_prefill` (doc comment): the BF16 activations A[M, K]
 *      are requantised the same way (`requant_a_kernel`), then
 *      `faith2_kernel` forms each 32-wide block's int32 dot product, multiplies
 *      it by a_scale * w_scale, accumulates in F32 and writes BF16 out[M, N].
 *
 * Conventions fixed by this library where the page is silent:
 *   - E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, bit 3 = sign; element 2i of
 *     a row is the low nibble of byte i.  E4M3 as in the OCP FP8 spec; the NaN
 *     codes 0x7F / 0xFF are outside the contract (results unspecified).
 *   - Dequantised weight v = (e2m1 * e4m3) * scale2 in float32.
 *   - Per 32-element group: scale = RN_f32(amax / 127),
 *     code = clamp(rint_half_even(RN_f32(x / scale)), -127, 127); an all-zero
 *     group (or one whose scale underflows to 0) has scale 0 and codes 0.
 *     Codes and scales are bit-exact with the CPU oracle in oracle/.
 *   - Per block b the GPU adds RN(float(P) * w_scale) * a_scale into a float32
 *     accumulator with one rounding (FMA); the order of the blocks' additions
 *     is the library's, so BF16 outputs agree with the oracle within
 *     |err| <= 2^-7 |ref| + 1e-3 rms(ref), not bit for bit.  Within one path
 *     a row's output bits do not depend on M, on the other rows, on N or on
 *     which rows of a stacked weight are launched together.
 *
 * Memory: every pointer is a device pointer (except where noted) owned by the
 * caller; no call allocates device memory (the library's own device storage
 * is a status word and the bsr_proj_noalloc array, both reserved when the
 * library's GPU code is loaded).  All arrays are dense
 * row-major.  Every call is asynchronous on `stream` (a cudaStream_t, NULL =
 * the legacy default stream) and returns before the kernels finish.
 *
 * Errors: arguments are checked before anything is launched; on a non-OK
 * status nothing was launched and bsr_last_error() returns a message (thread
 * local).  M == 0 or N == 0 is a no-op that returns BSR_OK.  A CUDA launch
 * failure returns BSR_ECUDA.  Kernels never trap: a pipeline wait that runs
 * out (1 s) makes the kernel return early and sets a bit that
 * bsr_device_status() reports.
 */
#ifndef BSR_H_
#define BSR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BSR_ABI_VERSION 1

typedef enum bsr_status {
  BSR_OK = 0,
  BSR_EINVAL = 1,   /* null pointer, negative or too large dimension */
  BSR_EALIGN = 2,   /* a pointer is not 16-byte aligned */
  BSR_ESHAPE = 3,   /* K not a positive multiple of 32 (or of 128 where stated) */
  BSR_ESCRATCH = 4, /* scratch missing or smaller than bsr_proj_scratch_bytes() */
  BSR_ECUDA = 5,    /* a CUDA runtime/driver call failed */
  BSR_ETIMEOUT = 6, /* reported by bsr_device_status() */
  BSR_ENODEV = 7    /* no CUDA device, or not an sm_100 device */
} bsr_status;

/* Largest M, N or K accepted (the TMA coordinates are 32-bit). */
#define BSR_MAX_DIM 2147483647LL

/* Rows of A at or below which bsr_proj takes the decode path. */
#define BSR_DECODE_MAX_M 16

int bsr_abi_version(void);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* bsr_last_error(void);

/* Synchronises the current device, returns and clears the device status
 * word: 0 if no kernel aborted a wait since the last call, else the OR of
 * bits naming the waits that ran out (GEMM: 1 TMA producer, 2 MMA issuer,
 * 4 epilogue, 8 scale preparation; 16 decode kernel; 32 the test entry
 * bsr_debug_wait_timeout).  Returns -1 if the device could not be queried. */
int bsr_device_status(void);

/*
 * bsr_requant_w -- gemm_dense_int8.rs, `requant_w_nvfp4_int8`.
 *   w_packed  [N, K/2]  uint8, two E2M1 codes per byte, low nibble first
 *   w_e4m3    [N, K/16] uint8, E4M3 scale of each 16-element block
 *   scale2    per-tensor F32 scale (host value), folded into w_scale
 *   w_i8      [N, K]    int8 out: codes
 *   w_scale   [N, K/32] float out: scale of each 32-element group
 * Requirements: K > 0, K % 32 == 0; all pointers 16-byte aligned.
 * HBM-bound; call once per weight and keep (w_i8, w_scale).
 */
bsr_status bsr_requant_w(const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2, int8_t* w_i8,
                         float* w_scale, int64_t n, int64_t k, void* stream);

/* Leading dimension (in floats) of the block-major activation scales for M
 * rows: M rounded up to a multiple of 4. */
int64_t bsr_a_scale_ld(int64_t m);

/*
 * bsr_requant_a -- gemm_dense_int8.rs, `requant_a_kernel` (first launch of
 * `int8_gemm_faith2_prefill`).
 *   a          [M, K] BF16 (raw uint16 bit patterns)
 *   a_i8       [M, K] int8 out
 *   a_scale_t  [K/32, ld] float out, block-major: the scale of row m, block b
 *              is a_scale_t[b * ld + m], ld = bsr_a_scale_ld(M); entries
 *              m >= M are not written
 * Requirements: K > 0, K % 32 == 0; pointers 16-byte aligned.
 */
bsr_status bsr_requant_a(const uint16_t* a, int8_t* a_i8, float* a_scale_t, int64_t m, int64_t k, void* stream);

/*
 * bsr_gemm -- gemm_dense_int8.rs, `faith2_kernel` (second launch of
 * `int8_gemm_faith2_prefill`): the tcgen05 kind::i8 tensor-core GEMM with
 * per-32-block rescale.
 *   a_i8, a_scale_t  as written by bsr_requant_a (ld = bsr_a_scale_ld(M))
 *   w_i8, w_scale    as written by bsr_requant_w
 *   out              [M, N] BF16 out (uint16 bit patterns)
 * Requirements: K % 128 == 0 (the W_scale row pitch must be a multiple of 16
 * bytes for the tensor-memory-access copies); pointers 16-byte aligned.
 */
bsr_status bsr_gemm(const int8_t* a_i8, const float* a_scale_t, const int8_t* w_i8, const float* w_scale,
                    uint16_t* out, int64_t m, int64_t n, int64_t k, void* stream);

/*
 * Scratch bytes bsr_proj needs for M rows (0 when M <= BSR_DECODE_MAX_M, or
 * when K % 128 != 0, where the decode kernel serves every M): the int8
 * activation codes (M*K bytes) then, 256-byte aligned, the block-major scales
 * ((K/32) * bsr_a_scale_ld(M) floats) -- the caller-owned `a_i8_scratch` and
 * `a_scale_scratch` of `int8_gemm_faith2_prefill`, in one buffer.
 */
size_t bsr_proj_scratch_bytes(int64_t m, int64_t k);

/* Activation rows per tile (128, 192 or 256) that the tensor-core GEMM uses
 * for an M x N problem on the current device: 128 when M <= 128, else the
 * width whose whole waves of persistent tiles take the least estimated time.
 * Informational (no launch); 0 if there is no usable device or M, N < 1. */
int bsr_gemm_block_m(int64_t m, int64_t n);

/*
 * bsr_proj -- gemm_dense_int8.rs, `int8_gemm_faith2_prefill`:
 * out[M, N] = A[M, K] . W[N, K]^T from BF16 A and the requantised weight.
 *   M <= BSR_DECODE_MAX_M: one launch of the decode kernel (CUDA cores,
 *     activation requantisation fused, split over K across a warp); scratch
 *     may be NULL.
 *   M >  BSR_DECODE_MAX_M: bsr_requant_a into `scratch`, then bsr_gemm, both
 *     on `stream`.  If K % 128 != 0 the decode kernel serves the rows instead
 *     (in chunks of 16 rows per CTA row).
 *   scratch        device buffer of at least bsr_proj_scratch_bytes(M, K)
 *                  bytes, 256-byte aligned; contents are overwritten
 * Requirements: K > 0, K % 32 == 0; a, w_i8, w_scale 16-byte aligned; out
 * 2-byte aligned.
 */
bsr_status bsr_proj(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m, int64_t n,
                    int64_t k, void* scratch, size_t scratch_bytes, void* stream);

/*
 * bsr_decode -- the decode kernel of bsr_proj for any M (activation rows in
 * groups of up to 16 per CTA row), exposed so both paths can be run on the
 * same shapes.  No scratch.  Requirements as bsr_proj.
 */
bsr_status bsr_decode(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m,
                      int64_t n, int64_t k, void* stream);

/*
 * bsr_gemm_partials -- bsr_gemm that also writes every block partial
 * P[m, n, b] (int32, [M, N, K/32]) exactly as the tensor cores produced it,
 * for bit-exact checks.  Test use; slow.
 */
bsr_status bsr_gemm_partials(const int8_t* a_i8, const float* a_scale_t, const int8_t* w_i8, const float* w_scale,
                             uint16_t* out, int32_t* partials, int64_t m, int64_t n, int64_t k, void* stream);

/* bsr_decode_ex flag: no kernel that writes w_i8 or w_scale is in flight or
 * queued ahead of this call on the stream (e.g. a decode loop over a
 * resident weight).  The kernel then issues part of its first weight copies
 * before waiting for the previous kernel on the stream, so they overlap that
 * kernel's tail.  Activations are still read only after that wait. */
#define BSR_DECODE_STATIC_WEIGHT 1u

/* bsr_decode with flags (0 or BSR_DECODE_STATIC_WEIGHT; other bits:
 * BSR_EINVAL).  Same arguments, results and errors as bsr_decode. */
bsr_status bsr_decode_ex(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m,
                         int64_t n, int64_t k, unsigned flags, void* stream);

/*
 * Decode with the activations and the result in HOST memory: a decode loop
 * driven by the host.  Same operation, results and errors as bsr_decode_ex
 * (flags 0 or BSR_DECODE_STATIC_WEIGHT); out_host holds exactly the bits
 * bsr_decode writes.
 *   a_host   [M, K] BF16, page-locked host memory mapped into the device's
 *            address space (cudaHostAlloc, or cudaHostRegister with the
 *            mapped flag; with unified addressing every page-locked
 *            allocation is), 16-byte aligned, owned by the caller;
 *   out_host [M, N] BF16, the same kind of memory, 16-byte aligned;
 *   a_dev    [M, K] BF16 and out_dev [M, N] BF16: device staging buffers
 *            owned by the caller, 16-byte aligned.
 * Three launches on `stream`, each with programmatic dependent launch: a
 * copy kernel reads a_host into a_dev over the host link, the decode kernel
 * computes out_dev, a copy kernel writes out_dev into out_host.  The host
 * may read out_host (or rewrite a_host) only once the stream has passed
 * this call.  A host buffer that is not page-locked and mapped gives
 * BSR_EINVAL, with nothing launched.
 */
bsr_status bsr_decode_host(const uint16_t* a_host, const int8_t* w_i8, const float* w_scale, uint16_t* out_host,
                           int64_t m, int64_t n, int64_t k, uint16_t* a_dev, uint16_t* out_dev, unsigned flags,
                           void* stream);

/*
 * bsr_proj with the activations and the result in HOST memory, pipelined:
 * the rows go in chunks of `chunk_rows` (0: about four chunks of whole
 * 128-row tiles, at least 512 rows; never more than 64 chunks), and while
 * chunk c is requantised and multiplied on `stream`, chunk c+1 is copied in
 * and chunk c-1 copied out on the library's own copy streams (DMA copies).
 * Same operation, results and errors as bsr_proj on each chunk of rows: a
 * row's bits do not depend on the other rows, so out_host holds exactly the
 * bits bsr_proj writes.
 *   a_host   [M, K] BF16 and out_host [M, N] BF16: page-locked host memory
 *            (cudaHostAlloc / cudaHostRegister), owned by the caller;
 *   a_dev    [M, K] BF16 (16-byte aligned) and out_dev [M, N] BF16: device
 *            staging buffers owned by the caller;
 *   scratch  bsr_proj_host_scratch_bytes(M, K, chunk_rows) bytes, 256-byte
 *            aligned (0 bytes when every chunk takes the decode kernel).
 * `stream` passes the call once the last chunk's result is in out_host. A
 * host buffer that is not page-locked gives BSR_EINVAL, with nothing
 * launched; every chunk's launch is prepared before the first is queued.
 */
int64_t bsr_proj_host_scratch_bytes(int64_t m, int64_t k, int64_t chunk_rows);
bsr_status bsr_proj_host(const uint16_t* a_host, const int8_t* w_i8, const float* w_scale, uint16_t* out_host,
                         int64_t m, int64_t n, int64_t k, uint16_t* a_dev, uint16_t* out_dev, void* scratch,
                         size_t scratch_bytes, int64_t chunk_rows, void* stream);

/*
 * Stacked weights (w8a8_decode/parts.rs, `W8a8Weight`: a weight stacked from
 * segments, e.g. Q, K and V, whose `segment(i)` "writes the bits the stacked
 * launch writes for those rows").  Segment s is a weight of its own
 * (w_i8[s] [n_segs[s], K], w_scale[s] [n_segs[s], K/32], each 16-byte
 * aligned, anywhere in device memory); the host arrays w_i8, w_scale and
 * n_segs hold num_segs (1..BSR_MAX_SEGMENTS) entries.  The output is
 * out [M, N] BF16 with N = sum of n_segs: segment s fills columns
 * [off_s, off_s + n_segs[s]), off_s the sum of the earlier counts, with the
 * bits a launch on that segment alone writes.
 */
#define BSR_MAX_SEGMENTS 8

/* The decode kernel over all segments in one launch (flags as bsr_decode_ex). */
bsr_status bsr_decode_stacked(const uint16_t* a, const int8_t* const* w_i8, const float* const* w_scale,
                              const int64_t* n_segs, int num_segs, uint16_t* out, int64_t m, int64_t k, unsigned flags,
                              void* stream);

/* bsr_proj over a stacked weight: M <= BSR_DECODE_MAX_M (or K % 128 != 0):
 * one decode launch over all segments; otherwise requant_a once into scratch
 * (bsr_proj_scratch_bytes(M, K)) and one tensor-core GEMM per segment. */
bsr_status bsr_proj_stacked(const uint16_t* a, const int8_t* const* w_i8, const float* const* w_scale,
                            const int64_t* n_segs, int num_segs, uint16_t* out, int64_t m, int64_t k, void* scratch,
                            size_t scratch_bytes, void* stream);

/*
 * bsr_w4a16_decode -- gemv_sw.rs, `w4a16_gemv` / `w4a16_gemv_sw`: the
 * NVFP4 W4A16 decode GEMV on the weight as stored (no requantisation).
 *   a         [M, K]    BF16
 *   w_packed  [N, K/2]  uint8, E2M1 pairs, element 2i in the low nibble of byte i
 *   w_e4m3    [N, K/16] uint8, E4M3 scale of each 16-element block
 *   scale2    per-tensor F32 scale (host value)
 *   out       [M, N]    BF16: sum_k a * (e2m1 * e4m3) * scale2, float32 sums
 * (per 16-block p = the 16 products summed in element order, then
 * acc = fma(p, e4m3, acc), scale2 once at the end; the blocks of a row are
 * summed in an order that depends on K only, so an output's bits depend
 * only on K and its own row and column).  Elements more than 2^32 below the
 * largest magnitude of their 16-block are rounded to the half-precision
 * subnormal grid (2^-24 relative to a block scaled into [2^15, 2^16)).  Not
 * bit-compatible with bsr_proj (that path requantises to int8).
 * 0 < K <= 65536, K % 32 == 0; pointers 16-byte aligned (out 2-byte); any M
 * up to 4 * 65535 (built for M <= 16).  Weight rows stream through shared
 * memory by bulk copies when K % 256 == 0, else are read from global memory.
 */
bsr_status bsr_w4a16_decode(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                            uint16_t* out, int64_t m, int64_t n, int64_t k, void* stream);

/* bsr_w4a16_decode with flags (0 or BSR_DECODE_STATIC_WEIGHT: no kernel that
 * writes w_packed or w_e4m3 is in flight or queued ahead on the stream; the
 * kernel then issues its weight copies before waiting for the previous
 * kernel on the stream).  Same results and errors. */
bsr_status bsr_w4a16_decode_ex(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                               uint16_t* out, int64_t m, int64_t n, int64_t k, unsigned flags, void* stream);

/*
 * NVFP4 W4A4 (w4a4_proj/fixed.rs, `nvfp4_proj_mx`: a per-row NVFP4 quantiser
 * of the BF16 input, then the "mx" GEMV on the NVFP4 weight; a row's output
 * bits do not depend on M or on the other rows).  The page gives no
 * arithmetic; reading taken: each activation row is encoded the way the
 * weight is stored,
 *   scale2 = RN(amax_row / 2688),  s16 = E4M3_RNE(RN(amax16 / RN(6 * scale2))),
 *   code = E2M1_RNE(RN(x / RN(s16 * scale2)))
 * (float32 operations rounded to nearest; E4M3 saturating at 448, E2M1 at 6
 * with ties to the even mantissa and the sign kept; a zero row or block gets
 * scale 0 and codes 0), and the product is
 *   out[m, n] = bf16( scale2_a[m] * scale2_w * sum_b s16a * s16w * sum_16 ea * ew ).
 * K > 0, K % 16 == 0; pointers 16-byte aligned (out 2-byte).  Inputs finite.
 */

/* The row quantiser alone: a [M, K] BF16 in; a_packed [M, K/2] (element 2i in
 * the low nibble of byte i), a_e4m3 [M, K/16] and a_scale2 [M] float out,
 * bit-exact with the CPU oracle. */
bsr_status bsr_nvfp4_quant_rows(const uint16_t* a, uint8_t* a_packed, uint8_t* a_e4m3, float* a_scale2, int64_t m,
                                int64_t k, void* stream);

/* The W4A4 decode GEMV, the quantiser fused in (each CTA quantises its rows
 * of A): a [M, K] BF16, w_packed [N, K/2], w_e4m3 [N, K/16], scale2 the
 * weight's F32 scale (host value), out [M, N] BF16.  The products of a
 * 16-block are exact, the sum over blocks is float32 in an order that
 * depends on K only: results agree with the exact product within the BF16
 * tolerance, and an output's bits depend only on K and its own row and
 * column (not on M, N or the other rows).  0 < K <= 65536, K % 16 == 0; any
 * M up to 4 * 65535 (built for M <= 16). */
bsr_status bsr_w4a4_decode(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                           uint16_t* out, int64_t m, int64_t n, int64_t k, void* stream);

/* bsr_w4a4_decode with flags (as bsr_w4a16_decode_ex). */
bsr_status bsr_w4a4_decode_ex(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_e4m3, float scale2,
                              uint16_t* out, int64_t m, int64_t n, int64_t k, unsigned flags, void* stream);

/*
 * W4A4 on the tensor cores (block-scaled FP4 MMA, kind::mxf4nvf4): the same
 * product as bsr_w4a4_decode, accumulated in FP32 by the MMA.  The E4M3 scale
 * bytes must be non-negative (sign bit clear) and are passed in a blocked
 * layout: for 128-row tile t and K group g (64 elements) a 512-byte atom at
 * offset (t * K/64 + g) * 512 whose 32-bit word 4*r0 + r1 holds the four
 * scales of row 128t + r0 + 32*r1 (r0 < 32, r1 < 4), scale 4g + j in byte j;
 * rows past the matrix are zero.
 */

/* Bytes of the blocked layout for `rows` rows: ceil(rows/128) * K/64 * 512
 * (0 for invalid sizes; K % 64 == 0). */
size_t bsr_nvfp4_sf_blocked_bytes(int64_t rows, int64_t k);

/* Row-major E4M3 scales e4m3 [rows, K/16] -> blocked [bsr_nvfp4_sf_blocked_bytes]
 * (once per weight; per call for activations).  16-byte aligned pointers. */
bsr_status bsr_nvfp4_sf_blocked(const uint8_t* e4m3, uint8_t* blocked, int64_t rows, int64_t k, void* stream);

/* out [M, N] BF16 = W4A4 product of a_packed [M, K/2] (scales a_sf_blocked,
 * a_scale2 [M]) and w_packed [N, K/2] (scales w_sf_blocked, scale2 host
 * value).  K % 256 == 0; every array 16-byte aligned.  status_dev: a
 * caller-owned device int into which a wait that runs out ORs its bit. */
bsr_status bsr_w4a4_gemm(const uint8_t* a_packed, const uint8_t* a_sf_blocked, const float* a_scale2,
                         const uint8_t* w_packed, const uint8_t* w_sf_blocked, float scale2, uint16_t* out, int64_t m,
                         int64_t n, int64_t k, int* status_dev, void* stream);

/* Scratch bytes bsr_w4a4_proj needs for M activation rows: the quantised
 * rows (M*K/2 packed bytes, M*K/16 E4M3 bytes), their blocked scales and the
 * M row scales, each rounded up to 256 bytes (0 for invalid sizes; K % 256
 * == 0). */
size_t bsr_w4a4_proj_scratch_bytes(int64_t m, int64_t k);

/*
 * bsr_w4a4_proj -- the whole W4A4 projection on the tensor cores
 * (w4a4_proj/fixed.rs, `nvfp4_proj_mx`: quantise the BF16 rows, then the
 * FP4 product): a [M, K] BF16 -> bsr_nvfp4_quant_rows into scratch ->
 * bsr_nvfp4_sf_blocked of the row scales -> bsr_w4a4_gemm against w_packed
 * [N, K/2] with its scales already in the blocked layout (w_sf_blocked, from
 * bsr_nvfp4_sf_blocked once per weight) and scale2 (host value); out [M, N]
 * BF16.  Bit-identical to the three calls made separately.  Scratch
 * (caller-owned, device, 256-byte aligned) of at least
 * bsr_w4a4_proj_scratch_bytes(M, K); a, w_packed, w_sf_blocked and out
 * 16-byte aligned; K % 256 == 0.  Timed-out waits are reported through
 * bsr_device_status().  Every tensor map is encoded before the first
 * launch: on a non-OK status nothing was queued.
 */
bsr_status bsr_w4a4_proj(const uint16_t* a, const uint8_t* w_packed, const uint8_t* w_sf_blocked, float scale2,
                         uint16_t* out, int64_t m, int64_t n, int64_t k, void* scratch, size_t scratch_bytes,
                         void* stream);

/*
 * SiLU.mul quantiser for the down projection (w8a8_decode/parts.rs names it,
 * `W8a8Kernels::quant_silu`; the pages give no arithmetic).  Reading taken:
 *   x = bf16_rne(silu(g) * u),  silu(g) = g / (1 + exp(-g)),
 * the exact product rounded once to BF16.  The kernels evaluate it in
 * float32 (exp of -|g| by range reduction and the hardware base-2
 * exponential, an approximate quotient) within 2^-20 relative of the exact
 * product, so x equals the exact rounding except within 2^-20 of a BF16
 * rounding boundary (one BF16 step there); for g < -104 x is a signed zero.
 * Inputs gate, up: [M, K] BF16, finite.  Requirements and errors as
 * bsr_requant_a.
 */

/* x [M, K] BF16 out: the product itself (the unfused activation). */
bsr_status bsr_silu_mul(const uint16_t* gate, const uint16_t* up, uint16_t* x, int64_t m, int64_t k, void* stream);

/* requant_a of the product without writing it: a_i8 [M, K] int8 and
 * a_scale_t [K/32, bsr_a_scale_ld(M)] float out, bit-identical to
 * bsr_silu_mul followed by bsr_requant_a. */
bsr_status bsr_requant_silu_a(const uint16_t* gate, const uint16_t* up, int8_t* a_i8, float* a_scale_t, int64_t m,
                              int64_t k, void* stream);

/* Scratch bytes bsr_proj_silu needs: bsr_proj_scratch_bytes(M, K) on the
 * tensor-core route (M > BSR_DECODE_MAX_M and K % 128 == 0), else the BF16
 * product, 2*M*K rounded up to 256 (0 for invalid sizes). */
size_t bsr_proj_silu_scratch_bytes(int64_t m, int64_t k);

/*
 * bsr_proj_silu -- the down projection from gate and up:
 *   out = proj(bf16(silu(gate) * up), W).
 * M > BSR_DECODE_MAX_M and K % 128 == 0: bsr_requant_silu_a into scratch,
 * then the tensor-core GEMM (the BF16 product is never written).  Otherwise:
 * bsr_silu_mul into scratch, then the decode kernel.  Same results as
 * bsr_silu_mul followed by bsr_proj.  Scratch (caller-owned, device,
 * 256-byte aligned) of at least bsr_proj_silu_scratch_bytes(M, K).
 */
bsr_status bsr_proj_silu(const uint16_t* gate, const uint16_t* up, const int8_t* w_i8, const float* w_scale,
                         uint16_t* out, int64_t m, int64_t n, int64_t k, void* scratch, size_t scratch_bytes,
                         void* stream);

/* Size of the device array bsr_proj_noalloc uses as its scratch: 16 MiB,
 * enough for M*K + (K/32)*round_up(M,4)*4 <= 16 MiB (e.g. M=2048, K=4096 or
 * M=3584, K=4096; not M=4095, K=8192). */
#define BSR_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * bsr_proj_noalloc -- bsr_proj for callers that cannot allocate device memory
 * at call time (a runtime that plans all device memory ahead and passes only
 * inputs and outputs, or code where cudaMalloc, which synchronises the
 * device, is not allowed).  No counterpart on the launcher pages: it is this
 * library's addition.  Same arguments, results and errors as bsr_proj without
 * the scratch pair; the activation codes and scales live in a device array
 * inside the library (BSR_NOALLOC_SCRATCH_BYTES, held on every GPU that loads
 * the library until the process exits).  Calls that need more return
 * BSR_ESCRATCH without launching.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current);
 * make that first call before any stream capture.  Every call reuses the same
 * array: calls that may overlap on the GPU (other streams, other host
 * threads) race on it and must be serialised by the caller.  Allocates
 * nothing, never calls cudaMalloc or cudaFree.
 */
bsr_status bsr_proj_noalloc(const uint16_t* a, const int8_t* w_i8, const float* w_scale, uint16_t* out, int64_t m,
                            int64_t n, int64_t k, void* stream);

/*
 * bsr_debug_wait_timeout -- test entry for the failure path; no counterpart
 * on the launcher pages.  Launches one CTA that waits on an mbarrier nothing
 * ever arrives on, through the same bounded wait the pipelined kernels use,
 * with a limit of limit_ms milliseconds (1..2000, else BSR_EINVAL).  When the
 * limit runs out the kernel sets bit 32 of the device status word and
 * returns; no fault, no trap, and the device stays usable.  Returns once the
 * kernel is queued; bsr_device_status() then waits for it and reports 32.
 */
bsr_status bsr_debug_wait_timeout(int limit_ms, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSR_H_ */
