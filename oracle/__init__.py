"""CPU oracle for the block-scaled int8 projection -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct numpy restatement of what the projection
computes.  Only the test suite, the smoke check and the benchmark's CPU
baseline leg may import it; the product path (the CUDA library and its
Python binding) never does, and shares no code, table or helper with it.

Sources (the launcher pages of the ``metrale_model_layers`` ops crate):

* ``gemm_dense_int8.rs`` -- doc comment of ``requant_w_nvfp4_int8``: an NVFP4
  weight (packed E2M1 ``W_packed[N, K/2]``, per-16 E4M3 scales
  ``W_e4m3[N, K/16]``, per-tensor F32 ``scale2``) is requantised to signed
  int8 ``W_i8[N, K]`` with one F32 scale per 32 elements ``W_scale[N, K/32]``.
* ``gemm_dense_int8.rs`` -- doc comment of ``int8_gemm_faith2_prefill``: BF16
  ``A[M, K]`` is requantised the same way (``requant_a_kernel``: one F32 scale
  per 32 elements), then ``faith2_kernel`` multiplies with the int8 weight and
  writes BF16 ``out[M, N]``.  ``faith2_kernel`` takes no ``scale2`` argument,
  so ``scale2`` is folded into ``W_scale`` by the weight requantisation.
* ``w4a4_proj/fixed.rs`` -- doc comment of ``nvfp4_proj_mx``: a row's output
  bits do not depend on the row count or on the other rows; the same page's
  W4A4 projection (a per-row NVFP4 quantiser of the BF16 input, then the
  "mx" GEMV on the NVFP4 weight; its arithmetic is this module's reading,
  see ``quantize_nvfp4_rows`` and ``w4a4_proj``).
* ``w8a8_decode/parts.rs`` -- doc comment of ``W8a8Weight::segment``: a
  segment of a stacked weight yields the bits the stacked launch yields for
  those rows; ``W8a8Kernels::quant_silu``: the SiLU.mul quantiser (its
  arithmetic is this module's reading, see ``silu_mul_bf16``: the exact
  product rounded once to BF16, then requant_a).
* ``gemv_sw.rs`` -- the ``w4a16_gemv`` / ``w4a16_gemv_sw`` launches: the NVFP4
  W4A16 decode GEMV's arguments (its arithmetic is this module's reading, see
  ``w4a16_gemv``).

Conventions the pages leave open, fixed here (each is listed, with the reading
taken, in the design notes of this repository):

* E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, bit 3 the sign, element 2i in
  the low nibble of byte i.
* E4M3 per OCP FP8 (bias 7, subnormal step 2^-9, 0x7F/0xFF NaN).
* Dequantised weight ``v = (e2m1 * e4m3) * scale2`` in float32 (the first
  product is exact, the second rounds once).
* Per 32-group: ``amax = max|x|``, ``scale = amax / 127`` (float32, round to
  nearest), ``q = clamp(rint_half_even(x / scale), -127, 127)`` with the
  division in float32; a group whose scale is 0 gets scale 0 and codes 0.
* Block partial ``P[m, n, b] = sum_j a_i8[m, 32b+j] * w_i8[n, 32b+j]`` (exact
  integer).
* Accumulation in float32, blocks in ascending order from +0:
  ``s = a_scale * w_scale``, ``t = float(P) * s``, ``acc = acc + t``, each
  step rounded to nearest (no fused multiply-add).
* Output ``bf16_rne(acc)``.

Where a code or an integer is decided by floating point (the quantised codes),
the oracle takes the decision in float32, the precision of the scales.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "E2M1_MAGNITUDES",
    "e2m1_decode",
    "e4m3_decode",
    "unpack_nvfp4",
    "dequant_nvfp4",
    "quantize_groups",
    "requant_w",
    "bf16_bits_to_f32",
    "requant_a",
    "block_partials",
    "accumulate",
    "bf16_rne",
    "proj_rows",
    "proj",
    "f64_to_bf16_bits",
    "silu_mul_bf16",
    "requant_silu_a",
    "w4a16_gemv",
    "e4m3_encode_rne",
    "e2m1_encode_rne",
    "quantize_nvfp4_rows",
    "w4a4_proj",
]

GROUP = 32  # elements per int8 scale group
QMAX = 127

# ---------------------------------------------------------------------------
# Formats
# ---------------------------------------------------------------------------

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """E2M1 nibble (0..15) -> float32: magnitude table indexed by the low three
    bits, negative when bit 3 is set (``requant_w_nvfp4_int8``: "packed E2M1")."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where(codes & 8, -mag, mag).astype(np.float32)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """E4M3 byte -> float32 (``requant_w_nvfp4_int8``: "per-16 E4M3 block
    scales").  Sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0;
    exponent 0 is subnormal ``m * 2^-9``; 0x7F and 0xFF are NaN, which is
    outside the projection's contract and raises."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    if np.any((b & 0x7F) == 0x7F):
        raise ValueError("E4M3 NaN code in weight scales")
    s = b >> 7
    e = (b >> 3) & 0xF
    m = b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    return np.where(s == 1, -mag, mag).astype(np.float32)


def unpack_nvfp4(w_packed: np.ndarray, k: int) -> np.ndarray:
    """``W_packed[N, K/2]`` -> nibble codes ``[N, K]``: element ``2i`` is the low
    nibble of byte ``i``, element ``2i+1`` the high nibble."""
    w_packed = np.asarray(w_packed, dtype=np.uint8)
    n = w_packed.shape[0]
    assert w_packed.shape == (n, k // 2)
    codes = np.empty((n, k), dtype=np.uint8)
    codes[:, 0::2] = w_packed & 0xF
    codes[:, 1::2] = w_packed >> 4
    return codes


def dequant_nvfp4(w_packed, w_e4m3, scale2, k: int) -> np.ndarray:
    """Dequantised NVFP4 weight ``v[n, k] = (e2m1(c) * e4m3(s[n, k // 16])) * scale2``
    in float32."""
    codes = unpack_nvfp4(w_packed, k)
    n = codes.shape[0]
    e4 = e4m3_decode(np.asarray(w_e4m3).reshape(n, k // 16))
    e4_per_elem = np.repeat(e4, 16, axis=1)
    prod = e2m1_decode(codes) * e4_per_elem  # exact in float32
    return (prod * np.float32(scale2)).astype(np.float32)


# ---------------------------------------------------------------------------
# Group quantisation (shared definition for W and A)
# ---------------------------------------------------------------------------


def quantize_groups(x: np.ndarray):
    """Quantise float32 ``x[R, K]`` per 32-element group along K.

    Returns (codes int8 [R, K], scale float32 [R, K/32]).  For each group:
    ``amax = max|x|``; ``scale = amax / 127`` in float32; if ``scale == 0`` all
    codes are 0; else ``q = clamp(rint(x / scale), -127, 127)`` with the
    division in float32 and rint rounding half to even.
    """
    x = np.asarray(x, dtype=np.float32)
    r, k = x.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 32")
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input")
    g = x.reshape(r, k // GROUP, GROUP)
    amax = np.max(np.abs(g), axis=2)
    scale = (amax / np.float32(QMAX)).astype(np.float32)
    zero = scale == 0
    safe = np.where(zero, np.float32(1.0), scale).astype(np.float32)
    q = np.rint(g / safe[..., None]).astype(np.float32)
    q = np.clip(q, -QMAX, QMAX)
    q = np.where(zero[..., None], 0.0, q)
    return q.astype(np.int8).reshape(r, k), scale


def requant_w(w_packed, w_e4m3, scale2, k: int):
    """``requant_w_nvfp4_int8``: NVFP4 -> (W_i8 [N, K] int8, W_scale [N, K/32] f32)."""
    v = dequant_nvfp4(w_packed, w_e4m3, scale2, k)
    return quantize_groups(v)


def bf16_bits_to_f32(a_bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) -> float32, exact (the bits are the high half)."""
    a_bits = np.asarray(a_bits, dtype=np.uint16)
    return (a_bits.astype(np.uint32) << 16).view(np.float32)


def requant_a(a_bits: np.ndarray):
    """``requant_a_kernel``: BF16 A[M, K] -> (a_i8 [M, K] int8, a_scale [M, K/32] f32)."""
    return quantize_groups(bf16_bits_to_f32(a_bits))


# ---------------------------------------------------------------------------
# GEMM (int8 x int8, per-32 block rescale, F32 accumulation, BF16 out)
# ---------------------------------------------------------------------------


def block_partials(a_i8: np.ndarray, w_i8: np.ndarray) -> np.ndarray:
    """Exact integer block dot products ``P[m, n, b]`` (int64) for a_i8 [M, K],
    w_i8 [N, K]: the sum over the 32 elements of block b of a * w."""
    a = np.asarray(a_i8, dtype=np.int8)
    w = np.asarray(w_i8, dtype=np.int8)
    m, k = a.shape
    n = w.shape[0]
    nb = k // GROUP
    ab = a.reshape(m, nb, GROUP).astype(np.int64)
    wb = w.reshape(n, nb, GROUP).astype(np.int64)
    out = np.empty((m, n, nb), dtype=np.int64)
    for i in range(m):
        out[i] = np.einsum("bj,nbj->nb", ab[i], wb)
    return out


def accumulate(p: np.ndarray, a_scale: np.ndarray, w_scale: np.ndarray) -> np.ndarray:
    """F32 accumulation over blocks in ascending order:
    ``acc = acc + float(P) * (a_scale * w_scale)``, each operation rounded to
    float32.  p: [M, N, B]; a_scale: [M, B]; w_scale: [N, B] -> acc [M, N]."""
    m, n, nb = p.shape
    acc = np.zeros((m, n), dtype=np.float32)
    for b in range(nb):
        s = (a_scale[:, b][:, None] * w_scale[:, b][None, :]).astype(np.float32)
        t = (p[:, :, b].astype(np.float32) * s).astype(np.float32)
        acc = (acc + t).astype(np.float32)
    return acc


def bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns (uint16), round to nearest, ties to even.
    NaN stays NaN (quiet)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return np.where(nan, ((u >> 16) | 0x40).astype(np.uint16), r).astype(np.uint16)


def proj_rows(a_bits: np.ndarray, w_i8: np.ndarray, w_scale: np.ndarray) -> np.ndarray:
    """``int8_gemm_faith2_prefill`` on the given activation rows:
    requant_a, block partials, F32 accumulation, BF16 output bits [M, N].

    Rows are computed independently, one at a time."""
    a_bits = np.atleast_2d(np.asarray(a_bits, dtype=np.uint16))
    m = a_bits.shape[0]
    out = np.empty((m, np.asarray(w_i8).shape[0]), dtype=np.uint16)
    for i in range(m):
        a_i8, a_scale = requant_a(a_bits[i : i + 1])
        p = block_partials(a_i8, w_i8)
        out[i] = bf16_rne(accumulate(p, a_scale, w_scale))[0]
    return out


def proj(a_bits, w_packed, w_e4m3, scale2, k: int) -> np.ndarray:
    """The whole path from the NVFP4 weight: requant_w, then proj_rows."""
    w_i8, w_scale = requant_w(w_packed, w_e4m3, scale2, k)
    return proj_rows(a_bits, w_i8, w_scale)


# ---------------------------------------------------------------------------
# SiLU.mul quantiser
#
# The pages name a quantiser of the SiLU product (w8a8_decode/parts.rs,
# ``W8a8Kernels::quant_silu``; the gate+up step of the grouped decode page,
# ``moe_expert_gate_up_act_fp8_grouped_tc_w8a8``, writes "quantized
# products") but give no arithmetic for it.  Reading taken: the product is
# the BF16 activation the down projection would otherwise receive,
#     x = bf16_rne(silu(g) * u),   silu(g) = g / (1 + exp(-g)),
# every step a float32 operation rounded to nearest, and the quantiser is
# requant_a of x.  exp is spelled out below so that a GPU implementation can
# follow the same steps and agree bit for bit.
# ---------------------------------------------------------------------------

# float32 constants, by bit pattern
def f64_to_bf16_bits(x) -> np.ndarray:
    """BF16 bits of float64 values rounded once to nearest, ties to even.

    The value goes to float32 rounded to odd (round to nearest, then, when
    that was inexact and landed on an even significand, step one float32 ulp
    towards the value), then to BF16 by bf16_rne.  With 16 more significand
    bits in float32 than in BF16, rounding to odd first makes the second
    rounding equal to one direct rounding of the float64 value.  BF16 has
    float32's exponent range, so subnormal results follow the same rule."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        f = x.astype(np.float32)
        inexact = np.isfinite(f) & (f.astype(np.float64) != x)
        even = (f.view(np.uint32) & np.uint32(1)) == 0
        fix = inexact & even
        toward = np.where(x > f.astype(np.float64), np.float32(np.inf), np.float32(-np.inf)).astype(np.float32)
        f = np.where(fix, np.nextafter(f, toward), f).astype(np.float32)
    return bf16_rne(f)


def silu_mul_bf16(g_bits: np.ndarray, u_bits: np.ndarray) -> np.ndarray:
    """BF16 bits of silu(g) * u from BF16 g and u (bit patterns): the
    mathematical function silu(g) = g / (1 + e^-g) times u, evaluated in
    float64 and rounded once to BF16 (round to nearest, ties to even).

    float64 carries 29 bits more than float32, so the only values this can
    misround are those within a few float64 ulps of a BF16 rounding boundary.
    For g < -709.78 e^-g overflows float64 and the quotient is -0; the exact
    product there is below 10^-300 * |u|, which rounds to zero in BF16."""
    g = bf16_bits_to_f32(np.asarray(g_bits, dtype=np.uint16)).astype(np.float64)
    u = bf16_bits_to_f32(np.asarray(u_bits, dtype=np.uint16)).astype(np.float64)
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        x = g / (1.0 + np.exp(-g)) * u
    return f64_to_bf16_bits(x)


def requant_silu_a(g_bits: np.ndarray, u_bits: np.ndarray):
    """The SiLU.mul quantiser: requant_a of silu_mul_bf16(g, u)."""
    return requant_a(silu_mul_bf16(g_bits, u_bits))


# ---------------------------------------------------------------------------
# NVFP4 W4A16 decode GEMV (gemv_sw.rs: `w4a16_gemv` / `w4a16_gemv_sw`, the
# decode GEMV launched with the BF16 input, the packed E2M1 weight, its E4M3
# scales, the F32 scale_2, the BF16 output, n and k).  The page gives the
# arguments, not the arithmetic.  Reading taken: the weight is dequantised as
# in requant_w (v = (e2m1 * e4m3) * scale2) and
#     out[m, n] = bf16_rne( sum_k float(A[m, k]) * v[n, k] ),
# with the sum taken here in float64 (the exact reference of any float32
# summation order; a GPU result is compared within the BF16 tolerance).
# ---------------------------------------------------------------------------


def w4a16_gemv(a_bits, w_packed, w_e4m3, scale2, k: int) -> np.ndarray:
    """BF16 output bits [M, N] of the W4A16 GEMV (float64 sum)."""
    v = dequant_nvfp4(w_packed, w_e4m3, scale2, k).astype(np.float64)
    x = bf16_bits_to_f32(np.atleast_2d(np.asarray(a_bits, dtype=np.uint16))).astype(np.float64)
    return bf16_rne((x @ v.T).astype(np.float32))


# ---------------------------------------------------------------------------
# W4A4: NVFP4 activations (w4a4_proj/fixed.rs, `nvfp4_proj_mx`: a per-row
# NVFP4 quantiser of the BF16 input, then the "mx" GEMV on the NVFP4 weight;
# "the quantizer is per row, so a row's output bits do not depend on m or on
# the other rows").  The page gives no arithmetic.  Readings taken
# (provisional, for a later kernel):
#   * the quantiser encodes each row as the weight is stored: per-row F32
#     scale2 = RN(amax_row / 2688) (2688 = 6 * 448), per-16 E4M3 scale
#     s16 = E4M3_RNE(RN(amax16 / RN(6 * scale2))), codes
#     E2M1_RNE(RN(x / RN(s16 * scale2))); an all-zero row (or block) gets
#     scale 0 and codes 0;
#   * the product is the dot product of the dequantised operands,
#     scale2_a * scale2_w * sum_k (e2m1_a * s16_a) * (e2m1_w * s16_w), in
#     float64 (each term is exact there) and rounded to BF16 at the end; a GPU
#     sums in float32 and is compared within the BF16 tolerance.
# ---------------------------------------------------------------------------

def _e4m3_table():
    """All non-negative finite E4M3 values with their byte codes (0x00..0x7E)."""
    codes = np.arange(0x7F, dtype=np.uint8)
    return codes, e4m3_decode(codes).astype(np.float64)


def e4m3_encode_rne(x) -> np.ndarray:
    """Nearest E4M3 byte of non-negative x (ties to the even mantissa, i.e.
    the even code; values above 448 saturate to 448), by search over the
    table of all finite values."""
    x = np.minimum(np.asarray(x, dtype=np.float64), 448.0)  # saturation first: no ties among huge distances
    codes, vals = _e4m3_table()
    d = np.abs(x[..., None] - vals)
    best = d.min(axis=-1, keepdims=True)
    tie_ok = d == best
    # among equally near values prefer the even code (even mantissa)
    pref = np.where(tie_ok & ((codes & 1) == 0), 0, np.where(tie_ok, 1, 2))
    return codes[np.argmin(pref, axis=-1)].astype(np.uint8)


def e2m1_encode_rne(y) -> np.ndarray:
    """E2M1 nibble of y (sign of y in bit 3; magnitude rounded to the nearest
    of {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even mantissa, saturating at
    6), by search over the table."""
    y = np.asarray(y, dtype=np.float64)
    mags = E2M1_MAGNITUDES.astype(np.float64)
    d = np.abs(np.minimum(np.abs(y), 6.0)[..., None] - mags)  # saturation first, as for E4M3
    best = d.min(axis=-1, keepdims=True)
    tie_ok = d == best
    idx = np.arange(8)
    pref = np.where(tie_ok & ((idx & 1) == 0), 0, np.where(tie_ok, 1, 2))
    mag = np.argmin(pref, axis=-1).astype(np.uint8)
    sign = np.signbit(y).astype(np.uint8) << 3  # a negative value rounded to 0 is -0 (0x8)
    return (mag | sign).astype(np.uint8)


def quantize_nvfp4_rows(a_bits: np.ndarray):
    """The per-row NVFP4 quantiser of BF16 rows [M, K] (K % 16 == 0):
    (packed codes u8 [M, K/2], E4M3 bytes u8 [M, K/16], scale2 f32 [M])."""
    x = bf16_bits_to_f32(np.atleast_2d(np.asarray(a_bits, dtype=np.uint16)))
    m, k = x.shape
    f32 = np.float32
    amax = np.max(np.abs(x), axis=1)
    scale2 = (amax / f32(2688.0)).astype(np.float32)
    blocks = x.reshape(m, k // 16, 16)
    amax16 = np.max(np.abs(blocks), axis=2)
    six_s2 = (f32(6.0) * scale2).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(six_s2[:, None] > 0, (amax16 / six_s2[:, None]).astype(np.float32), f32(0.0))
    e4 = e4m3_encode_rne(t)
    s16 = e4m3_decode(e4)
    denom = (s16 * scale2[:, None]).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(denom[..., None] > 0, (blocks / denom[..., None]).astype(np.float32), f32(0.0))
    codes = e2m1_encode_rne(y).reshape(m, k)
    packed = ((codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)).astype(np.uint8)
    return packed, e4.astype(np.uint8), scale2


def _nvfp4_unscaled(packed, e4, k: int) -> np.ndarray:
    """e2m1(c) * e4m3(s16) per element, float64 (exact), without scale2."""
    codes = unpack_nvfp4(packed, k)
    n = codes.shape[0]
    s16 = np.repeat(e4m3_decode(np.asarray(e4).reshape(n, k // 16)), 16, axis=1)
    return e2m1_decode(codes).astype(np.float64) * s16.astype(np.float64)


def w4a4_proj(a_bits, w_packed, w_e4m3, scale2_w, k: int) -> np.ndarray:
    """BF16 output bits [M, N] of the W4A4 projection: the row quantiser
    above, then the dequantised dot product (float64) times both F32 scales."""
    ap, ae, as2 = quantize_nvfp4_rows(a_bits)
    va = _nvfp4_unscaled(ap, ae, k)
    vw = _nvfp4_unscaled(w_packed, w_e4m3, k)
    acc = (va @ vw.T) * (as2.astype(np.float64)[:, None] * float(np.float32(scale2_w)))
    return bf16_rne(acc.astype(np.float32))
