"""Pins of the oracle's SiLU.mul quantiser (oracle.f64_to_bf16_bits,
silu_mul_bf16, requant_silu_a) against mathematics, not against itself:

* f64_to_bf16_bits against a direct search of the table of every finite
  BF16 value (nearest, ties to the even bit pattern), on random values, on
  exact BF16 midpoints and on values one float64 ulp either side of them --
  the cases a plain float64 -> float32 -> BF16 double rounding gets wrong;
* silu(g) * u against a 50-digit decimal evaluation of g / (1 + e^-g) * u,
  rounded to BF16 with exact rational comparisons: equal bits everywhere
  (the float64 evaluation is accurate to a few float64 ulps, and no sampled
  value lies that close to a BF16 rounding boundary -- the test checks that
  too);
* closed forms: silu(0) = 0, silu(g) * u = g * u for large g, and a very
  negative g gives a signed zero;
* the quantiser: requant_a of the decimal reference's BF16 product gives the
  same codes and scales.
"""
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np

import oracle

F32 = np.float32


def _bf16(x):
    return oracle.bf16_rne(np.asarray(x, dtype=np.float32))


def _val(bits):
    return oracle.bf16_bits_to_f32(bits).astype(np.float64)


# Every finite non-negative BF16 value, ascending, with its bit pattern.
_POS_BITS = np.arange(0x0000, 0x7F80, dtype=np.uint16)
_POS_VALS = _val(_POS_BITS)


def _nearest_bf16_exact(x: Fraction) -> int:
    """BF16 bits nearest to the rational x (ties to the even pattern),
    by search in the value table; beyond the largest finite value halfway
    to 2^128, infinity."""
    sign = 0x8000 if x < 0 else 0
    a = -x if x < 0 else x
    top = Fraction(_POS_VALS[-1]) + (Fraction(2) ** 128 - Fraction(_POS_VALS[-1])) / 2
    if a > top or (a == top and (int(_POS_BITS[-1]) & 1)):
        return sign | 0x7F80
    i = int(np.searchsorted(_POS_VALS, float(a), side="right")) - 1
    i = max(0, min(i, len(_POS_VALS) - 1))
    # float(a) may round across a table entry; settle with exact comparisons
    while i + 1 < len(_POS_VALS) and Fraction(_POS_VALS[i + 1]) <= a:
        i += 1
    while i > 0 and Fraction(_POS_VALS[i]) > a:
        i -= 1
    lo = Fraction(_POS_VALS[i])
    if lo == a or i + 1 == len(_POS_VALS):
        return sign | int(_POS_BITS[i])
    hi = Fraction(_POS_VALS[i + 1])
    d_lo, d_hi = a - lo, hi - a
    if d_lo < d_hi or (d_lo == d_hi and (int(_POS_BITS[i]) & 1) == 0):
        return sign | int(_POS_BITS[i])
    return sign | int(_POS_BITS[i + 1])


def test_f64_to_bf16_random_values():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(3000) * 10.0 ** rng.uniform(-40, 38, 3000)
    got = oracle.f64_to_bf16_bits(x)
    want = np.array([_nearest_bf16_exact(Fraction(float(v))) for v in x], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_f64_to_bf16_midpoints_and_neighbours():
    rng = np.random.default_rng(2)
    bits = rng.integers(0x0001, 0x7F7F, size=400).astype(np.uint16)
    lo = _val(bits)
    hi = _val(bits + 1)
    mid = (lo + hi) / 2  # exact in float64
    vals = np.concatenate([mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf)])
    vals = np.concatenate([vals, -vals])
    got = oracle.f64_to_bf16_bits(vals)
    want = np.array([_nearest_bf16_exact(Fraction(float(v))) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)
    # the double rounding this guards against does differ on some of them
    naive = oracle.bf16_rne(vals.astype(np.float32))
    assert np.any(naive != want)


def _silu_mul_decimal(g: float, u: float) -> Fraction:
    getcontext().prec = 50
    dg = Decimal(g)
    val = dg / (Decimal(1) + (-dg).exp()) * Decimal(u)
    return Fraction(val)


def _reference_bits(g_bits, u_bits):
    g = _val(g_bits)
    u = _val(u_bits)
    return np.array([_nearest_bf16_exact(_silu_mul_decimal(float(a), float(b))) for a, b in zip(g, u)],
                    dtype=np.uint16)


def _distance_to_boundary(x: Fraction) -> Fraction:
    """Relative distance from x to the nearest BF16 rounding boundary."""
    if x == 0:
        return Fraction(1)
    b = _nearest_bf16_exact(x)
    v = Fraction(float(_val(np.array([b], dtype=np.uint16))[0]))
    step = Fraction(float(_val(np.array([(b & 0x7FFF) + 1], dtype=np.uint16))[0])) - abs(v)
    return abs(step / 2 - abs(x - v)) / abs(x)


def test_silu_mul_matches_decimal_reference():
    rng = np.random.default_rng(7)
    g_bits = _bf16(np.concatenate([rng.standard_normal(1500) * 3, np.linspace(-120.0, 120.0, 500)]))
    u_bits = _bf16(rng.standard_normal(2000) * 10.0 ** rng.uniform(-3, 3, 2000))
    got = oracle.silu_mul_bf16(g_bits, u_bits)
    want = _reference_bits(g_bits, u_bits)
    # no sampled product lies within 2^-40 (relative) of a rounding boundary,
    # so the float64 evaluation must round the same way
    gs, us = _val(g_bits), _val(u_bits)
    for a, b in zip(gs[:200], us[:200]):
        assert _distance_to_boundary(_silu_mul_decimal(float(a), float(b))) > Fraction(1, 2 ** 40)
    assert np.array_equal(got, want)


def test_silu_closed_forms():
    u = _bf16(np.array([1.5, -2.0, 3.0, 0.75], dtype=np.float32))
    x = _val(oracle.silu_mul_bf16(_bf16(np.zeros(4)), u))
    assert np.all(x == 0.0)
    g = _bf16(np.full(4, 40.0))  # e^-40 < 2^-57: silu(40) = 40 (1 - 4e-18)
    assert np.array_equal(oracle.silu_mul_bf16(g, u), _bf16(_val(g) * _val(u)))
    g = _bf16(np.full(4, -100.0))  # |silu(-100)| = 3.7e-42, far below half the smallest BF16 subnormal
    got = oracle.silu_mul_bf16(g, u)
    assert np.array_equal(got, np.array([0x8000, 0x0000, 0x8000, 0x8000], dtype=np.uint16))
    g = _bf16(np.full(4, -89.0))  # silu(-89) = -89 e^-89 = -3.9e-37: a normal BF16 value, not zero
    assert np.all(_val(oracle.silu_mul_bf16(g, u)) != 0.0)


def test_quantiser_is_requant_of_the_exact_product():
    rng = np.random.default_rng(11)
    m, k = 5, 96
    g_bits = _bf16(rng.standard_normal((m, k)) * 2)
    u_bits = _bf16(rng.standard_normal((m, k)))
    q, s = oracle.requant_silu_a(g_bits, u_bits)
    ref_bits = _reference_bits(g_bits.reshape(-1), u_bits.reshape(-1)).reshape(m, k)
    q2, s2 = oracle.requant_a(ref_bits)
    assert np.array_equal(q, q2) and np.array_equal(s.view(np.uint32), s2.view(np.uint32))
    assert q.dtype == np.int8 and q.shape == (m, k) and s.shape == (m, k // 32)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
