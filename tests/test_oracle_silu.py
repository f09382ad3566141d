"""Pins of the oracle's SiLU.mul quantiser (oracle.exp_f32, silu_mul_bf16,
requant_silu_a) against mathematics, not against itself:

* exp_f32 against float64 exp: within 3 float32 ulps over [-88, 88]
  (measured worst 2.95), exact at 0, monotone, and the stated behaviour
  outside the range;
* silu(g) * u against a float64 evaluation of g / (1 + e^-g) * u rounded once
  to BF16: equal except at BF16 rounding boundaries, where they may differ by
  one BF16 step;
* closed forms: silu(0) = 0, silu(g) = g for large g, silu(g) = -0 for very
  negative g;
* the quantiser: requant_a of the float64 product's BF16 gives the same codes
  and scales.
"""
import numpy as np

import oracle

F32 = np.float32


def _bf16(x):
    return oracle.bf16_rne(np.asarray(x, dtype=np.float32))


def _val(bits):
    return oracle.bf16_bits_to_f32(bits).astype(np.float64)


def test_exp_within_three_ulp_of_float64():
    x = np.linspace(-88.0, 88.0, 400_001).astype(np.float32)
    got = oracle.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    ulp = np.maximum(np.spacing(np.abs(ref.astype(np.float32))).astype(np.float64), 2.0 ** -149)
    err = np.abs(got - ref) / ulp
    assert err.max() <= 3.0, (float(err.max()), float(x[np.argmax(err)]))
    assert np.all(np.diff(got) >= 0), "exp_f32 must be monotone"


def test_exp_special_values():
    x = np.array([0.0, 88.0, 88.5, 1e30, -88.0, -88.5, -1e30, np.inf, -np.inf, np.nan], dtype=np.float32)
    y = oracle.exp_f32(x)
    assert y[0] == F32(1.0)
    assert np.isfinite(y[1]) and y[1] > F32(1e38)
    assert np.isinf(y[2]) and np.isinf(y[3]) and np.isinf(y[7])
    assert 0.0 < y[4] < 1e-37  # exp(-88) is subnormal in float32
    assert y[5] == 0.0 and y[6] == 0.0 and y[8] == 0.0
    assert np.isnan(y[9])


def _reference_product_bits(g_bits, u_bits):
    g = _val(g_bits)
    u = _val(u_bits)
    with np.errstate(over="ignore"):
        ref = g / (1.0 + np.exp(-g)) * u  # float64
    return _bf16(ref.astype(np.float32))  # float64 -> float32 -> bf16


def _assert_product_close(got, want):
    same = got == want
    if not np.all(same):
        # only BF16 rounding boundaries may differ, by one BF16 step
        a = got[~same].astype(np.int32)
        b = want[~same].astype(np.int32)
        assert np.all(np.abs(a - b) == 1), "product differs by more than one BF16 step"
        assert (~same).mean() < 1e-3, f"{int((~same).sum())} of {same.size} products differ"


def test_silu_of_grid_matches_float64():
    g_bits = _bf16(np.linspace(-30.0, 30.0, 200_001))
    u_bits = _bf16(np.ones(g_bits.shape))
    _assert_product_close(oracle.silu_mul_bf16(g_bits, u_bits), _reference_product_bits(g_bits, u_bits))


def test_silu_mul_random_matches_float64():
    rng = np.random.default_rng(7)
    g_bits = _bf16(rng.standard_normal(200_000) * 3)
    u_bits = _bf16(rng.standard_normal(200_000) * 2)
    _assert_product_close(oracle.silu_mul_bf16(g_bits, u_bits), _reference_product_bits(g_bits, u_bits))


def test_silu_closed_forms():
    u = _bf16(np.array([1.5, -2.0, 3.0, 0.75], dtype=np.float32))
    x = _val(oracle.silu_mul_bf16(_bf16(np.zeros(4)), u))
    assert np.all(x == 0.0)
    g = _bf16(np.full(4, 40.0))  # 1 + e^-40 rounds to 1 in float32
    assert np.array_equal(oracle.silu_mul_bf16(g, u), _bf16(_val(g) * _val(u)))
    g = _bf16(np.full(4, -100.0))  # e^100 overflows: g / inf = -0
    x = _val(oracle.silu_mul_bf16(g, u))
    assert np.all(x == 0.0)


def test_quantiser_is_requant_of_the_product():
    rng = np.random.default_rng(11)
    m, k = 5, 96
    g_bits = _bf16(rng.standard_normal((m, k)) * 2)
    u_bits = _bf16(rng.standard_normal((m, k)))
    q, s = oracle.requant_silu_a(g_bits, u_bits)
    ref_bits = _reference_product_bits(g_bits, u_bits)
    assert np.array_equal(oracle.silu_mul_bf16(g_bits, u_bits), ref_bits)  # no rounding boundary hit here
    q2, s2 = oracle.requant_a(ref_bits)
    assert np.array_equal(q, q2) and np.array_equal(s.view(np.uint32), s2.view(np.uint32))
    assert q.dtype == np.int8 and q.shape == (m, k) and s.shape == (m, k // 32)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
