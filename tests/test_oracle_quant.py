"""Pins for the oracle's 32-group quantisation and both requantisations.

* hand-derived golden groups and NVFP4 rows (tests/golden),
* an exact re-derivation with rational arithmetic on random groups,
* invariants: the amax element maps to +-127, the reconstruction error is at
  most half a step, codes are odd in x, a power-of-two rescale of the input
  rescales the scale and keeps the codes.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._golden import cases, f32_round, rne_int


def _bits(x):
    return int(np.array(x, dtype=np.float32).view(np.uint32))


@pytest.mark.parametrize("case", cases("group_quant_cases.txt"), ids=lambda c: c["name"])
def test_golden_groups(case):
    x = np.array([float(v) for v in case["x"]], dtype=np.float32)[None, :]
    q, s = oracle.quantize_groups(x)
    assert q[0].tolist() == [int(v) for v in case["codes"]]
    if "scale" in case:
        assert _bits(s[0, 0]) == int(case["scale"][0], 16)


def test_golden_groups_through_requant_a():
    # the power-of-two group is BF16-representable: same codes via requant_a
    case = [c for c in cases("group_quant_cases.txt") if c["name"] == "power_of_two_roundtrip"][0]
    x = np.array([float(v) for v in case["x"]], dtype=np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), x)
    q, s = oracle.requant_a(bits[None, :])
    assert q[0].tolist() == [int(v) for v in case["codes"]]
    assert _bits(s[0, 0]) == 0x3E000000


@pytest.mark.parametrize("case", cases("nvfp4_rows.txt"), ids=lambda c: c["name"])
def test_golden_nvfp4_rows(case):
    k = int(case["k"][0])
    packed = np.array([int(b, 16) for b in case["packed"]], dtype=np.uint8)[None, :]
    e4 = np.array([int(b, 16) for b in case["e4m3"]], dtype=np.uint8)[None, :]
    scale2 = np.float32(float(case["scale2"][0]))
    q, s = oracle.requant_w(packed, e4, scale2, k)
    assert q[0].tolist() == [int(v) for v in case["codes"]]
    # scale re-derived exactly: amax of each 32-group over 127, rounded once
    v = oracle.dequant_nvfp4(packed, e4, scale2, k)[0]
    for g in range(k // 32):
        amax = max(abs(Fraction(float(t))) for t in v[32 * g : 32 * g + 32])
        assert _bits(s[0, g]) == _bits(f32_round(amax / 127))


def test_scale2_is_folded_into_w_scale():
    # same nibbles and E4M3 scales, scale2 doubled -> identical codes, doubled scales
    rng = np.random.default_rng(7)
    packed = rng.integers(0, 256, size=(4, 64), dtype=np.uint8)
    e4 = rng.integers(0x20, 0x60, size=(4, 8), dtype=np.uint8)
    q1, s1 = oracle.requant_w(packed, e4, np.float32(0.375), 128)
    q2, s2 = oracle.requant_w(packed, e4, np.float32(0.75), 128)
    assert np.array_equal(q1, q2)
    assert np.array_equal(s2, s1 * np.float32(2.0))


def _exact_quant(group):
    """Reference quantisation of one group with rational arithmetic and explicit
    float32 rounding after each step the oracle performs in float32."""
    xs = [Fraction(float(t)) for t in group]
    amax = max(abs(t) for t in xs)
    scale = f32_round(amax / 127)
    if scale == 0:
        return [0] * len(xs), scale
    sc = Fraction(float(scale))
    codes = []
    for t in xs:
        qf = f32_round(t / sc)
        codes.append(max(-127, min(127, rne_int(Fraction(float(qf))))))
    return codes, scale


def test_random_groups_exact_rederivation():
    rng = np.random.default_rng(11)
    for trial in range(60):
        mag = 2.0 ** rng.integers(-30, 30)
        x = (rng.standard_normal((1, 32)) * mag).astype(np.float32)
        if trial % 5 == 0:
            x[0, rng.integers(32)] *= np.float32(50.0)  # an outlier
        q, s = oracle.quantize_groups(x)
        codes, scale = _exact_quant(x[0])
        assert q[0].tolist() == codes
        assert _bits(s[0, 0]) == _bits(scale)


def test_invariants_random():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((200, 32 * 16)) * rng.uniform(1e-3, 1e3, (200, 1))).astype(np.float32)
    q, s = oracle.quantize_groups(x)
    g = x.reshape(200, 16, 32).astype(np.float64)
    qg = q.reshape(200, 16, 32).astype(np.float64)
    sc = s.astype(np.float64)[..., None]
    # the largest element maps to +-127
    idx = np.argmax(np.abs(g), axis=2)
    top = np.take_along_axis(qg, idx[..., None], axis=2)[..., 0]
    assert np.all(np.abs(top) == 127)
    # reconstruction within half a step (plus float32 slack)
    assert np.all(np.abs(g - qg * sc) <= sc * (0.5 + 2.0 ** -20))
    # odd symmetry
    qn, sn = oracle.quantize_groups(-x)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    # power-of-two rescale: same codes, scale scaled exactly
    q4, s4 = oracle.quantize_groups(x * np.float32(4.0))
    assert np.array_equal(q4, q) and np.array_equal(s4, s * np.float32(4.0))
    # codes never reach -128
    assert q.min() >= -127


def test_all_six_group_gives_127():
    # every nibble +-6 under one E4M3 scale -> codes +-127 whatever the scale
    rng = np.random.default_rng(9)
    for e4 in (0x01, 0x30, 0x38, 0x55, 0x7E):
        signs = rng.integers(0, 2, size=32)
        nib = (7 | (signs << 3)).astype(np.uint8)
        packed = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)[None, :]
        q, _ = oracle.requant_w(packed, np.array([[e4, e4]], dtype=np.uint8), np.float32(0.01), 32)
        assert np.array_equal(q[0], np.where(signs == 1, -127, 127))


def test_e4m3_nan_rejected():
    packed = np.zeros((1, 16), dtype=np.uint8)
    with pytest.raises(ValueError):
        oracle.requant_w(packed, np.array([[0x7F, 0x38]], dtype=np.uint8), np.float32(1.0), 32)


def test_k_not_multiple_of_32_rejected():
    with pytest.raises(ValueError):
        oracle.quantize_groups(np.zeros((1, 48), dtype=np.float32))
