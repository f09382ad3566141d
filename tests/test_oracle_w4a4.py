"""Pins of the oracle's W4A4 path (oracle.e4m3_encode_rne, e2m1_encode_rne,
quantize_nvfp4_rows, w4a4_proj) against things other than the oracle:

* the E4M3 encoder against PyTorch's float32 -> float8_e4m3fn cast (round to
  nearest even) on every value in [0, 448] that matters: each code, each
  midpoint, and points just beside each midpoint; saturation above 448;
* the E2M1 encoder on its midpoints and neighbours, worked out by hand from
  the grid {0, .5, 1, 1.5, 2, 3, 4, 6};
* whole rows derived by hand (tests/golden/w4a4_rows.txt): an exact ladder,
  a rounded E4M3 scale, saturation, every E2M1 midpoint, an E4M3 midpoint,
  zero and negative-zero rows;
* the row quantiser against the weight generator's encoder (an independent
  implementation: thresholds and float64 intermediates instead of table
  search and float32 steps) -- equal except where the float32 quotient lands
  on an E2M1 midpoint that the float64 one misses, which the test checks is
  the only cause of any difference; and against the quantisation error
  bound of one E2M1 step per element;
* the product against exact rational arithmetic on a tiny case (bit-exact),
  against the W4A16 result within the error the activation quantiser adds,
  and the invariances the definition implies: each row's bits are
  independent of the other rows, sign symmetry, and scaling a row by a power
  of two scales its outputs exactly.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from block_scaled_precision_requant_b200 import synth
from tests import _golden

F32 = np.float32


def _bf16(x):
    return oracle.bf16_rne(np.asarray(x, dtype=np.float32))


def _val(bits):
    return oracle.bf16_bits_to_f32(bits)


# --------------------------------------------------------------------------
# Encoders
# --------------------------------------------------------------------------


def test_e4m3_encoder_matches_torch_cast():
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    eps = np.spacing(mids.astype(np.float32)).astype(np.float64)
    x = np.concatenate([vals, mids, mids - 4 * eps, mids + 4 * eps, np.linspace(0, 448, 20001)])
    x = x.astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode_rne(x), want)


def test_e4m3_encoder_saturates():
    assert np.all(oracle.e4m3_encode_rne(np.array([448.0, 464.0, 470.0, 1e6, 1e30, np.inf])) == 0x7E)


def test_e2m1_encoder_by_hand():
    ys = {
        0.0: 0, 0.24: 0, 0.25: 0, 0.26: 1, 0.5: 1, 0.75: 2, 1.0: 2, 1.25: 2, 1.26: 3,
        1.5: 3, 1.75: 4, 2.0: 4, 2.5: 4, 2.51: 5, 3.0: 5, 3.5: 6, 4.0: 6, 4.99: 6,
        5.0: 6, 5.01: 7, 6.0: 7, 7.0: 7, 1e9: 7, 1e30: 7, float("inf"): 7,
    }
    y = np.array(list(ys), dtype=np.float32)
    want = np.array(list(ys.values()), dtype=np.uint8)
    assert np.array_equal(oracle.e2m1_encode_rne(y), want)
    assert np.array_equal(oracle.e2m1_encode_rne(-y), want | 8)  # sign in bit 3, -0 kept


# --------------------------------------------------------------------------
# Row quantiser
# --------------------------------------------------------------------------


def golden_rows():
    """(name, BF16 bits [1, K], scale2, e4m3 bytes, codes) of each hand-derived row."""
    out = []
    for c in _golden.cases("w4a4_rows.txt"):
        x = np.array([float(v) for v in c["x"]], dtype=np.float32)
        bits = oracle.bf16_rne(x)
        # the fixture's decimals are exact in BF16, signs of zero included
        assert np.array_equal(oracle.bf16_bits_to_f32(bits).view(np.uint32), x.view(np.uint32)), c["name"]
        out.append((c["name"], bits[None], np.float32(c["scale2"][0]),
                    np.array([int(v, 16) for v in c["e4m3"]], dtype=np.uint8),
                    np.array([int(v, 16) for v in c["codes"]], dtype=np.uint8)))
    return out


def test_row_quantiser_hand_derived_rows():
    for name, bits, s2, e4, codes in golden_rows():
        k = bits.shape[1]
        p, e, s = oracle.quantize_nvfp4_rows(bits)
        assert s[0] == s2, name
        assert np.array_equal(e[0], e4), name
        assert np.array_equal(oracle.unpack_nvfp4(p, k)[0], codes), name


def _rows(m, k, seed):
    a, _ = synth.make_activations(m, k, seed, "normal_outlier_channels")
    return a


def test_row_quantiser_agrees_with_generator_encoder():
    m, k = 24, 512
    a = _rows(m, k, 3)
    p, e, s2 = oracle.quantize_nvfp4_rows(a)
    x = _val(a)
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    e4_mids = set(((vals[:-1] + vals[1:]) / 2).tolist())
    diffs = 0
    for i in range(m):
        gp, ge, gs = synth.quantize_nvfp4(x[i:i + 1])
        assert gs == s2[i]
        same_scale = ge[0] == e[i]
        for b in np.nonzero(~same_scale)[0]:
            # the float32 quotient amax16 / (6 scale2) sits on an E4M3 midpoint
            t32 = F32(np.abs(x[i, 16 * b:16 * b + 16]).max() / F32(F32(6.0) * s2[i]))
            assert float(t32) in e4_mids, (i, b, t32)
        c1 = oracle.unpack_nvfp4(p[i:i + 1], k)[0]
        c2 = oracle.unpack_nvfp4(gp, k)[0]
        bad = np.nonzero((c1 != c2) & np.repeat(same_scale, 16))[0]
        diffs += bad.size + 16 * int((~same_scale).sum())
        s16 = oracle.e4m3_decode(e[i]).astype(np.float32)
        for j in bad:
            den = F32(s16[j // 16] * s2[i])
            y32 = abs(F32(x[i, j] / den))
            # the float32 quotient sits exactly on a midpoint of the E2M1 grid
            assert y32 in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0), (i, j, y32)
    assert diffs <= m * k // 100


def test_row_quantiser_error_bound_and_shapes():
    m, k = 16, 1024
    a = _rows(m, k, 4)
    p, e, s2 = oracle.quantize_nvfp4_rows(a)
    assert p.shape == (m, k // 2) and e.shape == (m, k // 16) and s2.shape == (m,)
    assert p.dtype == np.uint8 and e.dtype == np.uint8 and s2.dtype == np.float32
    x = _val(a).astype(np.float64)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(s2, (amax / 2688.0).astype(np.float32)) or np.allclose(s2, amax / 2688.0, rtol=2 ** -23)
    s16 = np.repeat(oracle.e4m3_decode(e).astype(np.float64), 16, axis=1)
    deq = oracle.e2m1_decode(oracle.unpack_nvfp4(p, k)).astype(np.float64) * s16 * s2[:, None]
    step = s16 * s2[:, None]
    # in units of the block scale: within half the widest E2M1 gap (4 -> 6)
    # below saturation, |y| - 6 above it, with a float32-rounding slack for
    # quotients that round onto a midpoint
    y = np.abs(x) / np.where(step > 0, step, np.inf)
    bound = np.maximum(1.0, y - 6.0) * step * (1 + 2.0 ** -20)
    assert np.all(np.abs(x - deq) <= np.where(step > 0, bound, np.abs(x)))
    # the largest element of each row is represented within 1/8 relative
    j = np.argmax(np.abs(x), axis=1)
    r = np.arange(m)
    assert np.all(np.abs(deq[r, j] - x[r, j]) <= np.abs(x[r, j]) / 8)


def test_rounding_decision_taken_on_the_float32_quotient():
    # where the float32 quotient x / (s16 * scale2) lands on an E2M1 midpoint
    # that the exact quotient does not, the code is the even neighbour of the
    # float32 value (the precision a kernel decides in), not the nearest
    # value to the exact quotient
    m, k = 32, 1024
    a = _rows(m, k, 10)
    p, e, s2 = oracle.quantize_nvfp4_rows(a)
    x = _val(a)
    codes = oracle.unpack_nvfp4(p, k)
    s16 = np.repeat(oracle.e4m3_decode(e), 16, axis=1)
    den = (s16 * s2[:, None]).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y32 = np.abs((x / den).astype(np.float32)).astype(np.float64)
        y64 = np.abs(x.astype(np.float64) / den.astype(np.float64))
    even_down = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    hits = 0
    for mid, code in even_down.items():
        sel = (y32 == mid) & (y64 != mid) & (den > 0)
        hits += int(sel.sum())
        assert np.all((codes[sel] & 7) == code), mid
    assert hits > 0


def test_row_quantiser_zero_row_and_zero_block():
    k = 64
    a = _rows(3, k, 5).copy()
    a[1] = 0
    a[2, 16:32] = 0
    p, e, s2 = oracle.quantize_nvfp4_rows(a)
    assert s2[1] == 0 and np.all(e[1] == 0) and np.all(p[1] == 0)
    assert e[2, 1] == 0 and np.all(p[2, 8:16] == 0) and s2[2] > 0


# --------------------------------------------------------------------------
# Product
# --------------------------------------------------------------------------


def _exact_product_bits(a_bits, w, k):
    """Rational reference: quantised codes -> exact sum -> float32 -> BF16."""
    p, e, s2 = oracle.quantize_nvfp4_rows(a_bits)
    ca = oracle.unpack_nvfp4(p, k)
    cw = oracle.unpack_nvfp4(w["w_packed"], k)
    ea = oracle.e4m3_decode(e)
    ew = oracle.e4m3_decode(w["w_e4m3"])
    m, n = ca.shape[0], cw.shape[0]
    out = np.zeros((m, n), dtype=np.float32)
    for i in range(m):
        for c in range(n):
            acc = Fraction(0)
            for kk in range(k):
                va = Fraction(float(oracle.e2m1_decode(ca[i, kk]))) * Fraction(float(ea[i, kk // 16]))
                vw = Fraction(float(oracle.e2m1_decode(cw[c, kk]))) * Fraction(float(ew[c, kk // 16]))
                acc += va * vw
            acc *= Fraction(float(s2[i])) * Fraction(float(w["scale2"]))
            out[i, c] = F32(float(acc))
    return _bf16(out)


def test_product_exact_on_tiny_case():
    m, n, k = 3, 5, 48
    w = synth.make_weight(n, k, 6)
    a = _rows(m, k, 6)
    assert np.array_equal(oracle.w4a4_proj(a, w["w_packed"], w["w_e4m3"], w["scale2"], k),
                          _exact_product_bits(a, w, k))


def test_product_close_to_w4a16_within_quantiser_error():
    m, n, k = 8, 96, 512
    w = synth.make_weight(n, k, 7)
    a = _rows(m, k, 7)
    got = _val(oracle.w4a4_proj(a, w["w_packed"], w["w_e4m3"], w["scale2"], k)).astype(np.float64)
    ref = _val(oracle.w4a16_gemv(a, w["w_packed"], w["w_e4m3"], w["scale2"], k)).astype(np.float64)
    p, e, s2 = oracle.quantize_nvfp4_rows(a)
    s16 = np.repeat(oracle.e4m3_decode(e).astype(np.float64), 16, axis=1)
    deq = oracle.e2m1_decode(oracle.unpack_nvfp4(p, k)).astype(np.float64) * s16 * s2[:, None]
    wv = oracle.dequant_nvfp4(w["w_packed"], w["w_e4m3"], w["scale2"], k).astype(np.float64)
    bound = np.abs(_val(a).astype(np.float64) - deq) @ np.abs(wv).T
    bound += (np.abs(got) + np.abs(ref)) * 2.0 ** -8 + 1e-30  # two BF16 roundings
    assert np.all(np.abs(got - ref) <= bound)
    assert np.corrcoef(got.ravel(), ref.ravel())[0, 1] > 0.98


def test_product_row_independence_sign_and_power_of_two():
    m, n, k = 6, 40, 256
    w = synth.make_weight(n, k, 8)
    args = (w["w_packed"], w["w_e4m3"], w["scale2"], k)
    a = _rows(m, k, 8)
    full = oracle.w4a4_proj(a, *args)
    for i in range(m):
        assert np.array_equal(full[i:i + 1], oracle.w4a4_proj(a[i:i + 1], *args))
    # other rows changed (scaled by 1000): row 0 unchanged
    b = _bf16(_val(a) * np.array([1.0] + [1000.0] * (m - 1), dtype=np.float32)[:, None])
    assert np.array_equal(oracle.w4a4_proj(b, *args)[0], full[0])
    # sign symmetry
    neg = oracle.w4a4_proj(a ^ np.uint16(0x8000), *args)
    assert np.array_equal(_val(neg), -_val(full))
    # a row scaled by 2^5 gives outputs scaled by 2^5 exactly
    up = _bf16(_val(a) * F32(32.0))
    assert np.array_equal(_val(oracle.w4a4_proj(up, *args)), _val(full) * F32(32.0))


def test_product_zero_row():
    k = 128
    w = synth.make_weight(16, k, 9)
    a = _rows(2, k, 9).copy()
    a[0] = 0
    out = oracle.w4a4_proj(a, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert np.all(_val(out[0]) == 0.0) and np.any(out[1] != 0)
