"""Pins for the oracle's number formats: E4M3 and E2M1 decode, nibble order,
float32 -> BF16 rounding.  Each is checked against something outside the
oracle: published format tables (tests/golden), PyTorch's own float8 and
bfloat16 conversions, and the OCP closed forms."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests._golden import value_table


def _same_float(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


def test_e4m3_golden_table():
    tab = value_table("e4m3_values.txt")
    for byte, val in tab.items():
        if math.isnan(val):
            with pytest.raises(ValueError):
                oracle.e4m3_decode(np.array([byte], dtype=np.uint8))
        else:
            got = float(oracle.e4m3_decode(np.array([byte], dtype=np.uint8))[0])
            assert _same_float(got, val), (hex(byte), got, val)


def test_e4m3_all_codes_match_torch_float8():
    codes = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_e2m1_golden_table_and_closed_form():
    tab = value_table("e2m1_values.txt")
    for nib, val in tab.items():
        got = float(oracle.e2m1_decode(np.array([nib], dtype=np.uint8))[0])
        assert _same_float(got, val)
        # OCP MX FP4 E2M1 closed form: bias 1, one mantissa bit
        s, e, m = nib >> 3, (nib >> 1) & 3, nib & 1
        mag = 0.5 * m if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
        assert _same_float(got, -mag if s else mag)


def test_nibble_order_low_first():
    packed = np.array([[0x21, 0xF7]], dtype=np.uint8)
    codes = oracle.unpack_nvfp4(packed, 4)
    assert codes.tolist() == [[0x1, 0x2, 0x7, 0xF]]


def _f32_specials():
    return np.array(
        [0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.4028235e38, -3.4028235e38,
         1e-45, -1e-45, 1.1754944e-38, 3.3895314e38, 3.3961776e38, 65504.0],
        dtype=np.float32,
    )


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(123)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[~np.isnan(x)]
    # ties: low 16 bits exactly 0x8000 with both parities of bit 16
    tie = (rng.integers(0, 2**16, size=5000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    tie = tie.view(np.float32)
    tie = tie[~np.isnan(tie)]
    x = np.concatenate([x, tie, _f32_specials()])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_rne(x)
    assert np.array_equal(got, ref)


def test_bf16_rne_nan_stays_nan():
    x = np.array([np.nan], dtype=np.float32)
    out = oracle.bf16_rne(x)
    back = (out.astype(np.uint32) << 16).view(np.float32)
    assert np.isnan(back[0])


def test_bf16_bits_to_f32_exact():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(10000).astype(np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(oracle.bf16_bits_to_f32(bits).view(np.uint32), ref.view(np.uint32))
