"""The NVFP4 W4A16 decode GEMV against the oracle (float64 sums of the
dequantised weight): BF16 outputs within the projection tolerance, for M = 1
at the decode size, ragged N and K % 256 != 0, every M up to 16 and beyond,
extreme scale2, and an all-zero activation row (-> +0 bits)."""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, up_bf16, up_u8

pytestmark = pytest.mark.gpu


def _run(m, n, k, seed, recipe="normal_outlier_channels", scale2=None):
    w = synth.make_weight(n, k, seed=seed)
    s2 = float(w["scale2"]) if scale2 is None else scale2
    a_bits, _ = synth.make_activations(m, k, seed + 1, recipe)
    out = bsr.w4a16_decode(up_bf16(a_bits), up_u8(w["w_packed"]), up_u8(w["w_e4m3"]), s2)
    torch.cuda.synchronize()
    ref = oracle.w4a16_gemv(a_bits, w["w_packed"], w["w_e4m3"], np.float32(s2), k)
    return bf16_bits(out), ref, a_bits


@pytest.mark.parametrize("m,n,k", [(1, 4096, 4096), (1, 1000, 2080), (3, 300, 512), (7, 129, 1024),
                                   (16, 256, 512), (17, 200, 256)])
def test_w4a16_matches_oracle(m, n, k):
    got, ref, _ = _run(m, n, k, seed=81 + m)
    assert_close_bf16(got, ref, f"w4a16 m={m} n={n} k={k}")
    assert bsr.device_status() == 0


def test_w4a16_scale2_extremes_and_zero_row():
    got, ref, a_bits = _run(5, 256, 1024, seed=90, recipe="laplace_zero_row", scale2=3.0e-6)
    assert_close_bf16(got, ref, "w4a16 small scale2, zero row")
    zr = int(np.flatnonzero(~a_bits.any(axis=1))[0])
    assert np.all(got[zr] == 0)
    got, ref, _ = _run(2, 128, 512, seed=91, scale2=1000.0)
    assert_close_bf16(got, ref, "w4a16 large scale2")


@pytest.mark.parametrize("m,n,k", [(1, 300, 8192), (3, 130, 8192), (1, 260, 14336), (2, 100, 20480),
                                   (1, 36, 53248), (6, 300, 4096), (1, 14336, 4096)])
def test_w4a16_lane_layouts(m, n, k):
    # one case per (activation rows per CTA, blocks per lane, warps) variant,
    # the K = 53248 one with a single-stage ring, the last with ring refills
    got, ref, _ = _run(m, n, k, seed=140 + m)
    assert_close_bf16(got, ref, f"w4a16 m={m} n={n} k={k}")
    assert bsr.device_status() == 0


def test_w4a16_bits_depend_only_on_own_row_and_column():
    m, n, k = 5, 600, 4096
    w = synth.make_weight(n, k, seed=95)
    a_bits, _ = synth.make_activations(m, k, 96, "normal_outlier_channels")
    a, wp, we, s2 = up_bf16(a_bits), up_u8(w["w_packed"]), up_u8(w["w_e4m3"]), float(w["scale2"])
    full = bf16_bits(bsr.w4a16_decode(a, wp, we, s2))
    assert np.array_equal(bf16_bits(bsr.w4a16_decode(a, wp, we, s2, static_weight=True)), full)
    part = bf16_bits(bsr.w4a16_decode(a, wp[100:357], we[100:357], s2))  # other N, other CTA ranges
    assert np.array_equal(part, full[:, 100:357])
    one = bf16_bits(bsr.w4a16_decode(a[3:4], wp, we, s2))
    assert np.array_equal(one[0], full[3])
    assert bsr.device_status() == 0


def test_w4a16_wide_range_within_blocks():
    # magnitudes spread over 2^-60 .. 2^60 inside every 16-block (the kernel
    # scales each block by a power of two into half precision)
    m, n, k = 2, 200, 1024
    rng = np.random.default_rng(97)
    x = rng.standard_normal((m, k)) * np.exp2(rng.integers(-60, 61, size=(m, k)))
    a_bits = oracle.f64_to_bf16_bits(x)
    w = synth.make_weight(n, k, seed=98)
    out = bsr.w4a16_decode(up_bf16(a_bits), up_u8(w["w_packed"]), up_u8(w["w_e4m3"]), float(w["scale2"]))
    ref = oracle.w4a16_gemv(a_bits, w["w_packed"], w["w_e4m3"], np.float32(w["scale2"]), k)
    assert_close_bf16(bf16_bits(out), ref, "w4a16 wide range")
