"""The NVFP4 W4A4 path against the oracle.

* The row quantiser: codes, E4M3 scales and F32 row scales bit-exact with
  oracle.quantize_nvfp4_rows on ragged shapes, rows whose float32 quotients
  land on E2M1 / E4M3 midpoints, zero rows and blocks, -0 entries, subnormal
  rows and rows near the BF16 maximum, and equal to the hand-derived rows of
  tests/golden/w4a4_rows.txt.
* The decode GEMV: BF16 outputs within the projection tolerance of
  oracle.w4a4_proj (exact sums) for M = 1 at the decode size, every M up to
  16 and beyond, ragged N, K % 256 != 0 and K = 16; a row's bits do not
  depend on M or on the other rows; an all-zero row gives +0 bits.
* The relayout of row-major E4M3 scales into the tensor-core GEMM's blocked
  layout, byte for byte against the layout restated in numpy.
"""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, f32, up_bf16, up_u8

pytestmark = pytest.mark.gpu


def _bf16(x):
    return oracle.bf16_rne(np.asarray(x, dtype=np.float32))


def _check_quant(a_bits):
    p, e, s = bsr.quant_nvfp4_rows(up_bf16(a_bits))
    torch.cuda.synchronize()
    rp, re_, rs = oracle.quantize_nvfp4_rows(a_bits)
    assert np.array_equal(f32(s).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(e.cpu().numpy(), re_)
    assert np.array_equal(p.cpu().numpy(), rp)


@pytest.mark.parametrize("m,k,seed", [(1, 16, 1), (7, 48, 2), (33, 1024, 3), (130, 4096, 4), (32, 1024, 10)])
def test_quantiser_bit_exact(m, k, seed):
    a, _ = synth.make_activations(m, k, seed, "normal_outlier_channels")
    _check_quant(a)


def test_quantiser_special_rows():
    rng = np.random.default_rng(5)
    k = 256
    rows = [
        np.zeros(k),
        np.concatenate([np.zeros(16), rng.standard_normal(k - 16)]),
        rng.standard_normal(k) * 1e-39,
        rng.standard_normal(k) * 1e-42,
        rng.uniform(-1.0, 1.0, k) * 3.3e38,
        np.full(k, -1.0),
        np.tile([6.0, -3.0, 0.5, -0.25, 1e-3, 4.0, -2.0, 1.0], k // 8),
    ]
    a = _bf16(np.stack(rows))
    a[5, ::7] = 0x8000  # -0 inside non-zero blocks
    _check_quant(a)


def test_quantiser_hand_derived_rows():
    from tests.test_oracle_w4a4 import golden_rows

    for name, bits, s2, e4, codes in golden_rows():
        p, e, s = bsr.quant_nvfp4_rows(up_bf16(bits))
        torch.cuda.synchronize()
        assert f32(s)[0] == s2 and np.array_equal(e.cpu().numpy()[0], e4), name
        assert np.array_equal(oracle.unpack_nvfp4(p.cpu().numpy(), bits.shape[1])[0], codes), name


def _run(m, n, k, seed, recipe="normal_outlier_channels"):
    w = synth.make_weight(n, k, seed=seed)
    a_bits, _ = synth.make_activations(m, k, seed + 1, recipe)
    out = bsr.w4a4_decode(up_bf16(a_bits), up_u8(w["w_packed"]), up_u8(w["w_e4m3"]), float(w["scale2"]))
    torch.cuda.synchronize()
    return bf16_bits(out), w, a_bits


@pytest.mark.parametrize("m,n,k", [(1, 4096, 4096), (1, 1000, 2080), (2, 33, 16), (3, 300, 512),
                                   (7, 129, 1024), (16, 256, 528), (17, 200, 256)])
def test_w4a4_matches_oracle(m, n, k):
    got, w, a_bits = _run(m, n, k, seed=101 + m)
    ref = oracle.w4a4_proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(got, ref, f"w4a4 m={m} n={n} k={k}")
    assert bsr.device_status() == 0


def test_w4a4_row_invariance_and_zero_row():
    m, n, k = 16, 300, 1024
    got, w, a_bits = _run(m, n, k, seed=120, recipe="laplace_zero_row")
    wp, we, s2 = up_u8(w["w_packed"]), up_u8(w["w_e4m3"]), float(w["scale2"])
    for i in (0, 5, 15):
        one = bsr.w4a4_decode(up_bf16(a_bits[i:i + 1]), wp, we, s2)
        assert np.array_equal(bf16_bits(one)[0], got[i])
    b = a_bits.copy()
    b[1:] = _bf16(oracle.bf16_bits_to_f32(b[1:]) * np.float32(1000.0))
    other = bsr.w4a4_decode(up_bf16(b), wp, we, s2)
    assert np.array_equal(bf16_bits(other)[0], got[0])
    zr = int(np.flatnonzero(~(a_bits & 0x7FFF).any(axis=1))[0])
    assert np.all(got[zr] == 0)
    ref = oracle.w4a4_proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(got, ref, "w4a4 laplace rows")


def _blocked_reference(e4, rows, k):
    """The blocked scale layout restated in numpy: atom (t, g) at
    (t * K/64 + g) * 512, word 4*r0 + r1 = the four scales 4g..4g+3 of row
    128t + r0 + 32*r1, zero past the last row."""
    tiles, groups = -(-rows // 128), k // 64
    out = np.zeros((tiles, groups, 32, 4, 4), dtype=np.uint8)  # [t][g][r0][r1][byte]
    for t in range(tiles):
        for r1 in range(4):
            for r0 in range(32):
                row = 128 * t + r0 + 32 * r1
                if row < rows:
                    out[t, :, r0, r1, :] = e4[row].reshape(groups, 4)
    return out.reshape(-1)


@pytest.mark.parametrize("rows,k", [(1, 64), (130, 256), (300, 1024)])
def test_scale_relayout_to_blocked(rows, k):
    rng = np.random.default_rng(rows + k)
    e4 = rng.integers(0, 0x7F, size=(rows, k // 16), dtype=np.uint8)
    got = bsr.sf_blocked(up_u8(e4))
    torch.cuda.synchronize()
    assert got.numel() == bsr.sf_blocked_bytes(rows, k)
    assert np.array_equal(got.cpu().numpy(), _blocked_reference(e4, rows, k))


@pytest.mark.parametrize("m,n,k", [(1, 300, 8192), (3, 130, 8192), (1, 260, 14336), (2, 100, 20480),
                                   (1, 36, 53248), (6, 300, 4096), (1, 14336, 4096)])
def test_w4a4_lane_layouts(m, n, k):
    # one case per (activation rows per CTA, blocks per lane, warps) variant,
    # the K = 53248 one with a single-stage ring, the last with ring refills
    got, w, a_bits = _run(m, n, k, seed=150 + m)
    ref = oracle.w4a4_proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(got, ref, f"w4a4 m={m} n={n} k={k}")
    assert bsr.device_status() == 0


def test_w4a4_bits_independent_of_n_and_static_flag():
    m, n, k = 3, 600, 4096
    got, w, a_bits = _run(m, n, k, seed=160)
    a, wp, we, s2 = up_bf16(a_bits), up_u8(w["w_packed"]), up_u8(w["w_e4m3"]), float(w["scale2"])
    assert np.array_equal(bf16_bits(bsr.w4a4_decode(a, wp, we, s2, static_weight=True)), got)
    part = bf16_bits(bsr.w4a4_decode(a, wp[100:357], we[100:357], s2))  # other N, other CTA ranges
    assert np.array_equal(part, got[:, 100:357])
    assert bsr.device_status() == 0
