"""GPU parity of the two requantisation kernels against the oracle: int8
codes and F32 scales must be bit-exact."""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._golden import cases
from tests._gpu import DEV, f32, up_bf16, up_u8, weight_to_dev

pytestmark = pytest.mark.gpu


def _check_w(w, n, k):
    wp, we, s2 = weight_to_dev(w)
    w_i8, w_s = bsr.requant_w(wp, we, s2)
    q, s = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert np.array_equal(w_i8.cpu().numpy(), q)
    assert np.array_equal(f32(w_s).view(np.uint32), s.view(np.uint32))


def test_requant_w_tiny(tiny):
    _check_w(tiny, 256, 512)


@pytest.mark.parametrize("case", cases("nvfp4_rows.txt"), ids=lambda c: c["name"])
def test_requant_w_golden_rows(case):
    k = int(case["k"][0])
    w = {"w_packed": np.array([[int(b, 16) for b in case["packed"]]], dtype=np.uint8),
         "w_e4m3": np.array([[int(b, 16) for b in case["e4m3"]]], dtype=np.uint8),
         "scale2": np.float32(float(case["scale2"][0]))}
    _check_w(w, 1, k)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_requant_w_random_bytes(seed):
    # every nibble, every non-NaN E4M3 byte (both signs), awkward scale2
    rng = np.random.default_rng(seed)
    n, k = 77, 1024
    e4 = rng.integers(0, 256, size=(n, k // 16), dtype=np.uint8)
    e4[(e4 & 0x7F) == 0x7F] = 0x38
    e4[0, :] = 0  # zero-scale blocks
    w = {"w_packed": rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8), "w_e4m3": e4,
         "scale2": np.float32([1.0, 3.1e-5, -0.7][seed])}
    _check_w(w, n, k)


def test_requant_w_subnormal_outputs():
    # scale2 tiny: dequantised values and the 32-group scales are float32 subnormals
    rng = np.random.default_rng(5)
    n, k = 16, 256
    w = {"w_packed": rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8),
         "w_e4m3": rng.integers(0, 0x30, size=(n, k // 16), dtype=np.uint8),
         "scale2": np.float32(1e-36)}
    _check_w(w, n, k)


@pytest.mark.parametrize("name", ["decode", "ffn_up", "ffn_down", "square_ragged"])
def test_requant_w_full_size(name):
    wl = synth.WORKLOADS[name]
    w = synth.make_weight(wl.n, wl.k, wl.seed, wl.weight_outlier_rows)
    _check_w(w, wl.n, wl.k)


def _check_a(a_bits):
    m, k = a_bits.shape
    a_i8, a_st = bsr.requant_a(up_bf16(a_bits))
    q, s = oracle.requant_a(a_bits)
    assert np.array_equal(a_i8.cpu().numpy(), q)
    st = f32(a_st)
    assert st.shape == (k // 32, bsr.a_scale_ld(m))
    assert np.array_equal(st[:, :m].T.view(np.uint32), s.view(np.uint32))


def test_requant_a_tiny(tiny):
    _check_a(tiny["a_bits"])


@pytest.mark.parametrize("m", [1, 2, 3, 7, 8, 9, 15, 16, 17, 127, 128, 129])
def test_requant_a_edge_rows(m):
    a, _ = synth.make_activations(m, 256, seed=m, recipe="laplace_zero_row")
    _check_a(a)


@pytest.mark.parametrize("m,k", [(37, 2080), (9, 1024), (130, 3168), (8, 32)])
def test_requant_a_ragged_column_tiles(m, k):
    """K spanning several 1024-column tiles with a ragged last tile, and
    row counts around the 8-row tile."""
    a, _ = synth.make_activations(m, k, seed=k + m, recipe="laplace_zero_row")
    _check_a(a)


def test_requant_a_specials():
    # zero groups, subnormal BF16, huge values, exact halves (ties)
    k = 128
    x = np.zeros((6, k), dtype=np.float32)
    x[1, :32] = np.float32(1e-40)
    x[1, 5] = np.float32(3e-39)
    x[2, :] = np.float32(3.0e38)
    x[2, 1::2] = np.float32(-1.5e38)
    x[3, :32] = np.arange(32, dtype=np.float32) * np.float32(0.125) - 2
    x[4, :] = np.linspace(-7.9375, 7.9375, k, dtype=np.float32)
    x[5, 32:64] = np.float32(-0.0)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    _check_a(bits)


@pytest.mark.parametrize("name", ["ffn_up", "ffn_down", "square_ragged"])
def test_requant_a_full_size(name):
    """Every code and scale of the full activation (outlier channels, SiLU(g)*u
    with near-zero groups, Laplace with an all-zero row)."""
    wl = synth.WORKLOADS[name]
    a, info = synth.make_activations(wl.m, wl.k, wl.seed, wl.act)
    _check_a(a)
    if "near_zero_groups" in info:
        _, s = oracle.requant_a(a[int(info["near_zero_groups"][0]) // (wl.k // 32)][None])
        assert np.any(s < 1e-6)


def test_no_device_timeouts():
    assert bsr.device_status() == 0
