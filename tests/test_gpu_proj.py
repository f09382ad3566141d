"""GPU parity of the projection against the oracle.

* block partials from the tensor cores: bit-exact (small ragged shapes, the
  16 x 256 x 512 workload in full, and the M-tail tile of the
  4095 x 8192 x 8192 workload at full K),
* BF16 outputs of both paths (decode kernel, tcgen05 GEMM): within
  |err| <= 2^-7 |ref| + 1e-3 rms(ref),
* the invariants: row bits independent of M and of the other rows (within a
  path), stacked-segment bits, zero inputs -> +0 bits, weight-row permutation,
* edge shapes (M = 1..129, ragged N, one K stage), the fallback epilogue for
  scales outside the fast window, and every workload at full size on 64
  sampled output rows (first and last rows, the ragged tail, the all-zero row,
  a row with near-zero groups),
* every activation-tile width the GEMM can choose (128, 192, 256 rows):
  partials bit-exact and outputs within tolerance on a ragged shape that
  selects it.
"""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import DEV, assert_close_bf16, bf16_bits, up_bf16, up_u8, weight_to_dev

pytestmark = pytest.mark.gpu


def _weights(w):
    wp, we, s2 = weight_to_dev(w)
    return bsr.requant_w(wp, we, s2)


def _oracle_w(w, k):
    return oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)


def _case(m, n, k, seed, recipe="normal", outlier_rows=0.0):
    w = synth.make_weight(n, k, seed, outlier_rows)
    a, _ = synth.make_activations(m, k, seed, recipe)
    return w, a


# --------------------------------------------------------------------------- partials


@pytest.mark.parametrize("shape", [(16, 256, 512), (129, 200, 384), (300, 131, 256)])
def test_gemm_partials_bit_exact(shape):
    m, n, k = shape
    w, a = _case(m, n, k, seed=m, recipe="laplace_zero_row", outlier_rows=0.02)
    w_i8, w_s = _weights(w)
    a_i8, a_st = bsr.requant_a(up_bf16(a))
    out, p = bsr.gemm_partials(a_i8, a_st, w_i8, w_s)
    qa, sa = oracle.requant_a(a)
    qw, sw = _oracle_w(w, k)
    ref_p = oracle.block_partials(qa, qw)
    assert np.array_equal(p.cpu().numpy().astype(np.int64), ref_p)
    ref = oracle.bf16_rne(oracle.accumulate(ref_p, sa, sw))
    assert_close_bf16(bf16_bits(out), ref, "gemm output")
    # the dump variant and the plain kernel give the same output bits
    assert np.array_equal(bf16_bits(bsr.gemm(a_i8, a_st, w_i8, w_s)), bf16_bits(out))


def _shape_for_width(width):
    """A ragged (M, N) for which the GEMM chooses activation tiles of `width`
    rows on this device."""
    for m in (129, 200, 300, 385, 520, 700, 1000, 1300, 2000):
        for n in (136, 300, 1000, 4000, 9000, 19000):
            if bsr.gemm_block_m(m, n) == width:
                return m, n
    return None


@pytest.mark.parametrize("width", [128, 192, 256])
def test_gemm_partials_each_tile_width(width):
    shape = _shape_for_width(width)
    if shape is None:
        pytest.skip(f"no searched shape selects {width}-row tiles on this device")
    m, n = shape
    k = 256
    w, a = _case(m, n, k, seed=width, recipe="laplace_zero_row", outlier_rows=0.01)
    w_i8, w_s = _weights(w)
    a_i8, a_st = bsr.requant_a(up_bf16(a))
    out, p = bsr.gemm_partials(a_i8, a_st, w_i8, w_s)
    qa, sa = oracle.requant_a(a)
    qw, sw = _oracle_w(w, k)
    ref_p = oracle.block_partials(qa, qw)
    assert np.array_equal(p.cpu().numpy().astype(np.int64), ref_p)
    ref = oracle.bf16_rne(oracle.accumulate(ref_p, sa, sw))
    assert_close_bf16(bf16_bits(out), ref, f"gemm output, {width}-row tiles")
    assert np.array_equal(bf16_bits(bsr.gemm(a_i8, a_st, w_i8, w_s)), bf16_bits(out))
    assert bsr.device_status() == 0


def test_tile_width_choice_is_valid():
    for m, n in [(17, 4096), (128, 100), (129, 4096), (2048, 14336), (8192, 4096), (4095, 8192)]:
        assert bsr.gemm_block_m(m, n) in (128, 192, 256)
    assert bsr.gemm_block_m(100, 4096) == 128


def test_gemm_partials_tiny_workload_in_full(tiny):
    # the 16 x 256 x 512 workload's own inputs, every partial
    k = 512
    w_i8, w_s = _weights(tiny)
    a_i8, a_st = bsr.requant_a(up_bf16(tiny["a_bits"]))
    out, p = bsr.gemm_partials(a_i8, a_st, w_i8, w_s)
    qa, sa = oracle.requant_a(tiny["a_bits"])
    qw, sw = _oracle_w(tiny, k)
    ref_p = oracle.block_partials(qa, qw)
    assert np.array_equal(p.cpu().numpy().astype(np.int64), ref_p)
    assert_close_bf16(bf16_bits(out), oracle.bf16_rne(oracle.accumulate(ref_p, sa, sw)), "tiny workload")


def test_gemm_partials_square_ragged_tail_tile():
    # one 127 x 256 tile of the 4095 x 8192 x 8192 workload at full K: the
    # last 127 activation rows (the ragged M tail, 4095 = 31 * 128 + 127) and
    # the 256 weight rows around one of its x100 outlier rows.  Partials are
    # per (m, n, block) and both requantisations are row-local, so this
    # sub-problem is that tile of the full launch.
    d = synth.make_workload("square_ragged")
    m, n, k = d["workload"].shape
    n0 = int(d["outlier_rows"][0]) // 256 * 256
    w = {"w_packed": d["w_packed"][n0:n0 + 256], "w_e4m3": d["w_e4m3"][n0:n0 + 256], "scale2": d["scale2"]}
    a = d["a_bits"][m - m % 128:]
    assert a.shape == (127, k)
    w_i8, w_s = _weights(w)
    a_i8, a_st = bsr.requant_a(up_bf16(a))
    out, p = bsr.gemm_partials(a_i8, a_st, w_i8, w_s)
    qa, sa = oracle.requant_a(a)
    qw, sw = _oracle_w(w, k)
    ref_p = oracle.block_partials(qa, qw)
    assert np.array_equal(p.cpu().numpy().astype(np.int64), ref_p)
    assert_close_bf16(bf16_bits(out), oracle.bf16_rne(oracle.accumulate(ref_p, sa, sw)), "tail tile output")
    assert bsr.device_status() == 0


# --------------------------------------------------------------------------- both paths


def test_tiny_both_paths(tiny):
    k = 512
    w_i8, w_s = _weights(tiny)
    a = up_bf16(tiny["a_bits"])
    ref = oracle.proj_rows(tiny["a_bits"], *_oracle_w(tiny, k))
    dec = bsr.proj(a, w_i8, w_s)  # M = 16 -> decode kernel
    assert_close_bf16(bf16_bits(dec), ref, "decode")
    a_i8, a_st = bsr.requant_a(a)
    pre = bsr.gemm(a_i8, a_st, w_i8, w_s)  # forced prefill path
    assert_close_bf16(bf16_bits(pre), ref, "prefill")
    assert np.array_equal(bf16_bits(bsr.decode(a, w_i8, w_s)), bf16_bits(dec))


@pytest.mark.parametrize("m", [1, 2, 3, 15, 16, 17, 64, 127, 128, 129, 257])
def test_edge_rows(m):
    n, k = 264, 640
    w, a = _case(m, n, k, seed=100 + m, recipe="normal_outlier_channels", outlier_rows=0.01)
    w_i8, w_s = _weights(w)
    ref = oracle.proj_rows(a, *_oracle_w(w, k))
    got = bsr.proj(up_bf16(a), w_i8, w_s)
    assert_close_bf16(bf16_bits(got), ref, f"proj m={m}")
    dec = bsr.decode(up_bf16(a), w_i8, w_s)
    assert_close_bf16(bf16_bits(dec), ref, f"decode m={m}")


def test_k_not_multiple_of_128_uses_decode_kernel():
    m, n, k = 40, 96, 160
    w, a = _case(m, n, k, seed=7)
    w_i8, w_s = _weights(w)
    assert bsr.proj_scratch_bytes(m, k) == 0
    got = bsr.proj(up_bf16(a), w_i8, w_s)
    assert_close_bf16(bf16_bits(got), oracle.proj_rows(a, *_oracle_w(w, k)), "k=160")


def test_single_k_stage_and_long_k():
    for (m, n, k) in [(130, 128, 128), (33, 130, 4096 + 128)]:
        w, a = _case(m, n, k, seed=k)
        w_i8, w_s = _weights(w)
        got = bsr.proj(up_bf16(a), w_i8, w_s)
        assert_close_bf16(bf16_bits(got), oracle.proj_rows(a, *_oracle_w(w, k)), f"{m}x{n}x{k}")


# --------------------------------------------------------------------------- invariants


def test_row_bits_independent_of_m_prefill():
    m, n, k = 300, 256, 512
    w, a = _case(m, n, k, seed=11, recipe="laplace_zero_row")
    w_i8, w_s = _weights(w)
    full = bf16_bits(bsr.proj(up_bf16(a), w_i8, w_s))
    for lo, hi in [(0, 17), (40, 200), (283, 300)]:
        part = bf16_bits(bsr.proj(up_bf16(a[lo:hi]), w_i8, w_s))
        assert np.array_equal(part, full[lo:hi])
    other = a.copy()
    other[1:] = synth.make_activations(m - 1, k, 12, "normal")[0]
    assert np.array_equal(bf16_bits(bsr.proj(up_bf16(other), w_i8, w_s))[0], full[0])


def test_row_bits_independent_of_m_decode():
    m, n, k = 16, 300, 1024
    w, a = _case(m, n, k, seed=13)
    w_i8, w_s = _weights(w)
    full = bf16_bits(bsr.proj(up_bf16(a), w_i8, w_s))
    for r in (0, 7, 15):
        one = bf16_bits(bsr.proj(up_bf16(a[r:r + 1]), w_i8, w_s))
        assert np.array_equal(one[0], full[r])


def test_stacked_segments_bits():
    m, n, k = 160, 384, 512
    w, a = _case(m, n, k, seed=17)
    w_i8, w_s = _weights(w)
    ad = up_bf16(a)
    full_p = bf16_bits(bsr.proj(ad, w_i8, w_s))
    full_d = bf16_bits(bsr.proj(ad[:4], w_i8, w_s))
    for n0, n1 in [(0, 128), (128, 300), (300, 384)]:
        seg = {"w_packed": w["w_packed"][n0:n1], "w_e4m3": w["w_e4m3"][n0:n1], "scale2": w["scale2"]}
        s_i8, s_s = _weights(seg)
        assert torch.equal(s_i8, w_i8[n0:n1]) and torch.equal(s_s, w_s[n0:n1])
        assert np.array_equal(bf16_bits(bsr.proj(ad, s_i8, s_s)), full_p[:, n0:n1])
        assert np.array_equal(bf16_bits(bsr.proj(ad[:4], s_i8, s_s)), full_d[:, n0:n1])


def test_zero_inputs_give_zero_bits():
    m, n, k = 140, 130, 256
    w, a = _case(m, n, k, seed=19)
    w_i8, w_s = _weights(w)
    for mm in (140, 5):
        z = np.zeros((mm, k), dtype=np.uint16)
        assert np.all(bf16_bits(bsr.proj(up_bf16(z), w_i8, w_s)) == 0)
    zw = {"w_packed": np.zeros_like(w["w_packed"]), "w_e4m3": w["w_e4m3"], "scale2": w["scale2"]}
    z_i8, z_s = _weights(zw)
    for mm in (140, 5):
        assert np.all(bf16_bits(bsr.proj(up_bf16(a[:mm]), z_i8, z_s)) == 0)


def test_weight_row_permutation():
    m, n, k = 136, 256, 384
    w, a = _case(m, n, k, seed=23)
    perm = np.random.default_rng(0).permutation(n)
    w_i8, w_s = _weights(w)
    out = bf16_bits(bsr.proj(up_bf16(a), w_i8, w_s))
    pw = {"w_packed": w["w_packed"][perm], "w_e4m3": w["w_e4m3"][perm], "scale2": w["scale2"]}
    p_i8, p_s = _weights(pw)
    assert np.array_equal(bf16_bits(bsr.proj(up_bf16(a), p_i8, p_s)), out[:, perm])


# --------------------------------------------------------------------------- scale window


@pytest.mark.parametrize("variant", ["huge_activations", "tiny_weight_scale", "mixed"])
def test_scales_outside_fast_window(variant):
    m, n, k = 150, 140, 512
    w, a = _case(m, n, k, seed=29)
    x = oracle.bf16_bits_to_f32(a).copy()
    if variant in ("huge_activations", "mixed"):
        x[3, :64] *= np.float32(1e30)  # a_scale ~ 1e28 > 2^79
    if variant in ("tiny_weight_scale", "mixed"):
        w = dict(w)
        w["scale2"] = np.float32(1e-30)  # w_scale ~ 1e-30 < 2^-77
    a = (x.view(np.uint32) >> 16).astype(np.uint16)
    w_i8, w_s = _weights(w)
    ref = oracle.proj_rows(a, *_oracle_w(w, k))
    assert_close_bf16(bf16_bits(bsr.proj(up_bf16(a), w_i8, w_s)), ref, variant)
    assert_close_bf16(bf16_bits(bsr.decode(up_bf16(a), w_i8, w_s)), ref, variant + " decode")


# --------------------------------------------------------------------------- full size


@pytest.fixture(scope="module")
def full_cases():
    return {}


@pytest.mark.parametrize("name", ["decode", "ffn_up", "ffn_down", "square_ragged"])
def test_full_size_sampled_rows(name):
    wl = synth.WORKLOADS[name]
    d = synth.make_workload(name)
    w_i8, w_s = _weights(d)
    a = up_bf16(d["a_bits"])
    out = bsr.proj(a, w_i8, w_s)
    torch.cuda.synchronize()
    info = d["act_info"]
    must = [info["zero_row"]] if "zero_row" in info else []
    if "near_zero_groups" in info:
        must.append(int(info["near_zero_groups"][0]) // (wl.k // 32))
    rows = synth.sample_rows(wl.m, 64 if wl.m > 1 else 1, wl.seed, must=must)
    # oracle weight requantisation on the full weight, then the sampled rows
    qw, sw = _oracle_w(d, wl.k)
    ref = oracle.proj_rows(d["a_bits"][rows], qw, sw)
    got = bf16_bits(out)[rows]
    assert_close_bf16(got, ref, name)
    if "zero_row" in info:
        zr = int(np.where(rows == info["zero_row"])[0][0])
        assert np.all(got[zr] == 0)


def test_no_device_timeouts_after_proj():
    assert bsr.device_status() == 0
