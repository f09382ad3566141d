"""Pins for the oracle's int8 block GEMM: exact block partials by brute force,
the float32 block accumulation against an exact sum where it must be exact,
the whole oracle against a float64 GEMM of the dequantised inputs within the
quantisation error bound, and the invariants the launcher pages state."""
import itertools

import numpy as np
import pytest

import oracle
from block_scaled_precision_requant_b200 import synth


def test_partials_brute_force():
    rng = np.random.default_rng(1)
    m, n, k = 3, 5, 96
    a = rng.integers(-127, 128, size=(m, k), dtype=np.int64).astype(np.int8)
    w = rng.integers(-127, 128, size=(n, k), dtype=np.int64).astype(np.int8)
    p = oracle.block_partials(a, w)
    for i, j, b in itertools.product(range(m), range(n), range(k // 32)):
        ref = 0
        for t in range(32 * b, 32 * b + 32):
            ref += int(a[i, t]) * int(w[j, t])
        assert p[i, j, b] == ref


def test_partials_extremes():
    a = np.full((1, 32), 127, dtype=np.int8)
    w = np.full((2, 32), 127, dtype=np.int8)
    w[1] = -127
    p = oracle.block_partials(a, w)
    assert p[0, 0, 0] == 516128 and p[0, 1, 0] == -516128


def test_accumulate_exact_when_representable():
    # power-of-two scales and small partials: every step is exact, so the
    # float32 result equals the exact rational sum
    rng = np.random.default_rng(2)
    m, n, nb = 4, 6, 10
    p = rng.integers(-1000, 1000, size=(m, n, nb))
    a_s = (2.0 ** rng.integers(-4, 4, size=(m, nb))).astype(np.float32)
    w_s = (2.0 ** rng.integers(-4, 4, size=(n, nb))).astype(np.float32)
    acc = oracle.accumulate(p, a_s, w_s)
    ref = np.einsum("mnb,mb,nb->mn", p.astype(np.float64), a_s.astype(np.float64), w_s.astype(np.float64))
    assert np.array_equal(acc.astype(np.float64), ref)


def test_accumulate_order_is_ascending_blocks():
    # 2^24 + 1 - 2^24: ascending order loses the 1 (float32), a different order keeps it
    p = np.array([[[1 << 24, 1, -(1 << 24)]]])
    ones = np.ones((1, 3), dtype=np.float32)
    acc = oracle.accumulate(p, ones, ones)
    assert acc[0, 0] == 0.0


def _dequant_a(a_bits):
    return oracle.bf16_bits_to_f32(a_bits).astype(np.float64)


def _error_bound(a_bits, w_i8, w_scale, x, v):
    """Per-element bound on |oracle - exact float64 product| from quantisation
    (half a step per code, with float32 slack), the float32 scale products
    and accumulation, and the final BF16 rounding."""
    a_i8, a_scale = oracle.requant_a(a_bits)
    m, k = x.shape
    n = v.shape[0]
    nb = k // 32
    vhat = w_i8.astype(np.float64) * np.repeat(w_scale.astype(np.float64), 32, axis=1)
    eps_w = 0.50001 * w_scale.astype(np.float64)  # [N, B]
    eps_a = 0.50001 * a_scale.astype(np.float64)  # [M, B]
    absx_b = np.abs(x).reshape(m, nb, 32).sum(2)  # [M, B]
    absv_b = np.abs(vhat).reshape(n, nb, 32).sum(2)  # [N, B]
    quant = absx_b @ eps_w.T + eps_a @ absv_b.T
    p = oracle.block_partials(a_i8, w_i8).astype(np.float64)
    s = a_scale.astype(np.float64)[:, None, :] * w_scale.astype(np.float64)[None, :, :]
    sum_abs = np.sum(np.abs(p) * s, axis=2)
    exact_q = np.sum(p * s, axis=2)
    rnd = (nb + 2) * 2.0 ** -24 * sum_abs + 2.0 ** -8 * (np.abs(exact_q) + (nb + 2) * 2.0 ** -24 * sum_abs)
    return quant, rnd, exact_q


def _check_against_f64(a_bits, w):
    k = a_bits.shape[1]
    w_i8, w_scale = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    out = oracle.proj_rows(a_bits, w_i8, w_scale)
    got = oracle.bf16_bits_to_f32(out).astype(np.float64)
    x = _dequant_a(a_bits)
    v = oracle.dequant_nvfp4(w["w_packed"], w["w_e4m3"], w["scale2"], k).astype(np.float64)
    ref = x @ v.T
    quant, rnd, exact_q = _error_bound(a_bits, w_i8, w_scale, x, v)
    err = np.abs(got - ref)
    bound = quant + rnd
    assert np.all(err <= 1.01 * bound), float(np.max(err / np.maximum(bound, 1e-30)))
    # the rounding part alone bounds the distance to the exact dequantised int8 product
    assert np.all(np.abs(got - exact_q) <= 1.01 * rnd + 1e-45)
    return got, ref


def test_whole_oracle_vs_float64_gemm_tiny(tiny):
    got, ref = _check_against_f64(tiny["a_bits"], tiny)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.05  # sanity: int8 requant of NVFP4/BF16 is a few percent off at most


@pytest.mark.parametrize("shape,recipe", [((5, 96, 256), "laplace_zero_row"),
                                          ((7, 64, 128), "normal_outlier_channels"),
                                          ((3, 33, 64), "silu_mul")])
def test_whole_oracle_vs_float64_gemm_random(shape, recipe):
    m, n, k = shape
    w = synth.make_weight(n, k, seed=41, outlier_rows=0.05)
    a, _ = synth.make_activations(m, k, seed=42, recipe=recipe)
    _check_against_f64(a, w)


@pytest.mark.parametrize("name", ["decode", "ffn_up", "ffn_down", "square_ragged"])
def test_whole_oracle_vs_float64_gemm_workloads(name):
    # the decode workload (1 x 4096 x 4096) in full; the prefill workloads on
    # sampled outputs: sampled activation rows (ends, the ragged tail, the
    # zero row or a row with near-zero groups) against three 128-row weight
    # windows (first, last, and around an outlier row when there is one).
    # Both requantisations are row-local, so each sampled output is computed
    # exactly as in the full problem.
    d = synth.make_workload(name)
    m, n, k = d["workload"].shape
    if name == "decode":
        _check_against_f64(d["a_bits"], d)
        return
    info = d["act_info"]
    must = [info["zero_row"]] if "zero_row" in info else []
    if "near_zero_groups" in info:
        must.append(int(info["near_zero_groups"][0]) // (k // 32))
    rows = synth.sample_rows(m, 4, d["workload"].seed, must=must)
    starts = [0, n - 128] + ([int(d["outlier_rows"][0]) // 128 * 128] if len(d["outlier_rows"]) else [])
    for n0 in starts:
        w = {"w_packed": d["w_packed"][n0:n0 + 128], "w_e4m3": d["w_e4m3"][n0:n0 + 128], "scale2": d["scale2"]}
        _check_against_f64(d["a_bits"][rows], w)


def test_row_bits_independent_of_m_and_other_rows(tiny):
    k = tiny["a_bits"].shape[1]
    w_i8, w_scale = oracle.requant_w(tiny["w_packed"], tiny["w_e4m3"], tiny["scale2"], k)
    full = oracle.proj_rows(tiny["a_bits"], w_i8, w_scale)
    for r in (0, 5, 15):
        alone = oracle.proj_rows(tiny["a_bits"][r : r + 1], w_i8, w_scale)
        assert np.array_equal(alone[0], full[r])
    other = tiny["a_bits"].copy()
    rng = np.random.default_rng(0)
    other[1:] = rng.integers(0, 0x7F00, size=other[1:].shape, dtype=np.uint16)
    assert np.array_equal(oracle.proj_rows(other, w_i8, w_scale)[0], full[0])


def test_stacked_segment_bits(tiny):
    k = tiny["a_bits"].shape[1]
    full_w = oracle.requant_w(tiny["w_packed"], tiny["w_e4m3"], tiny["scale2"], k)
    full = oracle.proj_rows(tiny["a_bits"], *full_w)
    for n0, n1 in ((0, 64), (64, 200), (200, 256)):
        seg_w = oracle.requant_w(tiny["w_packed"][n0:n1], tiny["w_e4m3"][n0:n1], tiny["scale2"], k)
        assert np.array_equal(seg_w[0], full_w[0][n0:n1]) and np.array_equal(seg_w[1], full_w[1][n0:n1])
        assert np.array_equal(oracle.proj_rows(tiny["a_bits"], *seg_w), full[:, n0:n1])


def test_zero_inputs_give_zero_bits(tiny):
    k = tiny["a_bits"].shape[1]
    w_i8, w_scale = oracle.requant_w(tiny["w_packed"], tiny["w_e4m3"], tiny["scale2"], k)
    z = np.zeros_like(tiny["a_bits"])
    assert np.all(oracle.proj_rows(z, w_i8, w_scale) == 0)
    zw = oracle.requant_w(np.zeros_like(tiny["w_packed"]), tiny["w_e4m3"], tiny["scale2"], k)
    assert np.all(oracle.proj_rows(tiny["a_bits"], *zw) == 0)


def test_weight_row_permutation_permutes_columns(tiny):
    k = tiny["a_bits"].shape[1]
    perm = np.random.default_rng(4).permutation(256)
    w_i8, w_scale = oracle.requant_w(tiny["w_packed"], tiny["w_e4m3"], tiny["scale2"], k)
    out = oracle.proj_rows(tiny["a_bits"], w_i8, w_scale)
    w2 = oracle.requant_w(tiny["w_packed"][perm], tiny["w_e4m3"][perm], tiny["scale2"], k)
    assert np.array_equal(oracle.proj_rows(tiny["a_bits"], *w2), out[:, perm])


def test_power_of_two_activation_scaling(tiny):
    # scaling A by 4 (exact in BF16) scales every a_scale by 4 and keeps codes,
    # so the float32 output is scaled by exactly 4 (before BF16 rounding, which
    # commutes with powers of two)
    k = tiny["a_bits"].shape[1]
    w_i8, w_scale = oracle.requant_w(tiny["w_packed"], tiny["w_e4m3"], tiny["scale2"], k)
    x = oracle.bf16_bits_to_f32(tiny["a_bits"])
    x4 = (x * np.float32(4.0)).view(np.uint32) >> 16
    out = oracle.bf16_bits_to_f32(oracle.proj_rows(tiny["a_bits"], w_i8, w_scale))
    out4 = oracle.bf16_bits_to_f32(oracle.proj_rows(x4.astype(np.uint16), w_i8, w_scale))
    assert np.array_equal(out4, out * np.float32(4.0))


def test_w4a16_gemv_brute_force_tiny():
    # brute force over the nibbles and scales, written out per element from the
    # E2M1 / E4M3 tables, against the oracle's vectorised dequantise-and-sum
    rng = np.random.default_rng(17)
    n, k = 3, 64
    w = synth.make_weight(n, k, seed=17)
    a_bits = oracle.bf16_rne(rng.standard_normal((2, k)).astype(np.float32))
    got = oracle.bf16_bits_to_f32(oracle.w4a16_gemv(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k))
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for r in range(2):
        for j in range(n):
            total = 0.0
            for c in range(k):
                byte = int(w["w_packed"][j, c // 2])
                nib = (byte >> (4 * (c % 2))) & 0xF
                e2 = mags[nib & 7] * (-1.0 if nib & 8 else 1.0)
                s16 = float(oracle.e4m3_decode(np.array([w["w_e4m3"][j, c // 16]], dtype=np.uint8))[0])
                v = np.float32(np.float32(e2 * s16) * np.float32(w["scale2"]))
                total += float(oracle.bf16_bits_to_f32(np.array([a_bits[r, c]], dtype=np.uint16))[0]) * float(v)
            want = oracle.bf16_bits_to_f32(oracle.bf16_rne(np.array([total], dtype=np.float32)))[0]
            assert got[r, j] == want


def test_w4a16_gemv_close_to_int8_projection():
    # both read the same NVFP4 weight: the int8 projection differs from the
    # exact W4A16 product only by the requantisation errors (a few percent)
    w = synth.make_weight(64, 512, seed=18)
    a_bits, _ = synth.make_activations(4, 512, 19, "normal")
    x = oracle.bf16_bits_to_f32(oracle.w4a16_gemv(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], 512))
    y = oracle.bf16_bits_to_f32(oracle.proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], 512))
    rel = np.linalg.norm(x - y) / np.linalg.norm(x)
    assert 0 < rel < 0.05
