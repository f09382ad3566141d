"""GPU parity of the SiLU.mul quantiser and the down projection from gate/up
against the oracle: the BF16 product, the int8 codes and the F32 scales must
be bit-exact; projection outputs within the BF16 tolerance.  Cases: tiny
ragged shapes, the whole exp range (|g| beyond 88, where exp saturates),
near-zero groups, both routes of bsr_proj_silu, and the full-size down
projection (M=8192, N=4096, K=14336) on sampled rows."""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import DEV, assert_close_bf16, bf16_bits, f32, up_bf16, weight_to_dev

pytestmark = pytest.mark.gpu


def _bf16(x):
    return oracle.bf16_rne(np.asarray(x, dtype=np.float32))


def _check_product(g_bits, u_bits):
    x = bsr.silu_mul(up_bf16(g_bits), up_bf16(u_bits))
    assert np.array_equal(bf16_bits(x), oracle.silu_mul_bf16(g_bits, u_bits))


def _check_quant(g_bits, u_bits):
    m, k = g_bits.shape
    a_i8, a_st = bsr.requant_silu_a(up_bf16(g_bits), up_bf16(u_bits))
    q, s = oracle.requant_silu_a(g_bits, u_bits)
    assert np.array_equal(a_i8.cpu().numpy(), q)
    assert np.array_equal(f32(a_st)[:, :m].T.copy().view(np.uint32), s.view(np.uint32))


@pytest.mark.parametrize("m,k", [(1, 32), (7, 96), (33, 256), (130, 512)])
def test_product_and_quantiser_random(m, k):
    g, u, _ = synth.make_gate_up(m, k, seed=m + k)
    _check_product(g, u)
    _check_quant(g, u)


def test_product_over_the_whole_exp_range():
    # g spans every BF16 magnitude class up to 1e4, both signs, including
    # |g| > 88 where exp saturates to +inf / 0, and g = +-0
    rng = np.random.default_rng(3)
    m, k = 64, 512
    mag = 10.0 ** rng.uniform(-8, 4, size=(m, k))
    g = mag * rng.choice([-1.0, 1.0], size=(m, k))
    g[0, :32] = 0.0
    g[1, :32] = -0.0
    g[2, :32] = np.linspace(-100, 100, 32)
    u = rng.standard_normal((m, k)) * 10.0 ** rng.uniform(-3, 3, size=(m, k))
    g_bits, u_bits = _bf16(g), _bf16(u)
    _check_product(g_bits, u_bits)
    _check_quant(g_bits, u_bits)


def test_quantiser_near_zero_and_zero_groups():
    m, k = 16, 1024
    g, u, info = synth.make_gate_up(m, k, seed=21)
    u = u.copy()
    u[3, 64:96] = 0  # an exactly-zero product group: scale 0, codes 0
    _check_quant(g, u)
    a_i8, a_st = bsr.requant_silu_a(up_bf16(g), up_bf16(u))
    assert f32(a_st)[2, 3] == 0.0 and np.all(a_i8.cpu().numpy()[3, 64:96] == 0)


def test_quantiser_matches_unfused_path():
    m, k = 300, 2048
    g, u, _ = synth.make_gate_up(m, k, seed=5)
    gd, ud = up_bf16(g), up_bf16(u)
    a1, s1 = bsr.requant_silu_a(gd, ud)
    a2, s2 = bsr.requant_a(bsr.silu_mul(gd, ud))
    assert torch.equal(a1, a2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))


@pytest.mark.parametrize("m", [5, 300])
def test_proj_silu_both_routes(m):
    n, k = 384, 2048
    w = synth.make_weight(n, k, seed=31)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    g, u, _ = synth.make_gate_up(m, k, seed=32 + m)
    out = bsr.proj_silu(up_bf16(g), up_bf16(u), w_i8, w_s)
    torch.cuda.synchronize()
    wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    ref = oracle.proj_rows(oracle.silu_mul_bf16(g, u), wq, ws)
    assert_close_bf16(bf16_bits(out), ref, f"proj_silu m={m}")
    assert bsr.device_status() == 0


def test_proj_silu_scratch_sizes():
    assert bsr.proj_silu_scratch_bytes(5, 2048) == 5 * 2048 * 2 + (256 - 5 * 2048 * 2 % 256) % 256
    assert bsr.proj_silu_scratch_bytes(300, 2048) == bsr.proj_scratch_bytes(300, 2048)
    assert bsr.proj_silu_scratch_bytes(300, 96) == 300 * 96 * 2  # K % 128 != 0: decode route


def test_down_projection_full_size_sampled_rows():
    wl = synth.WORKLOADS["ffn_down"]
    m, n, k = wl.shape
    w = synth.make_weight(n, k, wl.seed)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    g, u, info = synth.make_gate_up(m, k, wl.seed)
    gd, ud = up_bf16(g), up_bf16(u)
    a_i8, a_st = bsr.requant_silu_a(gd, ud)
    out = bsr.proj_silu(gd, ud, w_i8, w_s)
    torch.cuda.synchronize()
    rows = synth.sample_rows(m, 6, wl.seed, must=[int(info["near_zero_groups"][0]) // (k // 32)])
    q, s = oracle.requant_silu_a(g[rows], u[rows])
    assert np.array_equal(a_i8.cpu().numpy()[rows], q)
    assert np.array_equal(f32(a_st)[:, rows].T.copy().view(np.uint32), s.view(np.uint32))
    wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    ref = oracle.proj_rows(oracle.silu_mul_bf16(g[rows], u[rows]), wq, ws)
    assert_close_bf16(bf16_bits(out)[rows], ref, "down projection, sampled rows")
    assert bsr.device_status() == 0
