"""GPU parity of the SiLU.mul quantiser and the down projection from gate/up
against the oracle.

The oracle's product is the mathematical silu(g) * u rounded once to BF16.
The kernel evaluates it in float32 (exp by range reduction and the hardware
base-2 exponential, an approximate quotient), so its float32 value is within
2^-20 |x| of the exact x wherever |g| <= 104.  The BF16 products must
therefore be bit-exact except (a) where the exact value lies within
2^-20 |x| of a BF16 rounding boundary, where they may differ by one BF16
step (at most 0.1% of the elements), and (b) where g is very negative
(below -104 the kernel's product is a signed zero; the test allows it from
-88 on).  The int8 codes and
F32 scales must be bit-exact against oracle.requant_a of the kernel's own
product, and against oracle.requant_silu_a in every group whose 32 products
agree.  Projection outputs within the BF16 tolerance.  Cases: tiny ragged
shapes, the whole exp range (|g| beyond 88), near-zero groups, both routes
of bsr_proj_silu, and the full-size down projection (M=8192, N=4096,
K=14336) on sampled rows."""
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


def _exact_product(g_bits, u_bits):
    g = oracle.bf16_bits_to_f32(g_bits).astype(np.float64)
    u = oracle.bf16_bits_to_f32(u_bits).astype(np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        return g / (1.0 + np.exp(-g)) * u, g


def _near_boundary(x, ref_bits, rel=2.0 ** -20):
    """True where x lies within rel * |x| of the BF16 rounding boundary
    between ref_bits (its rounding) and the BF16 neighbour on x's side."""
    v = oracle.bf16_bits_to_f32(ref_bits).astype(np.float64)
    mag = ref_bits & 0x7FFF
    away = np.abs(x) > np.abs(v)
    nb = np.where(away, np.minimum(mag + 1, 0x7F80), np.maximum(mag.astype(np.int32) - 1, 0)).astype(np.uint16)
    other = np.abs(oracle.bf16_bits_to_f32(nb).astype(np.float64))
    boundary = (np.abs(v) + other) / 2
    return np.abs(np.abs(x) - boundary) <= rel * np.abs(x)


def _check_product_bits(g_bits, u_bits, got, max_frac=1e-3):
    """Kernel product bits `got` against the exact product; returns the
    oracle's bits.  At most max_frac of the products may differ."""
    ref = oracle.silu_mul_bf16(g_bits, u_bits)
    diff = got != ref
    if np.any(diff):
        x, g = _exact_product(g_bits, u_bits)
        saturated = diff & (g < -88.0)
        assert np.all((got[saturated] & 0x7FFF) == 0), "g < -88: the kernel's product is a signed zero"
        rest = diff & ~saturated
        same_sign = (got[rest] & 0x8000) == (ref[rest] & 0x8000)
        one_step = np.abs((got[rest] & 0x7FFF).astype(np.int32) - (ref[rest] & 0x7FFF).astype(np.int32)) == 1
        assert np.all(same_sign & one_step), "a product differs by more than one BF16 step"
        assert np.all(_near_boundary(x[rest], ref[rest])), "a product differs away from a rounding boundary"
        assert rest.sum() <= max(1, max_frac * got.size), f"{int(rest.sum())} of {got.size} products differ"
    return ref


def _check_quant_arrays(g_bits, u_bits, x_gpu, q_gpu, s_gpu, max_frac=1e-3):
    """Codes q_gpu [m, K] and scales s_gpu [m, K/32] of the fused quantiser,
    given the kernel's product bits x_gpu: bit-exact against requant_a of
    that product, and against the oracle's quantiser wherever a group's 32
    products agree with the exact product.  Returns the agreeing fraction."""
    m, k = g_bits.shape
    ref = _check_product_bits(g_bits, u_bits, x_gpu, max_frac)
    q, s = oracle.requant_a(x_gpu)
    assert np.array_equal(q_gpu, q)
    assert np.array_equal(s_gpu.view(np.uint32), s.view(np.uint32))
    q_r, s_r = oracle.requant_silu_a(g_bits, u_bits)
    agree = np.all((x_gpu == ref).reshape(m, k // 32, 32), axis=2)
    assert np.array_equal(s_gpu.view(np.uint32)[agree], s_r.view(np.uint32)[agree])
    assert np.array_equal(q_gpu.reshape(m, k // 32, 32)[agree], q_r.reshape(m, k // 32, 32)[agree])
    return float(agree.mean())


def _check_quant(g_bits, u_bits, max_frac=1e-3):
    m, k = g_bits.shape
    gd, ud = up_bf16(g_bits), up_bf16(u_bits)
    x_gpu = bf16_bits(bsr.silu_mul(gd, ud))
    a_i8, a_st = bsr.requant_silu_a(gd, ud)
    agree = _check_quant_arrays(g_bits, u_bits, x_gpu, a_i8.cpu().numpy(), f32(a_st)[:, :m].T.copy(), max_frac)
    assert agree > 0.9


@pytest.mark.parametrize("m,k", [(1, 32), (7, 96), (33, 256), (130, 512), (512, 4096)])
def test_product_and_quantiser_random(m, k):
    g, u, _ = synth.make_gate_up(m, k, seed=m + k)
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
    # Here many products sit exactly on a BF16 midpoint: for 16.6 < g < 36.7
    # the kernel's 1 + e^-g rounds to 1 in float32, so its product is the
    # exact g * u of two BF16 values, often a tie, while the exact product
    # lies just below it.  Those are boundary cases too; allow 0.5%.
    _check_quant(g_bits, u_bits, max_frac=5e-3)


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


def test_down_projection_full_size():
    """Product, codes and scales of the whole 8192 x 14336 activation
    (in row chunks), outputs of 64 sampled rows."""
    wl = synth.WORKLOADS["ffn_down"]
    m, n, k = wl.shape
    w = synth.make_weight(n, k, wl.seed)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    g, u, info = synth.make_gate_up(m, k, wl.seed)
    gd, ud = up_bf16(g), up_bf16(u)
    a_i8, a_st = bsr.requant_silu_a(gd, ud)
    x = bsr.silu_mul(gd, ud)
    out = bsr.proj_silu(gd, ud, w_i8, w_s)
    torch.cuda.synchronize()
    step = 512
    for r0 in range(0, m, step):
        r1 = min(m, r0 + step)
        _check_quant_arrays(g[r0:r1], u[r0:r1], bf16_bits(x[r0:r1]), a_i8[r0:r1].cpu().numpy(),
                            f32(a_st[:, r0:r1]).T.copy())
    near_zero_row = int(info["near_zero_groups"][0]) // (k // 32)
    rows = synth.sample_rows(m, 64, wl.seed, must=[0, m - 1, near_zero_row])
    wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    ref = oracle.proj_rows(oracle.silu_mul_bf16(g[rows], u[rows]), wq, ws)
    assert_close_bf16(bf16_bits(out)[rows], ref, "down projection, sampled rows")
    assert bsr.device_status() == 0
