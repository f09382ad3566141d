"""The W4A4 tensor-core GEMM (block-scaled FP4 MMA, `kind::mxf4nvf4`) against
the oracle (w4a4_proj/fixed.rs, `nvfp4_proj_mx`, in this library's reading:
NVFP4 activation rows against the NVFP4 weight, exact products, one BF16
rounding).

The activation rows are quantised on the GPU by the row quantiser (bit-exact
with oracle.quantize_nvfp4_rows, tests/test_gpu_w4a4.py), both operands' E4M3
scales are rearranged into the blocked layout, then the GEMM runs.  Checks:

* one 128 x 128 x 256 tile (one stage, one tile) within the projection
  tolerance of oracle.w4a4_proj, and the status word stays 0;
* ragged M and N (tile tails on both operands), K in {256, 512, 4096};
* the decode (1 x 4096 x 4096) and FFN-up (2048 x 14336 x 4096) shapes on
  sampled output rows;
* a row's bits do not depend on M or on the other rows (the page's row
  bit-invariance); an all-zero activation row gives +0 bits;
* the composite entry (quantise rows, relayout, GEMM) equals the three
  calls made separately, bit for bit.
"""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, up_bf16, up_u8

pytestmark = pytest.mark.gpu


def _weight(n, k, seed):
    w = synth.make_weight(n, k, seed=seed)
    wp, we = up_u8(w["w_packed"]), up_u8(w["w_e4m3"])
    return w, wp, we, bsr.sf_blocked(we)


def _gemm(a_bits, wp, w_sf, scale2):
    ap, ae, as2 = bsr.quant_nvfp4_rows(up_bf16(a_bits))
    a_sf = bsr.sf_blocked(ae)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda:0")
    out = bsr.w4a4_gemm(ap, a_sf, as2, wp, w_sf, scale2, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "a pipeline wait of the W4A4 GEMM timed out"
    return bf16_bits(out)


def test_one_tile():
    m, n, k = 128, 128, 256
    w, wp, _, w_sf = _weight(n, k, seed=301)
    a_bits, _ = synth.make_activations(m, k, 302, "normal")
    got = _gemm(a_bits, wp, w_sf, float(w["scale2"]))
    ref = oracle.w4a4_proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(got, ref, "w4a4 gemm one tile")


@pytest.mark.parametrize("m,n,k", [(128, 128, 512), (129, 200, 256), (300, 131, 512), (17, 640, 4096),
                                   (256, 384, 4096), (1, 256, 256)])
def test_ragged_shapes(m, n, k):
    w, wp, _, w_sf = _weight(n, k, seed=310 + m)
    a_bits, _ = synth.make_activations(m, k, 311 + n, "normal_outlier_channels")
    got = _gemm(a_bits, wp, w_sf, float(w["scale2"]))
    ref = oracle.w4a4_proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(got, ref, f"w4a4 gemm {m}x{n}x{k}")


@pytest.mark.parametrize("name,rows", [("decode", [0]), ("ffn_up", [0, 1, 127, 128, 1000, 2047])])
def test_workload_shapes_sampled_rows(name, rows):
    d = synth.make_workload(name)
    m, n, k = d["workload"].shape
    wp, we = up_u8(d["w_packed"]), up_u8(d["w_e4m3"])
    got = _gemm(d["a_bits"], wp, bsr.sf_blocked(we), float(d["scale2"]))
    ref = oracle.w4a4_proj(d["a_bits"][rows], d["w_packed"], d["w_e4m3"], d["scale2"], k)
    assert_close_bf16(got[rows], ref, f"w4a4 gemm {name} sampled rows")


def test_row_invariance_and_zero_row():
    m, n, k = 200, 300, 1024
    w, wp, _, w_sf = _weight(n, k, seed=330)
    a_bits, _ = synth.make_activations(m, k, 331, "laplace_zero_row")
    s2 = float(w["scale2"])
    got = _gemm(a_bits, wp, w_sf, s2)
    for i in (0, 77, 128, 199):
        one = _gemm(a_bits[i:i + 1], wp, w_sf, s2)
        assert np.array_equal(one[0], got[i]), f"row {i} differs when computed alone"
    b = a_bits.copy()
    b[1:] = oracle.bf16_rne(oracle.bf16_bits_to_f32(b[1:]) * np.float32(1000.0))
    assert np.array_equal(_gemm(b, wp, w_sf, s2)[0], got[0]), "row 0 depends on the other rows"
    zr = int(np.flatnonzero(~(a_bits & 0x7FFF).any(axis=1))[0])
    assert np.all(got[zr] == 0), "an all-zero row must give +0 bits"
    ref = oracle.w4a4_proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(got, ref, "w4a4 gemm laplace rows")


def test_composite_entry_equals_three_calls():
    m, n, k = 300, 256, 1024
    w, wp, we, w_sf = _weight(n, k, seed=340)
    a_bits, _ = synth.make_activations(m, k, 341, "normal_outlier_channels")
    s2 = float(w["scale2"])
    sep = _gemm(a_bits, wp, w_sf, s2)
    got = bsr.w4a4_proj(up_bf16(a_bits), wp, w_sf, s2)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(got), sep)
    assert bsr.device_status() == 0
