"""The W4A4 kernels' NVFP4 encoders (csrc/nvfp4_enc.cuh), compiled for the
host with g++, against the CPU oracle and PyTorch -- no GPU needed:

* E4M3: every 64th float32 in [0, 464] plus every E4M3 midpoint and its
  float32 neighbours against PyTorch's float8_e4m3fn cast; saturation above
  it; the value of every non-NaN code against the oracle's decoder;
* E2M1: every 256th float32 in [-8, 8] plus every midpoint and its
  neighbours, and +-0, against oracle.e2m1_encode_rne;
* the row quantiser (same order as the kernels) against
  oracle.quantize_nvfp4_rows bit for bit: random rows with outlier channels,
  a zero row, -0 entries, rows whose float32 quotients land on midpoints,
  subnormal BF16 rows (scale2 subnormal), rows near the BF16 maximum, and
  the hand-derived rows of tests/golden/w4a4_rows.txt.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_requant_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "block_scaled_precision_requant_b200", "csrc")

pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = tmp_path_factory.mktemp("nvfp4") / "libhostenc.so"
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                    "-I", CSRC, os.path.join(HERE, "host_nvfp4_enc.cpp"), "-o", str(out)], check=True)
    so = ctypes.CDLL(str(out))
    p = ctypes.c_void_p
    for name, args in {"h_e4m3_rne": [p, p, ctypes.c_long], "h_e4m3_value": [p, p, ctypes.c_long],
                       "h_e2m1_rne": [p, p, ctypes.c_long],
                       "h_quant_rows": [p, ctypes.c_long, ctypes.c_long, p, p, p]}.items():
        getattr(so, name).argtypes = args
        getattr(so, name).restype = None
    return so


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _e4m3(lib, t):
    t = np.ascontiguousarray(t, dtype=np.float32)
    out = np.empty(t.shape, dtype=np.uint8)
    lib.h_e4m3_rne(_ptr(t), _ptr(out), t.size)
    return out


def _e2m1(lib, y):
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, dtype=np.uint8)
    lib.h_e2m1_rne(_ptr(y), _ptr(out), y.size)
    return out


def _quant_rows(lib, a_bits):
    a = np.ascontiguousarray(a_bits, dtype=np.uint16)
    m, k = a.shape
    packed = np.empty((m, k // 2), dtype=np.uint8)
    e4 = np.empty((m, k // 16), dtype=np.uint8)
    s2 = np.empty(m, dtype=np.float32)
    lib.h_quant_rows(_ptr(a), m, k, _ptr(packed), _ptr(e4), _ptr(s2))
    return packed, e4, s2


def _neighbours(v):
    v = np.asarray(v, dtype=np.float32)
    return np.concatenate([v, np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(0))])


def test_e4m3_encoder_vs_torch_cast(lib):
    hi = np.float32(464.0).view(np.uint32)
    x = np.arange(0, int(hi) + 1, 64, dtype=np.uint32).view(np.float32)
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, _neighbours(mids), _neighbours(vals.astype(np.float32)), [np.float32(464.0)]])
    x = x[(x >= 0) & (x <= 464)]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(_e4m3(lib, x), want)


def test_e4m3_encoder_saturates_and_decodes(lib):
    assert np.all(_e4m3(lib, np.array([448.0, 464.0, 465.0, 1e6, 3e38, np.inf])) == 0x7E)
    codes = np.arange(0x7F, dtype=np.uint8)
    got = np.empty(codes.shape, dtype=np.float32)
    lib.h_e4m3_value(_ptr(codes), _ptr(got), codes.size)
    assert np.array_equal(got, oracle.e4m3_decode(codes))


def test_e2m1_encoder_vs_oracle(lib):
    hi = np.float32(8.0).view(np.uint32)
    pos = np.arange(0, int(hi) + 1, 256, dtype=np.uint32).view(np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0], dtype=np.float32)
    y = np.concatenate([pos, -pos, _neighbours(mids), -_neighbours(mids), [np.float32(0.0), np.float32(-0.0), 1e30, -1e30]])
    assert np.array_equal(_e2m1(lib, y), oracle.e2m1_encode_rne(y))


def _bf16(x):
    return oracle.bf16_rne(np.asarray(x, dtype=np.float32))


def _assert_rows_equal(lib, a_bits):
    p, e, s = _quant_rows(lib, a_bits)
    rp, re_, rs = oracle.quantize_nvfp4_rows(a_bits)
    assert np.array_equal(s.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(e, re_)
    assert np.array_equal(p, rp)


def test_row_quantiser_random_rows(lib):
    a, _ = synth.make_activations(48, 1024, 11, "normal_outlier_channels")
    _assert_rows_equal(lib, a)
    a, _ = synth.make_activations(17, 4096, 12, "laplace_zero_row")
    _assert_rows_equal(lib, a)


def test_row_quantiser_special_rows(lib):
    rng = np.random.default_rng(5)
    k = 256
    rows = [
        np.zeros(k),                                          # zero row
        np.where(rng.random(k) < 0.5, -0.0, 0.0),             # +-0 only
        np.concatenate([np.zeros(16), rng.standard_normal(k - 16)]),  # a zero block
        rng.standard_normal(k) * 1e-39,                       # subnormal BF16 values
        rng.standard_normal(k) * 1e-42,                       # deep subnormals: scale2 underflows
        rng.uniform(-1.0, 1.0, k) * 3.3e38,                   # near the BF16 maximum (finite)
        np.full(k, -1.0),                                     # constant row
        np.tile([6.0, -3.0, 0.5, -0.25, 1e-3, 4.0, -2.0, 1.0], k // 8),
    ]
    a = _bf16(np.stack(rows))
    a[1] = np.where(rng.random(k) < 0.5, 0x8000, 0).astype(np.uint16)  # exact -0 bit patterns
    a[6, ::7] = 0x8000  # -0 inside non-zero blocks: code 0x8
    _assert_rows_equal(lib, a)
    codes = oracle.unpack_nvfp4(_quant_rows(lib, a)[0], k)
    assert np.all(codes[6, ::7] == 0x8)


def test_row_quantiser_on_float32_midpoints(lib):
    # rows where float32 quotients land on E2M1 / E4M3 midpoints (found by
    # the oracle's own tie test on these seeds)
    for seed in (3, 10):
        a, _ = synth.make_activations(32, 1024, seed, "normal_outlier_channels")
        _assert_rows_equal(lib, a)


def test_row_quantiser_hand_derived_rows(lib):
    from tests.test_oracle_w4a4 import golden_rows

    for name, bits, s2, e4, codes in golden_rows():
        p, e, s = _quant_rows(lib, bits)
        assert s[0] == s2 and np.array_equal(e[0], e4), name
        assert np.array_equal(oracle.unpack_nvfp4(p, bits.shape[1])[0], codes), name
