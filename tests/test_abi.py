"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every function include/bsr.h declares with the binding's signatures, and
rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

import block_scaled_precision_requant_b200 as bsr
from block_scaled_precision_requant_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsr.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return bsr.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bsr_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_what_binding_wraps():
    assert _declared() == sorted(name for name, _, _ in bsr.SIGNATURES)


def _header_defines():
    src = open(HEADER).read()
    out = {}
    for name, val in re.findall(r"^#define (BSR_[A-Z0-9_]+) (.+)$", src, flags=re.M):
        val = re.sub(r"(?<=\d)(u|LL|ULL)\b", "", val.split("/*")[0].strip())
        if re.fullmatch(r"\d+", val):
            out[name] = int(val)
        elif m := re.fullmatch(r"\((\d+) << (\d+)\)", val):
            out[name] = int(m.group(1)) << int(m.group(2))
    return out


def test_header_constants_match_the_binding(L):
    # the binding restates a few header constants; they must agree (the
    # reference's one test checks the same for its kernel constants)
    d = _header_defines()
    assert d["BSR_ABI_VERSION"] == bsr.abi_version()
    assert d["BSR_DECODE_MAX_M"] == bsr.DECODE_MAX_M
    assert d["BSR_DECODE_STATIC_WEIGHT"] == bsr.DECODE_STATIC_WEIGHT
    assert d["BSR_MAX_SEGMENTS"] == bsr.MAX_SEGMENTS
    assert d["BSR_MAX_DIM"] == 2 ** 31 - 1
    assert d["BSR_NOALLOC_SCRATCH_BYTES"] == 16 << 20
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    enum = dict((int(v), "BSR_" + k) for k, v in re.findall(r"\bBSR_([A-Z]+) = (\d+)", src))
    assert enum == bsr.STATUS_NAMES
    common = open(os.path.join(ROOT, "block_scaled_precision_requant_b200", "csrc", "common.cuh")).read()
    assert int(re.search(r"DEV_ERR_TIMEOUT_DEBUG = (\d+)", common).group(1)) == bsr.DEV_STATUS_DEBUG_WAIT


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_abi_version(L):
    assert bsr.abi_version() == 1


def test_scratch_and_ld(L):
    assert bsr.a_scale_ld(1) == 4 and bsr.a_scale_ld(4) == 4 and bsr.a_scale_ld(4095) == 4096
    assert bsr.proj_scratch_bytes(16, 4096) == 0  # decode path needs none
    assert bsr.proj_scratch_bytes(17, 96) == 0  # K % 128 != 0: decode kernel serves it
    m, k = 4095, 8192
    codes = (m * k + 255) // 256 * 256
    assert bsr.proj_scratch_bytes(m, k) == codes + (k // 32) * 4096 * 4


P = ctypes.c_void_p


def _fake(addr):
    return P(addr)


def test_shape_errors_before_launch(L):
    s = L.bsr_proj(_fake(256), _fake(256), _fake(256), _fake(256), 4, 8, 48, None, 0, None)
    assert s == 3 and "multiple of 32" in bsr.last_error()
    assert L.bsr_gemm(_fake(256), _fake(256), _fake(256), _fake(256), _fake(256), 256, 256, 96, None) == 3
    assert L.bsr_requant_w(_fake(256), _fake(256), ctypes.c_float(1.0), _fake(256), _fake(256), 4, 0, None) == 3


def test_invalid_and_alignment_errors(L):
    assert L.bsr_proj(None, _fake(256), _fake(256), _fake(256), 4, 8, 64, None, 0, None) == 1
    assert L.bsr_proj(_fake(256), _fake(256), _fake(256), _fake(256), -1, 8, 64, None, 0, None) == 1
    assert L.bsr_requant_a(_fake(264), _fake(256), _fake(256), 4, 64, None) == 2
    assert L.bsr_gemm(_fake(256), _fake(256), _fake(256), _fake(256), _fake(257), 256, 256, 128, None) == 2
    assert L.bsr_gemm_partials(_fake(256), _fake(256), _fake(256), _fake(256), _fake(256), None, 4, 4, 128,
                               None) == 1


def test_debug_wait_limit_checked_before_launch(L):
    assert L.bsr_debug_wait_timeout(0, None) == 1
    assert L.bsr_debug_wait_timeout(2001, None) == 1
    assert "limit_ms" in bsr.last_error()


def test_decode_ex_rejects_unknown_flags(L):
    assert L.bsr_decode_ex(_fake(256), _fake(256), _fake(256), _fake(256), 1, 8, 64, 2, None) == 1
    assert "flags" in bsr.last_error()


def test_nvfp4_gemv_ex_argument_errors(L):
    f = ctypes.c_float(1.0)
    for entry in (L.bsr_w4a16_decode_ex, L.bsr_w4a4_decode_ex):
        assert entry(_fake(256), _fake(256), _fake(256), f, _fake(256), 1, 8, 64, 2, None) == 1
        assert "flags" in bsr.last_error()
        assert entry(None, None, None, f, None, 0, 8, 64, 1, None) == 0
    assert L.bsr_w4a16_decode_ex(_fake(256), _fake(256), _fake(256), f, _fake(256), 1, 8, 48, 0, None) == 3
    assert L.bsr_w4a16_decode_ex(_fake(264), _fake(256), _fake(256), f, _fake(256), 1, 8, 64, 1, None) == 2


def test_decode_host_argument_errors(L):
    ok = _fake(256)
    assert L.bsr_decode_host(ok, ok, ok, ok, 1, 8, 64, ok, ok, 2, None) == 1
    assert "flags" in bsr.last_error()
    assert L.bsr_decode_host(None, None, None, None, 0, 8, 64, None, None, 0, None) == 0
    assert L.bsr_decode_host(ok, ok, ok, ok, 1, 8, 48, ok, ok, 0, None) == 3
    assert L.bsr_decode_host(None, ok, ok, ok, 1, 8, 64, ok, ok, 0, None) == 1
    assert L.bsr_decode_host(ok, ok, ok, ok, 1, 8, 64, None, ok, 0, None) == 1
    assert L.bsr_decode_host(_fake(264), ok, ok, ok, 1, 8, 64, ok, ok, 0, None) == 2
    assert L.bsr_decode_host(ok, ok, ok, _fake(264), 1, 8, 64, ok, ok, 0, None) == 2
    assert L.bsr_decode_host(ok, ok, ok, ok, 1, 8, 64, ok, _fake(258), 0, None) == 2


def test_proj_host_argument_errors(L):
    ok = _fake(256)
    # scratch sizes: one chunk's bsr_proj scratch; none for the decode route
    assert L.bsr_proj_host_scratch_bytes(8192, 4096, 1024) == L.bsr_proj_scratch_bytes(1024, 4096)
    assert L.bsr_proj_host_scratch_bytes(8192, 4096, 0) == L.bsr_proj_scratch_bytes(2048, 4096)
    assert L.bsr_proj_host_scratch_bytes(16, 4096, 0) == 0
    assert L.bsr_proj_host_scratch_bytes(100000, 4096, 8) == L.bsr_proj_scratch_bytes(1563, 4096)  # <= 64 chunks
    args = (ok, ok, ok, ok, 4096, 64, 256, ok, ok)
    assert L.bsr_proj_host(*args, ok, 1 << 30, -1, None) == 1
    assert L.bsr_proj_host(None, None, None, None, 0, 64, 256, None, None, None, 0, 0, None) == 0
    assert L.bsr_proj_host(ok, ok, ok, ok, 4096, 64, 48, ok, ok, ok, 1 << 30, 0, None) == 3
    assert L.bsr_proj_host(None, ok, ok, ok, 4096, 64, 256, ok, ok, ok, 1 << 30, 0, None) == 1
    assert L.bsr_proj_host(*args, None, 0, 0, None) == 4
    assert L.bsr_proj_host(*args, _fake(272), 1 << 30, 0, None) == 2


def test_stacked_argument_errors(L):
    arr = (ctypes.c_void_p * 1)(_fake(256).value)
    n1 = (ctypes.c_int64 * 1)(8)
    assert L.bsr_decode_stacked(_fake(256), arr, arr, n1, 0, _fake(256), 1, 64, 0, None) == 1
    assert "num_segs" in bsr.last_error()
    assert L.bsr_decode_stacked(_fake(256), arr, arr, n1, 9, _fake(256), 1, 64, 0, None) == 1
    assert L.bsr_proj_stacked(_fake(256), None, arr, n1, 1, _fake(256), 1, 64, None, 0, None) == 1
    bad = (ctypes.c_void_p * 1)(_fake(264).value)
    assert L.bsr_decode_stacked(_fake(256), bad, arr, n1, 1, _fake(256), 1, 64, 0, None) == 2
    neg = (ctypes.c_int64 * 1)(-1)
    assert L.bsr_decode_stacked(_fake(256), arr, arr, neg, 1, _fake(256), 1, 64, 0, None) == 1
    assert L.bsr_decode_stacked(_fake(256), arr, arr, n1, 1, _fake(256), 1, 64, 4, None) == 1


def test_w4a4_argument_errors(L):
    f = ctypes.c_float(1.0)
    assert L.bsr_w4a4_decode(_fake(256), _fake(256), _fake(256), f, _fake(256), 1, 8, 40, None) == 3
    assert "multiple of 16" in bsr.last_error()
    assert L.bsr_w4a4_decode(_fake(256), _fake(256), _fake(256), f, _fake(256), 1, 8, 0, None) == 3
    assert L.bsr_w4a4_decode(_fake(256), _fake(256), _fake(256), f, _fake(256), 1, -1, 48, None) == 1
    assert L.bsr_w4a4_decode(None, _fake(256), _fake(256), f, _fake(256), 1, 8, 48, None) == 1
    assert L.bsr_w4a4_decode(_fake(264), _fake(256), _fake(256), f, _fake(256), 1, 8, 48, None) == 2
    assert L.bsr_w4a4_decode(_fake(256), _fake(256), _fake(256), f, _fake(257), 1, 8, 48, None) == 2
    assert L.bsr_w4a4_decode(None, None, None, f, None, 0, 8, 48, None) == 0
    assert L.bsr_w4a4_decode(None, None, None, f, None, 3, 0, 48, None) == 0
    assert L.bsr_nvfp4_quant_rows(_fake(256), _fake(256), _fake(256), _fake(256), 2, 24, None) == 3
    assert L.bsr_nvfp4_quant_rows(_fake(256), _fake(256), _fake(256), _fake(260), 2, 32, None) == 2
    assert L.bsr_nvfp4_quant_rows(_fake(256), None, _fake(256), _fake(256), 2, 32, None) == 1
    assert L.bsr_nvfp4_quant_rows(None, None, None, None, 0, 32, None) == 0


def test_w4a4_gemm_argument_errors(L):
    f = ctypes.c_float(1.0)
    assert L.bsr_nvfp4_sf_blocked_bytes(1, 64) == 512
    assert L.bsr_nvfp4_sf_blocked_bytes(129, 256) == 2 * 4 * 512
    assert L.bsr_nvfp4_sf_blocked_bytes(128, 96) == 0 and L.bsr_nvfp4_sf_blocked_bytes(0, 64) == 0
    assert L.bsr_nvfp4_sf_blocked(_fake(256), _fake(256), 4, 96, None) == 3
    assert L.bsr_nvfp4_sf_blocked(_fake(256), _fake(264), 4, 64, None) == 2
    assert L.bsr_nvfp4_sf_blocked(None, _fake(256), 4, 64, None) == 1
    assert L.bsr_nvfp4_sf_blocked(None, None, 0, 64, None) == 0
    args = [_fake(256)] * 5
    assert L.bsr_w4a4_gemm(*args, f, _fake(256), 4, 8, 128, _fake(256), None) == 3
    assert "multiple of 256" in bsr.last_error()
    assert L.bsr_w4a4_gemm(*args, f, _fake(256), 4, -8, 256, _fake(256), None) == 1
    assert L.bsr_w4a4_gemm(*args, f, _fake(256), 4, 8, 256, None, None) == 1
    assert L.bsr_w4a4_gemm(*args[:4], _fake(264), f, _fake(256), 4, 8, 256, _fake(256), None) == 2
    assert L.bsr_w4a4_gemm(None, None, None, None, None, f, None, 0, 8, 256, None, None) == 0


def test_w4a4_proj_argument_errors(L):
    f = ctypes.c_float(1.0)
    m, k = 64, 512
    need = L.bsr_w4a4_proj_scratch_bytes(m, k)
    # packed codes, E4M3 bytes, blocked scales, row scales, each 256-aligned
    assert need == 16384 + 2048 + 4096 + 256
    assert L.bsr_w4a4_proj_scratch_bytes(m, 320) == 0 and L.bsr_w4a4_proj_scratch_bytes(0, k) == 0
    a4 = [_fake(256)] * 3
    assert L.bsr_w4a4_proj(*a4, f, _fake(256), m, 8, 320, _fake(256), need, None) == 3
    assert L.bsr_w4a4_proj(*a4, f, _fake(256), m, 8, k, None, 0, None) == 4
    assert L.bsr_w4a4_proj(*a4, f, _fake(256), m, 8, k, _fake(256), need - 1, None) == 4
    assert L.bsr_w4a4_proj(*a4, f, _fake(256), m, 8, k, _fake(272), need, None) == 2
    assert L.bsr_w4a4_proj(*a4, f, _fake(264), m, 8, k, _fake(256), need, None) == 2
    assert L.bsr_w4a4_proj(None, *a4[:2], f, _fake(256), m, 8, k, _fake(256), need, None) == 1
    assert L.bsr_w4a4_proj(None, None, None, f, None, 0, 8, k, None, 0, None) == 0


def test_gemm_block_m_needs_a_device(L):
    # informational query: 0 for invalid sizes, and without a usable device
    assert L.bsr_gemm_block_m(0, 8) == 0 and L.bsr_gemm_block_m(8, -1) == 0


def test_scratch_errors(L):
    m, k = 64, 256
    need = L.bsr_proj_scratch_bytes(m, k)
    assert need > 0
    assert L.bsr_proj(_fake(256), _fake(256), _fake(256), _fake(256), m, 8, k, None, 0, None) == 4
    assert L.bsr_proj(_fake(256), _fake(256), _fake(256), _fake(256), m, 8, k, _fake(256), need - 1, None) == 4
    assert L.bsr_proj(_fake(256), _fake(256), _fake(256), _fake(256), m, 8, k, _fake(272), need, None) == 2


def test_empty_is_noop(L):
    # M == 0 or N == 0 returns OK without touching any pointer or device
    assert L.bsr_proj(None, None, None, None, 0, 8, 64, None, 0, None) == 0
    assert L.bsr_proj(None, None, None, None, 4, 0, 64, None, 0, None) == 0
    assert L.bsr_requant_w(None, None, ctypes.c_float(1.0), None, None, 0, 64, None) == 0
    assert L.bsr_requant_a(None, None, None, 0, 64, None) == 0
    assert L.bsr_gemm(None, None, None, None, None, 0, 4, 128, None) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(bsr, "_lib", None)
    monkeypatch.setattr(bsr, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        bsr.lib()
