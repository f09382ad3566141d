"""The W4A4 tensor-core GEMM's hardware plan against CUTLASS's CuTe, on the
host: tests/host_cute_plan.cu lets CuTe (header-only) derive, for the same
configuration (M = N = 128, K tile 256, E2M1 operands, UE4M3 scales per 16),

* the block-scaled MMA's instruction descriptor,
* the shared-memory scale layout (the blocked atoms bsr_nvfp4_sf_blocked
  writes: byte 16*r0 + 4*r1 + j + 512*kb for row r0 + 32*r1, scale j, K block kb),
* the tensor-memory placement of the scales (lane r0 + 32*rep, column
  r1 + 4*kb, byte j),
* the four tcgen05.cp copies per stage with their source descriptors and
  destination columns, and
* the operand descriptors of a 128 x 256 E2M1 tile with the 128-byte swizzle,

and each is compared with what csrc/w4a4_gemm.cu and its descriptor header
use.  Skipped where nvcc or the CUTLASS headers are missing.
"""
import importlib.util
import os
import re
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "block_scaled_precision_requant_b200", "csrc")


def _cutlass_include():
    cands = [os.environ.get("BSR_CUTLASS_INCLUDE", "")]
    for pkg in ("flashinfer", "tilelang"):
        spec = importlib.util.find_spec(pkg)
        if spec and spec.submodule_search_locations:
            root = list(spec.submodule_search_locations)[0]
            cands += [os.path.join(root, "data", "cutlass", "include"),
                      os.path.join(root, "3rdparty", "cutlass", "include")]
    for c in cands:
        if c and os.path.exists(os.path.join(c, "cute", "atom", "mma_traits_sm100.hpp")):
            return c
    return None


def _nvcc():
    for c in ("/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    return None


@pytest.fixture(scope="module")
def plan(tmp_path_factory):
    inc, nvcc = _cutlass_include(), _nvcc()
    if not inc or not nvcc:
        pytest.skip("needs nvcc and the CUTLASS/CuTe headers")
    exe = str(tmp_path_factory.mktemp("plan") / "plan")
    subprocess.run([nvcc, "-std=c++17", "-O2", "--expt-relaxed-constexpr", "-I", inc, "-I", CSRC,
                    os.path.join(HERE, "host_cute_plan.cu"), "-o", exe], check=True, capture_output=True, timeout=600)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60).stdout
    rows = {}
    for line in out.splitlines():
        parts = line.split()
        if parts and re.fullmatch(r"[a-z_]+", parts[0]) and all(re.fullmatch(r"-?\d+", p) for p in parts[1:]):
            rows.setdefault(parts[0], []).append([int(p) for p in parts[1:]])
    return rows


def test_instruction_descriptor(plan):
    assert plan["idesc_cute"] == plan["idesc_kernel"]


def test_shared_memory_scale_layout(plan):
    assert len(plan["smem_sf"]) == 4 * 5 * 4
    for row, j, kb, off in plan["smem_sf"]:
        assert off == 16 * (row % 32) + 4 * (row // 32) + j + 512 * kb


def test_tensor_memory_scale_placement(plan):
    # byte-column addressing: lane << 18 | (4 * column + byte)
    for row, rep, j, kb, off in plan["tmem_sf"]:
        lane, bytecol = off >> 18, off & ((1 << 18) - 1)
        assert lane == row % 32 + 32 * rep
        assert bytecol // 4 == row // 32 + 4 * kb and bytecol % 4 == j


def test_scale_copies_and_descriptors(plan):
    assert plan["copies"] == [[4]]
    for c, cute_desc, kernel_desc in plan["cp_desc"]:
        assert cute_desc == kernel_desc, c
    assert [d for _, d in plan["cp_dst"]] == [0, 16, 32, 48]  # 4 columns apart


def test_operand_descriptors(plan):
    # start advances 32 bytes per K = 64 MMA; LBO 1, SBO 1024 B, 128-byte
    # swizzle, version 1: the fields smem_desc_k_sw128 writes
    for kb, start, lbo, sbo, layout, version in plan["a_desc"]:
        assert (start, lbo, sbo, layout, version) == (2 * kb, 1, 64, 2, 1)
    common = open(os.path.join(CSRC, "common.cuh")).read()
    body = common[common.index("smem_desc_k_sw128"):]
    body = body[:body.index("return d;")]
    assert "(uint64_t)1 << 16" in body and "(1024u >> 4) << 32" in body
    assert "(uint64_t)1 << 46" in body and "(uint64_t)2 << 61" in body
