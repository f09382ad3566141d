"""Build libbsr.so in-tree with nvcc for sm_100a.

    python -m block_scaled_precision_requant_b200.build [--verbose-ptxas]

The library is a single shared object with a C ABI (include/bsr.h); it links
the CUDA runtime statically and reaches the driver API only through the
runtime's driver entry point, so it has no libcuda link-time dependency.
No fast-math flags: the quantisers depend on IEEE division, rounding and
subnormals.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libbsr.so")
SOURCES = ["api.cu", "requant.cu", "decode.cu", "gemm_tc.cu", "noalloc.cu", "debug.cu", "silu.cu", "nvfp4_gemv.cu",
           "w4a4.cu", "w4a4_gemm.cu", "host_io.cu"]
HEADERS = ["common.cuh", "quant.cuh", "kernels.h", "nvfp4_enc.cuh", "w4a4_desc.cuh", "fp_cvt.cuh", "occupancy.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "bsr.h"),
                                                                 os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES] + ["-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
