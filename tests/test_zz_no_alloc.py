"""bsr_proj_noalloc: the projection for callers that cannot allocate device
memory when they call it (a runtime that plans its device memory ahead and
passes only inputs and outputs, or code where cudaMalloc is not allowed).
Its activation scratch is an array inside the library.

Called through the C ABI (ctypes) and compared with bsr_proj -- the entry
point that takes caller scratch and runs the same kernels -- bit for bit, on
two calls in a row with different activations (the second call reuses the
array the first one filled), and with the CPU oracle within the projection's
output tolerance.  One shape fills the array almost to its limit
(M=3584, K=4096).  A shape needing more than the array returns BSR_ESCRATCH
and writes nothing.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, up_bf16, weight_to_dev

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 16 << 20  # BSR_NOALLOC_SCRATCH_BYTES in include/bsr.h


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(a, w_i8, w_s, out):
    m, k = a.shape
    n = w_i8.shape[0]
    L = bsr.lib()
    st = L.bsr_proj_noalloc(_ptr(a), _ptr(w_i8), _ptr(w_s), _ptr(out), m, n, k,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _two_calls(m, n, k, seed, oracle_rows):
    w = synth.make_weight(n, k, seed=seed)
    wp, we, s2 = weight_to_dev(w)
    w_i8, w_s = bsr.requant_w(wp, we, s2)
    wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert 0 < bsr.proj_scratch_bytes(m, k) <= NOALLOC_BYTES
    for call, aseed in enumerate((seed + 1, seed + 2)):
        a_bits, _ = synth.make_activations(m, k, aseed, "laplace_zero_row")
        a = up_bf16(a_bits)
        ref = bsr.proj(a, w_i8, w_s)  # caller-scratch entry point, same kernels
        out = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=a.device)
        assert _noalloc(a, w_i8, w_s, out) == 0, bsr.last_error()
        torch.cuda.synchronize()
        got = bf16_bits(out)
        assert np.array_equal(got, bf16_bits(ref)), f"noalloc call {call}: bits differ from bsr_proj"
        rows = synth.sample_rows(m, oracle_rows, aseed)
        assert_close_bf16(got[rows], oracle.proj_rows(a_bits[rows], wq, ws), f"noalloc call {call} vs oracle")
    assert bsr.device_status() == 0


def test_noalloc_matches_proj_on_two_calls():
    _two_calls(300, 384, 2048, seed=71, oracle_rows=300)


def test_noalloc_near_the_array_limit():
    m, k = 3584, 4096  # 14 MiB of codes + 1.75 MiB of scales: 15.75 of 16 MiB
    assert bsr.proj_scratch_bytes(m, k) > NOALLOC_BYTES - (1 << 20)
    _two_calls(m, 512, k, seed=76, oracle_rows=8)


def test_noalloc_decode_rows_match_proj():
    m, n, k = 5, 256, 1024
    w = synth.make_weight(n, k, seed=74)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    a = up_bf16(synth.make_activations(m, k, 75, "normal")[0])
    out = torch.empty((m, n), dtype=torch.bfloat16, device=a.device)
    assert _noalloc(a, w_i8, w_s, out) == 0, bsr.last_error()
    assert np.array_equal(bf16_bits(out), bf16_bits(bsr.proj(a, w_i8, w_s))), "noalloc decode rows"


def test_noalloc_rejects_shapes_beyond_the_array():
    m, n, k = 4096, 128, 4096  # needs 16 MiB + 2 MiB of scratch
    assert bsr.proj_scratch_bytes(m, k) > NOALLOC_BYTES
    a = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    w_i8 = torch.zeros((n, k), dtype=torch.int8, device="cuda")
    w_s = torch.zeros((n, k // 32), dtype=torch.float32, device="cuda")
    out = torch.full((m, n), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(a, w_i8, w_s, out) == 4  # BSR_ESCRATCH, nothing launched
    assert "BSR_NOALLOC_SCRATCH_BYTES" in bsr.last_error()
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
