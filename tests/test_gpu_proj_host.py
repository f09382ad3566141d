"""bsr_proj_host: the projection with page-locked host activations and result,
pipelined over row chunks.  Each chunk's rows must carry the bits bsr_proj
writes for those rows (the same route: tensor cores, or the decode kernel
for a chunk of at most 16 rows or K % 128 != 0), within tolerance of the
oracle; pageable host memory is refused with nothing launched."""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, up_bf16, weight_to_dev

pytestmark = pytest.mark.gpu


def _host_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


def _default_rows(m):
    """The documented default: about four chunks of whole 128-row tiles, at
    least 512 rows (at most M)."""
    quarter = -(-m // 4)
    return min(m, max(512, -(-quarter // 128) * 128))


@pytest.mark.parametrize(
    "m,n,k,chunk",
    [(300, 256, 512, 128), (1040, 384, 1024, 512), (37, 200, 96, 16), (2048, 520, 4096, 0), (9, 64, 256, 0)],
)
def test_chunks_same_bits_as_proj(m, n, k, chunk):
    w = synth.make_weight(n, k, seed=71)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    a_bits, _ = synth.make_activations(m, k, 72, "laplace_zero_row")
    a_host = _host_bf16(a_bits)
    out_host = torch.zeros((m, n), dtype=torch.bfloat16).pin_memory()
    a_dev = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    out_dev = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    bsr.proj_host(a_host, w_i8, w_s, out_host, a_dev, out_dev, chunk_rows=chunk)
    torch.cuda.synchronize()
    got = out_host.view(torch.int16).numpy().view(np.uint16)
    rows = _default_rows(m) if chunk == 0 else chunk
    a = up_bf16(a_bits)
    for r0 in range(0, m, rows):
        ref = bsr.proj(a[r0:r0 + rows].contiguous(), w_i8, w_s)
        torch.cuda.synchronize()
        assert np.array_equal(got[r0:r0 + rows], ref.view(torch.int16).cpu().numpy().view(np.uint16)), r0
    sample = sorted({0, m // 2, m - 1})
    wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(got[sample], oracle.proj_rows(a_bits[sample], wq, ws), "host-buffer projection")
    assert bsr.device_status() == 0


def test_pageable_refused():
    m, n, k = 256, 64, 256
    w = synth.make_weight(n, k, seed=73)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    a_dev = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    out_dev = torch.full((m, n), 3.0, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    with pytest.raises(bsr.BsrError):
        bsr.proj_host(torch.zeros((m, k), dtype=torch.bfloat16), w_i8, w_s,
                      torch.zeros((m, n), dtype=torch.bfloat16).pin_memory(), a_dev, out_dev)
    assert "page-locked" in bsr.last_error()
    torch.cuda.synchronize()
    assert torch.all(out_dev == 3.0)
