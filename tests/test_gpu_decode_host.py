"""bsr_decode_host: the decode step with the activations in, and the result
out to, page-locked host memory through copy kernels chained with the decode
kernel.  The result must be the bits bsr_decode writes (and within tolerance
of the oracle); pageable host memory is refused with nothing launched; a
CUDA-graph loop over fresh inputs per step gives each step's own result."""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, up_bf16, weight_to_dev

pytestmark = pytest.mark.gpu


def _host_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("static", [False, True])
@pytest.mark.parametrize("m,n,k", [(1, 4096, 4096), (3, 1001, 2080), (16, 256, 512), (5, 7, 32)])
def test_host_buffers_same_bits(m, n, k, static):
    w = synth.make_weight(n, k, seed=51)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    a_bits, _ = synth.make_activations(m, k, 52, "normal_outlier_channels")
    a_host = _host_bf16(a_bits)
    out_host = torch.zeros((m, n), dtype=torch.bfloat16).pin_memory()
    a_dev = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    out_dev = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    bsr.decode_host(a_host, w_i8, w_s, out_host, a_dev, out_dev, static_weight=static)
    torch.cuda.synchronize()
    ref = bsr.decode(up_bf16(a_bits), w_i8, w_s)
    torch.cuda.synchronize()
    assert torch.equal(out_host.view(torch.int16), ref.cpu().view(torch.int16))
    assert torch.equal(out_dev.view(torch.int16), ref.view(torch.int16))
    rows = list(range(min(m, 3)))
    wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    got = out_host.view(torch.int16).numpy().view(np.uint16)
    assert_close_bf16(got[rows], oracle.proj_rows(a_bits[rows], wq, ws), "host-buffer decode")
    assert bsr.device_status() == 0


def test_pageable_host_memory_refused():
    m, n, k = 1, 64, 128
    w = synth.make_weight(n, k, seed=53)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    a_dev = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    out_dev = torch.full((m, n), 7.0, dtype=torch.bfloat16, device="cuda")
    pinned = torch.zeros((m, k), dtype=torch.bfloat16).pin_memory()
    pageable = torch.zeros((m, n), dtype=torch.bfloat16)
    torch.cuda.synchronize()
    with pytest.raises(bsr.BsrError):
        bsr.decode_host(pinned, w_i8, w_s, pageable, a_dev, out_dev)
    assert "page-locked" in bsr.last_error()
    torch.cuda.synchronize()
    assert torch.all(out_dev == 7.0)  # nothing was launched


def test_host_graph_loop_fresh_inputs():
    """Each step of a captured loop reads its own pinned input and writes its
    own pinned output, as a host-driven decode loop does."""
    m, n, k, steps = 1, 2048, 4096, 5
    w = synth.make_weight(n, k, seed=54)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    bits = [synth.make_activations(m, k, 60 + i, "normal")[0] for i in range(steps)]
    a_host = [_host_bf16(b) for b in bits]
    out_host = [torch.zeros((m, n), dtype=torch.bfloat16).pin_memory() for _ in range(steps)]
    a_dev = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    out_dev = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            bsr.decode_host(a_host[i], w_i8, w_s, out_host[i], a_dev, out_dev, static_weight=True)
    g.replay()
    torch.cuda.synchronize()
    for i in range(steps):
        ref = bsr.decode(up_bf16(bits[i]), w_i8, w_s)
        torch.cuda.synchronize()
        assert torch.equal(out_host[i].view(torch.int16), ref.cpu().view(torch.int16)), i
    del g
    assert bsr.device_status() == 0
