"""bsr_decode_ex: the static-weight option only reorders the kernel's copies
(part of the weight copies issued before the wait on the previous kernel), so outputs
must be bit-identical to bsr_decode and within tolerance of the oracle; also
run as a CUDA-graph loop over two weight copies as the benchmark does."""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, up_bf16, weight_to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,k", [(1, 4096, 4096), (3, 1000, 2080), (16, 256, 512)])
def test_static_weight_same_bits(m, n, k):
    w = synth.make_weight(n, k, seed=41)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    torch.cuda.synchronize()
    a_bits, _ = synth.make_activations(m, k, 42, "normal_outlier_channels")
    a = up_bf16(a_bits)
    ref = bsr.decode(a, w_i8, w_s)
    got = bsr.decode(a, w_i8, w_s, static_weight=True)
    torch.cuda.synchronize()
    assert torch.equal(ref.view(torch.int16), got.view(torch.int16))
    rows = list(range(min(m, 3)))
    wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(bf16_bits(got)[rows], oracle.proj_rows(a_bits[rows], wq, ws), "static-weight decode")
    assert bsr.device_status() == 0


def test_static_weight_graph_loop():
    m, n, k = 1, 2048, 4096
    w = synth.make_weight(n, k, seed=43)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    copies = [(w_i8.clone(), w_s.clone()) for _ in range(2)]
    a = up_bf16(synth.make_activations(m, k, 44, "normal")[0])
    outs = [torch.empty((m, n), dtype=torch.bfloat16, device=a.device) for _ in range(6)]
    ref = bsr.decode(a, w_i8, w_s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i, o in enumerate(outs):
            wi, si = copies[i % 2]
            bsr.decode(a, wi, si, o, static_weight=True)
    g.replay()
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
    del g
    assert bsr.device_status() == 0
