"""Stacked weights: each segment's columns of a stacked launch must carry
the bits a launch on that segment alone writes (the segment invariance of
w8a8_decode/parts.rs, `W8a8Weight::segment`), on the decode kernel (one
launch over all segments, also with the static-weight option and inside a
CUDA graph) and on the tensor-core route (one GEMM per segment into column
slices of one output); and the stacked output must match the oracle."""
import numpy as np
import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, up_bf16, weight_to_dev

pytestmark = pytest.mark.gpu


def _segments(ns, k, seed):
    segs, host = [], []
    for i, n in enumerate(ns):
        if n == 0:  # an empty segment: no rows, no columns in the output
            segs.append((torch.empty((0, k), dtype=torch.int8, device="cuda"),
                         torch.empty((0, k // 32), dtype=torch.float32, device="cuda")))
            host.append(None)
            continue
        w = synth.make_weight(n, k, seed=seed + i)
        segs.append(bsr.requant_w(*weight_to_dev(w)))
        host.append(w)
    return segs, host


@pytest.mark.parametrize("m,ns,k", [(1, [4096, 1024, 1024], 4096), (5, [256, 0, 130, 77], 2080),
                                    (16, [128] * 8, 512)])
def test_decode_stacked_equals_segments(m, ns, k):
    segs, host = _segments(ns, k, 51)
    a_bits, _ = synth.make_activations(m, k, 52, "normal_outlier_channels")
    a = up_bf16(a_bits)
    for sw in (False, True):
        out = bsr.decode_stacked(a, segs, static_weight=sw)
        torch.cuda.synchronize()
        off = 0
        for (w_i8, w_s), n in zip(segs, ns):
            if n:
                alone = bsr.decode(a, w_i8, w_s)
                assert torch.equal(out[:, off:off + n].view(torch.int16), alone.view(torch.int16))
            off += n
    # against the oracle on the first rows of every segment
    off = 0
    for w, n in zip(host, ns):
        if n:
            wq, ws = oracle.requant_w(w["w_packed"], w["w_e4m3"], w["scale2"], k)
            ref = oracle.proj_rows(a_bits[:2], wq[: min(n, 64)], ws[: min(n, 64)])
            assert_close_bf16(bf16_bits(out)[:2, off:off + min(n, 64)], ref, "stacked decode vs oracle")
        off += n
    assert bsr.device_status() == 0


def test_proj_stacked_tensor_core_route():
    m, ns, k = 300, [384, 128, 200], 1024
    segs, host = _segments(ns, k, 61)
    a = up_bf16(synth.make_activations(m, k, 62, "laplace_zero_row")[0])
    out = bsr.proj_stacked(a, segs)
    torch.cuda.synchronize()
    off = 0
    for (w_i8, w_s), n in zip(segs, ns):
        alone = bsr.proj(a, w_i8, w_s)
        assert torch.equal(out[:, off:off + n].view(torch.int16), alone.view(torch.int16))
        off += n
    assert bsr.device_status() == 0


def test_decode_stacked_graph_loop():
    m, ns, k = 1, [2048, 512, 512], 4096
    segs, _ = _segments(ns, k, 71)
    a = up_bf16(synth.make_activations(m, k, 72, "normal")[0])
    ref = bsr.decode_stacked(a, segs)
    outs = [torch.empty_like(ref) for _ in range(4)]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for o in outs:
            bsr.decode_stacked(a, segs, o, static_weight=True)
    g.replay()
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
    del g
    assert bsr.device_status() == 0
