"""Failure path on the GPU without a fault: bsr_debug_wait_timeout queues a
kernel whose one pipeline wait (an mbarrier nothing arrives on) can never be
satisfied.  Its bounded wait must run out after the given limit, set bit 32
of the device status word and return; the context must stay usable, which the
test checks by running a projection afterwards and comparing it with the
oracle."""
import time

import pytest
import torch

import block_scaled_precision_requant_b200 as bsr
import oracle
from block_scaled_precision_requant_b200 import synth
from tests._gpu import assert_close_bf16, bf16_bits, up_bf16, weight_to_dev

pytestmark = pytest.mark.gpu


def test_wait_runs_out_reports_and_context_survives():
    assert bsr.device_status() == 0
    t0 = time.perf_counter()
    bsr.debug_wait_timeout(50)
    status = bsr.device_status()  # synchronises
    elapsed = time.perf_counter() - t0
    assert status == bsr.DEV_STATUS_DEBUG_WAIT
    assert elapsed >= 0.045, f"the wait gave up after {elapsed * 1e3:.1f} ms, before its 50 ms limit"
    assert bsr.device_status() == 0  # read-and-clear

    # the device still runs work correctly
    m, n, k = 8, 128, 256
    w = synth.make_weight(n, k, seed=91)
    w_i8, w_s = bsr.requant_w(*weight_to_dev(w))
    a_bits, _ = synth.make_activations(m, k, 92, "normal")
    out = bsr.proj(up_bf16(a_bits), w_i8, w_s)
    torch.cuda.synchronize()
    ref = oracle.proj(a_bits, w["w_packed"], w["w_e4m3"], w["scale2"], k)
    assert_close_bf16(bf16_bits(out), ref, "projection after the timed-out wait")
    assert bsr.device_status() == 0
