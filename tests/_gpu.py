"""Helpers for the GPU parity tests: upload numpy arrays, read BF16 back as
bits, and the output tolerance |gpu - ref| <= 2^-7 |ref| + 1e-3 rms(ref)."""
import numpy as np
import torch

import oracle

DEV = "cuda:0"


def up_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(DEV)


def up_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).to(DEV)


def bf16_bits(t):
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(t):
    return t.detach().cpu().numpy()


def assert_close_bf16(got_bits, ref_bits, what=""):
    got = oracle.bf16_bits_to_f32(got_bits).astype(np.float64)
    ref = oracle.bf16_bits_to_f32(ref_bits).astype(np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU output"
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    tol = 2.0 ** -7 * np.abs(ref) + 1e-3 * rms
    err = np.abs(got - ref)
    bad = err > tol
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} tol {tol[i]!r}")
    return float(np.max(err / np.maximum(tol, 1e-300))) if err.size else 0.0


def weight_to_dev(w):
    return up_u8(w["w_packed"]), up_u8(w["w_e4m3"]), float(w["scale2"])
