"""Seeded synthetic inputs for the block-scaled int8 projection.

This module only *draws* inputs: an NVFP4 weight (packed E2M1 nibbles, one
E4M3 scale per 16 elements, one F32 ``scale2`` per tensor) and BF16
activations.  It holds none of the projection's own arithmetic -- no decode of
E2M1/E4M3, no int8 requantisation, no block dot products -- so that the CPU
oracle and the CUDA path can both be fed from it without sharing any code.

Weight recipe (the same for every workload):
  * ``W_f32 ~ N(0, 0.02^2)`` (float32),
  * ``scale2 = amax(W) / (6 * 448)``,
  * per 16-element block ``s16 = E4M3_RNE(amax16 / (6 * scale2))`` (saturating
    at 448),
  * per element ``code = E2M1_RNE(w / (s16 * scale2))`` with ties to the even
    mantissa, saturating at 6, sign taken from ``w`` (so -0 encodes as 0x8);
    a block whose ``s16`` is 0 gets all-zero codes,
  * two codes per byte, element ``2i`` in the low nibble.

The NVFP4 layout (``W_packed[N, K/2]``, ``W_e4m3[N, K/16]``, F32 ``scale2``)
is the one the ``requant_w_nvfp4_int8`` launcher documents on the
``gemm_dense_int8.rs`` page.  The encoder below only decides which bytes are
produced; the projection is then defined on those bytes.

Activations are float32 draws rounded to BF16 (round to nearest even) by
PyTorch's CPU conversion and returned as raw ``uint16`` bit patterns.

Every array comes from ``numpy.random.default_rng`` (PCG64).  A workload with
seed ``s`` draws its weight from stream ``2*s`` and its activations from
stream ``2*s + 1``.
"""
from __future__ import annotations

import dataclasses
import hashlib

import numpy as np

# ---------------------------------------------------------------------------
# Workloads.  Shapes are (M, N, K) of out[M, N] = A[M, K] . W[N, K]^T.
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    m: int
    n: int
    k: int
    seed: int
    act: str  # activation recipe, see make_activations
    weight_outlier_rows: float = 0.0  # fraction of weight rows scaled x100

    @property
    def shape(self):
        return (self.m, self.n, self.k)


WORKLOADS = {
    "tiny": Workload("tiny", 16, 256, 512, 0, "normal"),
    "decode": Workload("decode", 1, 4096, 4096, 1, "normal_outlier_channels"),
    "ffn_up": Workload("ffn_up", 2048, 14336, 4096, 2, "normal_outlier_channels"),
    "ffn_down": Workload("ffn_down", 8192, 4096, 14336, 3, "silu_mul"),
    "square_ragged": Workload("square_ragged", 4095, 8192, 8192, 4, "laplace_zero_row",
                              weight_outlier_rows=0.001),
}

# ---------------------------------------------------------------------------
# Encoders (generation only).
# ---------------------------------------------------------------------------

_E4M3_MAX = 448.0


def _e4m3_rne_encode_nonneg(x: np.ndarray):
    """Round non-negative values to the nearest E4M3 value (ties to even
    mantissa, saturating at 448); return (byte encoding, rounded value).

    E4M3 (OCP FP8): bias 7, 3 mantissa bits, subnormal step 2^-9, largest
    finite 448 (0x7E); 0x7F is NaN and is never produced here.
    """
    x = np.asarray(x, dtype=np.float64)
    assert np.all(x >= 0) and np.all(np.isfinite(x))
    x = np.minimum(x, _E4M3_MAX)
    out = np.zeros(x.shape, dtype=np.uint8)
    # exponent of x (x = f * 2^e, f in [0.5, 1)) -> unbiased exponent e-1
    _, e = np.frexp(x)
    e = e - 1
    normal = x >= 2.0 ** -6
    # subnormals: multiples of 2^-9
    q_sub = np.rint(x / 2.0 ** -9)  # 0..8 (8 == 2^-6, the smallest normal)
    # normals: step 2^(e-3)
    step = np.ldexp(1.0, (e - 3).astype(np.int64))
    q_norm = np.rint(x / step) * step  # may round up to 2^(e+1)
    q_norm = np.minimum(q_norm, _E4M3_MAX)
    # encode
    sub_code = np.where(q_sub >= 8, 8, q_sub).astype(np.int64)  # 8 -> exponent field 1, mantissa 0
    _, en = np.frexp(np.where(normal, q_norm, 1.0))
    en = en - 1
    mant = np.where(normal, np.rint((q_norm / np.ldexp(1.0, en.astype(np.int64)) - 1.0) * 8.0), 0)
    norm_code = ((en + 7) << 3) | mant.astype(np.int64)
    out[...] = np.where(normal, norm_code, sub_code).astype(np.uint8)
    value = np.where(normal, q_norm, q_sub * 2.0 ** -9)
    return out, value


_E2M1_THRESH = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
# index i of magnitude grid {0,.5,1,1.5,2,3,4,6}; at a threshold the even-mantissa
# neighbour wins: index 0,2,4,6 are even (mantissa bit 0), so ties go to them.
_E2M1_TIE_TO_LOWER = np.array([True, False, True, False, True, False, True])


def _e2m1_rne_index(y: np.ndarray) -> np.ndarray:
    """Magnitude index (0..7) of |y| rounded to the E2M1 grid, RNE, saturating."""
    y = np.abs(np.asarray(y, dtype=np.float64))
    idx = np.zeros(y.shape, dtype=np.uint8)
    for i, (t, lower) in enumerate(zip(_E2M1_THRESH, _E2M1_TIE_TO_LOWER)):
        idx += (y > t) if lower else (y >= t)
    return idx


def quantize_nvfp4(w: np.ndarray):
    """Encode a float32 weight [N, K] as NVFP4: (W_packed u8 [N, K/2],
    W_e4m3 u8 [N, K/16], scale2 f32)."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % 16 == 0
    amax = float(np.max(np.abs(w)))
    scale2 = np.float32(amax / (6.0 * 448.0)) if amax > 0 else np.float32(1.0)
    blocks = w.reshape(n, k // 16, 16).astype(np.float64)
    amax16 = np.max(np.abs(blocks), axis=2)
    s16_code, s16_val = _e4m3_rne_encode_nonneg(amax16 / (6.0 * float(scale2)))
    denom = s16_val * float(scale2)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(denom[..., None] > 0, blocks / denom[..., None], 0.0)
    mag = _e2m1_rne_index(y)
    sign = np.signbit(blocks).astype(np.uint8) << 3
    code = np.where(denom[..., None] > 0, mag | sign, 0).astype(np.uint8).reshape(n, k)
    packed = (code[:, 0::2] & 0xF) | ((code[:, 1::2] & 0xF) << 4)
    return packed.astype(np.uint8), s16_code.reshape(n, k // 16), np.float32(scale2)


# ---------------------------------------------------------------------------
# Drawing.
# ---------------------------------------------------------------------------


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def make_weight_f32(n: int, k: int, seed: int, outlier_rows: float = 0.0):
    rng = np.random.default_rng(2 * seed)
    w = rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.02)
    rows = np.zeros(0, dtype=np.int64)
    if outlier_rows > 0:
        cnt = max(1, int(round(n * outlier_rows)))
        rows = np.sort(rng.choice(n, cnt, replace=False))
        w[rows] *= np.float32(100.0)
    return w, rows


def make_weight(n: int, k: int, seed: int, outlier_rows: float = 0.0):
    """NVFP4 weight: dict with w_packed, w_e4m3, scale2, outlier_rows."""
    w, rows = make_weight_f32(n, k, seed, outlier_rows)
    packed, e4m3, scale2 = quantize_nvfp4(w)
    return {"w_packed": packed, "w_e4m3": e4m3, "scale2": scale2, "outlier_rows": rows}


def make_activations(m: int, k: int, seed: int, recipe: str):
    """BF16 activations [M, K] as uint16 bit patterns, plus a description dict."""
    rng = np.random.default_rng(2 * seed + 1)
    info = {"recipe": recipe}
    if recipe == "normal":
        x = rng.standard_normal((m, k), dtype=np.float32)
    elif recipe == "normal_outlier_channels":
        x = rng.standard_normal((m, k), dtype=np.float32)
        ch = np.sort(rng.choice(k, max(1, k // 100), replace=False))
        x[:, ch] *= np.float32(20.0)
        info["outlier_channels"] = ch
    elif recipe == "silu_mul":
        g = rng.standard_normal((m, k), dtype=np.float32)
        u = rng.standard_normal((m, k), dtype=np.float32)
        x = (g / (np.float32(1.0) + np.exp(-g))) * u
        del g, u
        # SiLU(g)*u alone almost never yields a whole 32-group near zero; scale
        # 0.1% of the 32-groups by 1e-6 so that such groups are present.
        groups = m * (k // 32)
        cnt = max(1, groups // 1000)
        sel = rng.choice(groups, cnt, replace=False)
        xv = x.reshape(groups, 32)
        xv[sel] *= np.float32(1e-6)
        info["near_zero_groups"] = np.sort(sel)
    elif recipe == "laplace_zero_row":
        x = rng.laplace(0.0, 1.0, size=(m, k)).astype(np.float32)
        zr = int(rng.integers(m))
        x[zr] = 0.0
        info["zero_row"] = zr
    else:
        raise ValueError(recipe)
    return _to_bf16_bits(x), info


def make_gate_up(m: int, k: int, seed: int):
    """Gate and up activations [M, K] (BF16 bit patterns) for the SiLU.mul
    quantiser, g, u ~ N(0, 1), with 0.1% of the 32-groups of u scaled by 1e-6
    so that some products form a near-zero group (the down-projection
    activation recipe).  Returns (g_bits, u_bits, info)."""
    rng = np.random.default_rng(2 * seed + 1)
    g = rng.standard_normal((m, k), dtype=np.float32)
    u = rng.standard_normal((m, k), dtype=np.float32)
    groups = m * (k // 32)
    cnt = max(1, groups // 1000)
    sel = rng.choice(groups, cnt, replace=False)
    u.reshape(groups, 32)[sel] *= np.float32(1e-6)
    return _to_bf16_bits(g), _to_bf16_bits(u), {"recipe": "gate_up", "near_zero_groups": np.sort(sel)}


def make_workload(name_or_wl, weight_only=False):
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    wt = make_weight(wl.n, wl.k, wl.seed, wl.weight_outlier_rows)
    out = {"workload": wl, **wt}
    if not weight_only:
        a, info = make_activations(wl.m, wl.k, wl.seed, wl.act)
        out["a_bits"] = a
        out["act_info"] = info
    return out


def sha256(arr: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(arr).tobytes()).hexdigest()


def sample_rows(m: int, count: int, seed: int, must=()):
    """Deterministic row sample: first row, last row, rows in ``must``, and the
    last rows of a ragged 128-row tail, then random rows up to ``count``."""
    rng = np.random.default_rng(10_000 + seed)
    rows = {0, m - 1, *[int(r) for r in must]}
    tail = m % 128
    if tail:
        rows.update(range(m - tail, min(m, m - tail + 4)))
    rest = [r for r in rng.permutation(m)[: count * 2].tolist() if r not in rows]
    for r in rest:
        if len(rows) >= count:
            break
        rows.add(r)
    return np.array(sorted(rows), dtype=np.int64)
