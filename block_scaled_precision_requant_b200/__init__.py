"""Block-scaled int8 projection for NVIDIA B200 (sm_100a).

Thin ctypes binding over the C ABI of ``libbsr.so`` (declared in
``include/bsr.h``).  The functions here only marshal arguments: they check
dtypes, shapes and devices of ``torch.Tensor`` arguments, take raw device
pointers and the current CUDA stream, and call the library; every step of the
computation runs in the library's CUDA kernels.  PyTorch is used for device
memory and streams only.  There is no CPU fallback: if the library cannot be
loaded, every call raises.

Operations (gemm_dense_int8.rs launcher page):

* :func:`requant_w` -- ``requant_w_nvfp4_int8``: NVFP4 weight -> int8 codes +
  one F32 scale per 32 elements (scale2 folded in).
* :func:`requant_a` -- ``requant_a_kernel``: BF16 activations -> int8 codes +
  block-major F32 scales.
* :func:`gemm` -- ``faith2_kernel``: tcgen05 int8 GEMM with per-32-block
  rescale, F32 accumulation, BF16 output.
* :func:`proj` -- ``int8_gemm_faith2_prefill``: the whole projection from BF16
  activations (decode kernel for M <= 16, requant_a + gemm otherwise).
* :func:`silu_mul`, :func:`requant_silu_a`, :func:`proj_silu` -- the SiLU.mul
  quantiser (``W8a8Kernels::quant_silu``) and the down projection from gate
  and up activations.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "BsrError",
    "lib",
    "abi_version",
    "last_error",
    "device_status",
    "requant_w",
    "a_scale_ld",
    "requant_a",
    "gemm",
    "gemm_partials",
    "proj_scratch_bytes",
    "proj",
    "decode",
    "DECODE_MAX_M",
    "DECODE_STATIC_WEIGHT",
    "STATUS_NAMES",
    "DEV_STATUS_DEBUG_WAIT",
    "debug_wait_timeout",
    "MAX_SEGMENTS",
    "decode_stacked",
    "proj_stacked",
    "w4a16_decode",
    "quant_nvfp4_rows",
    "w4a4_decode",
    "sf_blocked_bytes",
    "sf_blocked",
    "w4a4_gemm",
    "w4a4_proj",
    "gemm_block_m",
    "w4a4_proj_scratch_bytes",
    "silu_mul",
    "requant_silu_a",
    "proj_silu_scratch_bytes",
    "proj_silu",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsr.so")
DECODE_MAX_M = 16
DEV_STATUS_DEBUG_WAIT = 32  # device status bit of bsr_debug_wait_timeout
DECODE_STATIC_WEIGHT = 1  # bsr_decode_ex flag: nothing ahead on the stream writes the weight
MAX_SEGMENTS = 8  # BSR_MAX_SEGMENTS: segments of a stacked weight

STATUS_NAMES = {
    0: "BSR_OK",
    1: "BSR_EINVAL",
    2: "BSR_EALIGN",
    3: "BSR_ESHAPE",
    4: "BSR_ESCRATCH",
    5: "BSR_ECUDA",
    6: "BSR_ETIMEOUT",
    7: "BSR_ENODEV",
}

# (name, restype, argtypes) of every exported symbol, mirroring include/bsr.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
SIGNATURES = [
    ("bsr_abi_version", ctypes.c_int, []),
    ("bsr_last_error", ctypes.c_char_p, []),
    ("bsr_device_status", ctypes.c_int, []),
    ("bsr_requant_w", ctypes.c_int, [_P, _P, ctypes.c_float, _P, _P, _I64, _I64, _P]),
    ("bsr_a_scale_ld", _I64, [_I64]),
    ("bsr_requant_a", ctypes.c_int, [_P, _P, _P, _I64, _I64, _P]),
    ("bsr_gemm", ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    ("bsr_proj_scratch_bytes", ctypes.c_size_t, [_I64, _I64]),
    ("bsr_gemm_block_m", ctypes.c_int, [_I64, _I64]),
    ("bsr_proj", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, ctypes.c_size_t, _P]),
    ("bsr_decode", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    ("bsr_gemm_partials", ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    ("bsr_proj_noalloc", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    ("bsr_debug_wait_timeout", ctypes.c_int, [ctypes.c_int, _P]),
    ("bsr_decode_ex", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_uint, _P]),
    ("bsr_decode_host", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, ctypes.c_uint, _P]),
    ("bsr_proj_host_scratch_bytes", _I64, [_I64, _I64, _I64]),
    ("bsr_proj_host", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_size_t, _I64, _P]),
    ("bsr_decode_stacked", ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, _P, _I64, _I64, ctypes.c_uint, _P]),
    ("bsr_proj_stacked", ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, _P, _I64, _I64, _P, ctypes.c_size_t, _P]),
    ("bsr_w4a16_decode", ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P, _I64, _I64, _I64, _P]),
    ("bsr_w4a16_decode_ex", ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P, _I64, _I64, _I64, ctypes.c_uint, _P]),
    ("bsr_nvfp4_quant_rows", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _P]),
    ("bsr_w4a4_decode", ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P, _I64, _I64, _I64, _P]),
    ("bsr_w4a4_decode_ex", ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P, _I64, _I64, _I64, ctypes.c_uint, _P]),
    ("bsr_nvfp4_sf_blocked_bytes", ctypes.c_size_t, [_I64, _I64]),
    ("bsr_nvfp4_sf_blocked", ctypes.c_int, [_P, _P, _I64, _I64, _P]),
    ("bsr_w4a4_gemm", ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_float, _P, _I64, _I64, _I64, _P, _P]),
    ("bsr_w4a4_proj_scratch_bytes", ctypes.c_size_t, [_I64, _I64]),
    ("bsr_w4a4_proj", ctypes.c_int, [_P, _P, _P, ctypes.c_float, _P, _I64, _I64, _I64, _P, ctypes.c_size_t, _P]),
    ("bsr_silu_mul", ctypes.c_int, [_P, _P, _P, _I64, _I64, _P]),
    ("bsr_requant_silu_a", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _P]),
    ("bsr_proj_silu_scratch_bytes", ctypes.c_size_t, [_I64, _I64]),
    ("bsr_proj_silu", ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, ctypes.c_size_t, _P]),
]


class BsrError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{self.name}: {message}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libbsr.so (built in-tree by ``build.py``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m block_scaled_precision_requant_b200.build`"
            )
        handle = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(status: int):
    if status != 0:
        raise BsrError(status, lib().bsr_last_error().decode())


def abi_version() -> int:
    return lib().bsr_abi_version()


def last_error() -> str:
    return lib().bsr_last_error().decode()


def device_status() -> int:
    """Synchronise and return/clear the device status word (0 = no wait timed out)."""
    return lib().bsr_device_status()


# ---------------------------------------------------------------------------
# tensor marshalling helpers
# ---------------------------------------------------------------------------


def _torch():
    import torch

    return torch


def _stream_ptr(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, dtype, shape, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host(t, dtype, shape, name):
    """A page-locked host tensor (its address; the library checks that it is
    mapped into the device's address space)."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _empty(shape, dtype, like):
    torch = _torch()
    return torch.empty(shape, dtype=dtype, device=like.device)


# ---------------------------------------------------------------------------
# operations
# ---------------------------------------------------------------------------


def requant_w(w_packed, w_e4m3, scale2: float, w_i8=None, w_scale=None, stream=None):
    """NVFP4 weight -> (w_i8 [N, K] int8, w_scale [N, K/32] float32)."""
    torch = _torch()
    n, k2 = w_packed.shape
    k = 2 * k2
    if w_i8 is None:
        w_i8 = _empty((n, k), torch.int8, w_packed)
    if w_scale is None:
        w_scale = _empty((n, k // 32), torch.float32, w_packed)
    _check(
        lib().bsr_requant_w(
            _dev(w_packed, torch.uint8, (n, k2), "w_packed"),
            _dev(w_e4m3, torch.uint8, (n, k // 16), "w_e4m3"),
            ctypes.c_float(float(scale2)),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            n,
            k,
            _stream_ptr(stream),
        )
    )
    return w_i8, w_scale


def a_scale_ld(m: int) -> int:
    return lib().bsr_a_scale_ld(m)


def requant_a(a, a_i8=None, a_scale_t=None, stream=None):
    """BF16 [M, K] -> (a_i8 [M, K] int8, a_scale_t [K/32, ld] float32 block-major)."""
    torch = _torch()
    m, k = a.shape
    ld = a_scale_ld(m)
    if a_i8 is None:
        a_i8 = _empty((m, k), torch.int8, a)
    if a_scale_t is None:
        a_scale_t = _empty((k // 32, ld), torch.float32, a)
    _check(
        lib().bsr_requant_a(
            _dev(a, torch.bfloat16, (m, k), "a"),
            _dev(a_i8, torch.int8, (m, k), "a_i8"),
            _dev(a_scale_t, torch.float32, (k // 32, ld), "a_scale_t"),
            m,
            k,
            _stream_ptr(stream),
        )
    )
    return a_i8, a_scale_t


def gemm(a_i8, a_scale_t, w_i8, w_scale, out=None, stream=None):
    """int8 block-scaled GEMM -> out [M, N] bfloat16."""
    torch = _torch()
    m, k = a_i8.shape
    n = w_i8.shape[0]
    if out is None:
        out = _empty((m, n), torch.bfloat16, a_i8)
    _check(
        lib().bsr_gemm(
            _dev(a_i8, torch.int8, (m, k), "a_i8"),
            _dev(a_scale_t, torch.float32, (k // 32, a_scale_ld(m)), "a_scale_t"),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            _dev(out, torch.bfloat16, (m, n), "out"),
            m,
            n,
            k,
            _stream_ptr(stream),
        )
    )
    return out


def gemm_partials(a_i8, a_scale_t, w_i8, w_scale, out=None, partials=None, stream=None):
    """:func:`gemm` that also returns the int32 block partials [M, N, K/32]."""
    torch = _torch()
    m, k = a_i8.shape
    n = w_i8.shape[0]
    if out is None:
        out = _empty((m, n), torch.bfloat16, a_i8)
    if partials is None:
        partials = _empty((m, n, k // 32), torch.int32, a_i8)
    _check(
        lib().bsr_gemm_partials(
            _dev(a_i8, torch.int8, (m, k), "a_i8"),
            _dev(a_scale_t, torch.float32, (k // 32, a_scale_ld(m)), "a_scale_t"),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            _dev(out, torch.bfloat16, (m, n), "out"),
            _dev(partials, torch.int32, (m, n, k // 32), "partials"),
            m,
            n,
            k,
            _stream_ptr(stream),
        )
    )
    return out, partials


def proj_scratch_bytes(m: int, k: int) -> int:
    return lib().bsr_proj_scratch_bytes(m, k)


def proj(a, w_i8, w_scale, out=None, scratch=None, stream=None):
    """out [M, N] bfloat16 = A [M, K] (bfloat16) . W^T from the requantised weight."""
    torch = _torch()
    m, k = a.shape
    n = w_i8.shape[0]
    if out is None:
        out = _empty((m, n), torch.bfloat16, a)
    need = proj_scratch_bytes(m, k)
    if scratch is None and need:
        scratch = _empty((need,), torch.uint8, a)
    sp = ctypes.c_void_p(scratch.data_ptr()) if scratch is not None else ctypes.c_void_p(0)
    sb = scratch.numel() * scratch.element_size() if scratch is not None else 0
    if scratch is not None and not scratch.is_cuda:
        raise ValueError("scratch must be a CUDA tensor")
    _check(
        lib().bsr_proj(
            _dev(a, torch.bfloat16, (m, k), "a"),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            _dev(out, torch.bfloat16, (m, n), "out"),
            m,
            n,
            k,
            sp,
            sb,
            _stream_ptr(stream),
        )
    )
    return out


def decode(a, w_i8, w_scale, out=None, stream=None, static_weight=False):
    """The decode kernel for any M (activation requantisation fused, CUDA cores).

    ``static_weight=True`` promises that no kernel in flight or queued ahead
    on the stream writes ``w_i8``/``w_scale`` (a decode loop over a resident
    weight); the kernel then starts part of its weight copies before waiting
    for the previous kernel."""
    torch = _torch()
    m, k = a.shape
    n = w_i8.shape[0]
    if out is None:
        out = _empty((m, n), torch.bfloat16, a)
    _check(
        lib().bsr_decode_ex(
            _dev(a, torch.bfloat16, (m, k), "a"),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            _dev(out, torch.bfloat16, (m, n), "out"),
            m,
            n,
            k,
            DECODE_STATIC_WEIGHT if static_weight else 0,
            _stream_ptr(stream),
        )
    )
    return out


def decode_host(a_host, w_i8, w_scale, out_host, a_dev, out_dev, stream=None, static_weight=False):
    """The decode step with the activations read from, and the result written
    to, page-locked host tensors (``tensor.pin_memory()``); ``a_dev`` [M, K]
    and ``out_dev`` [M, N] BF16 are device staging buffers.  The copies are
    kernels chained with the decode kernel by programmatic dependent launch.
    ``out_host`` holds the result once the stream has passed the call."""
    torch = _torch()
    m, k = a_host.shape
    n = w_i8.shape[0]
    _check(
        lib().bsr_decode_host(
            _host(a_host, torch.bfloat16, (m, k), "a_host"),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            _host(out_host, torch.bfloat16, (m, n), "out_host"),
            m,
            n,
            k,
            _dev(a_dev, torch.bfloat16, (m, k), "a_dev"),
            _dev(out_dev, torch.bfloat16, (m, n), "out_dev"),
            DECODE_STATIC_WEIGHT if static_weight else 0,
            _stream_ptr(stream),
        )
    )
    return out_host


def proj_host(a_host, w_i8, w_scale, out_host, a_dev, out_dev, scratch=None, chunk_rows=0, stream=None):
    """bsr_proj with page-locked host activations and result, pipelined over
    row chunks (copies of one chunk overlap the compute of its neighbours).
    ``a_dev`` [M, K] and ``out_dev`` [M, N] BF16 are device staging buffers;
    ``scratch`` (uint8, device) of ``proj_host_scratch_bytes(M, K,
    chunk_rows)`` bytes is allocated when not given."""
    torch = _torch()
    m, k = a_host.shape
    n = w_i8.shape[0]
    need = int(lib().bsr_proj_host_scratch_bytes(m, k, chunk_rows))
    if scratch is None and need > 0:
        scratch = torch.empty((need,), dtype=torch.uint8, device=a_dev.device)
    ptr = ctypes.c_void_p(scratch.data_ptr()) if scratch is not None else None
    size = scratch.numel() if scratch is not None else 0
    _check(
        lib().bsr_proj_host(
            _host(a_host, torch.bfloat16, (m, k), "a_host"),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            _host(out_host, torch.bfloat16, (m, n), "out_host"),
            m,
            n,
            k,
            _dev(a_dev, torch.bfloat16, (m, k), "a_dev"),
            _dev(out_dev, torch.bfloat16, (m, n), "out_dev"),
            ptr,
            size,
            chunk_rows,
            _stream_ptr(stream),
        )
    )
    return out_host


def proj_host_scratch_bytes(m: int, k: int, chunk_rows: int = 0) -> int:
    return int(lib().bsr_proj_host_scratch_bytes(m, k, chunk_rows))


def debug_wait_timeout(limit_ms: int, stream=None):
    """Queue the test kernel whose one pipeline wait can never be satisfied;
    it gives up after ``limit_ms`` and sets bit 32 of the device status word
    (read it with :func:`device_status`)."""
    _check(lib().bsr_debug_wait_timeout(int(limit_ms), _stream_ptr(stream)))


def silu_mul(gate, up, x=None, stream=None):
    """x = bf16(silu(gate) * up), all [M, K] bfloat16."""
    torch = _torch()
    m, k = gate.shape
    if x is None:
        x = _empty((m, k), torch.bfloat16, gate)
    _check(
        lib().bsr_silu_mul(
            _dev(gate, torch.bfloat16, (m, k), "gate"),
            _dev(up, torch.bfloat16, (m, k), "up"),
            _dev(x, torch.bfloat16, (m, k), "x"),
            m,
            k,
            _stream_ptr(stream),
        )
    )
    return x


def requant_silu_a(gate, up, a_i8=None, a_scale_t=None, stream=None):
    """requant_a of bf16(silu(gate) * up) -> (a_i8 [M, K], a_scale_t [K/32, ld])."""
    torch = _torch()
    m, k = gate.shape
    ld = a_scale_ld(m)
    if a_i8 is None:
        a_i8 = _empty((m, k), torch.int8, gate)
    if a_scale_t is None:
        a_scale_t = _empty((k // 32, ld), torch.float32, gate)
    _check(
        lib().bsr_requant_silu_a(
            _dev(gate, torch.bfloat16, (m, k), "gate"),
            _dev(up, torch.bfloat16, (m, k), "up"),
            _dev(a_i8, torch.int8, (m, k), "a_i8"),
            _dev(a_scale_t, torch.float32, (k // 32, ld), "a_scale_t"),
            m,
            k,
            _stream_ptr(stream),
        )
    )
    return a_i8, a_scale_t


def proj_silu_scratch_bytes(m: int, k: int) -> int:
    return lib().bsr_proj_silu_scratch_bytes(m, k)


def proj_silu(gate, up, w_i8, w_scale, out=None, scratch=None, stream=None):
    """out [M, N] bfloat16 = proj(bf16(silu(gate) * up), W)."""
    torch = _torch()
    m, k = gate.shape
    n = w_i8.shape[0]
    if out is None:
        out = _empty((m, n), torch.bfloat16, gate)
    need = proj_silu_scratch_bytes(m, k)
    if scratch is None and need:
        scratch = _empty((need,), torch.uint8, gate)
    if scratch is not None and not scratch.is_cuda:
        raise ValueError("scratch must be a CUDA tensor")
    sp = ctypes.c_void_p(scratch.data_ptr()) if scratch is not None else ctypes.c_void_p(0)
    sb = scratch.numel() * scratch.element_size() if scratch is not None else 0
    _check(
        lib().bsr_proj_silu(
            _dev(gate, torch.bfloat16, (m, k), "gate"),
            _dev(up, torch.bfloat16, (m, k), "up"),
            _dev(w_i8, torch.int8, (n, k), "w_i8"),
            _dev(w_scale, torch.float32, (n, k // 32), "w_scale"),
            _dev(out, torch.bfloat16, (m, n), "out"),
            m,
            n,
            k,
            sp,
            sb,
            _stream_ptr(stream),
        )
    )
    return out


def _segments(segments, k):
    """Host arrays (device pointers and row counts) for a stacked weight given
    as a list of (w_i8 [n_s, K], w_scale [n_s, K/32]) pairs."""
    torch = _torch()
    num = len(segments)
    if not 1 <= num <= MAX_SEGMENTS:
        raise ValueError(f"1..{MAX_SEGMENTS} segments, got {num}")
    w_arr = (ctypes.c_void_p * num)()
    s_arr = (ctypes.c_void_p * num)()
    n_arr = (ctypes.c_int64 * num)()
    for i, (w, ws) in enumerate(segments):
        n_s = w.shape[0]
        w_arr[i] = _dev(w, torch.int8, (n_s, k), f"w_i8[{i}]")
        s_arr[i] = _dev(ws, torch.float32, (n_s, k // 32), f"w_scale[{i}]")
        n_arr[i] = n_s
    return w_arr, s_arr, n_arr, num, sum(int(w.shape[0]) for w, _ in segments)


def decode_stacked(a, segments, out=None, stream=None, static_weight=False):
    """One decode launch over a stacked weight: out [M, sum n_s], segment s in
    its own column slice (segments: list of (w_i8, w_scale))."""
    torch = _torch()
    m, k = a.shape
    w_arr, s_arr, n_arr, num, n = _segments(segments, k)
    if out is None:
        out = _empty((m, n), torch.bfloat16, a)
    _check(
        lib().bsr_decode_stacked(
            _dev(a, torch.bfloat16, (m, k), "a"), ctypes.cast(w_arr, ctypes.c_void_p),
            ctypes.cast(s_arr, ctypes.c_void_p), ctypes.cast(n_arr, ctypes.c_void_p), num,
            _dev(out, torch.bfloat16, (m, n), "out"), m, k,
            DECODE_STATIC_WEIGHT if static_weight else 0, _stream_ptr(stream),
        )
    )
    return out


def proj_stacked(a, segments, out=None, scratch=None, stream=None):
    """bsr_proj over a stacked weight (decode launch for M <= 16, else
    requant_a once and one GEMM per segment)."""
    torch = _torch()
    m, k = a.shape
    w_arr, s_arr, n_arr, num, n = _segments(segments, k)
    if out is None:
        out = _empty((m, n), torch.bfloat16, a)
    need = proj_scratch_bytes(m, k)
    if scratch is None and need:
        scratch = _empty((need,), torch.uint8, a)
    sp = ctypes.c_void_p(scratch.data_ptr()) if scratch is not None else ctypes.c_void_p(0)
    sb = scratch.numel() * scratch.element_size() if scratch is not None else 0
    _check(
        lib().bsr_proj_stacked(
            _dev(a, torch.bfloat16, (m, k), "a"), ctypes.cast(w_arr, ctypes.c_void_p),
            ctypes.cast(s_arr, ctypes.c_void_p), ctypes.cast(n_arr, ctypes.c_void_p), num,
            _dev(out, torch.bfloat16, (m, n), "out"), m, k, sp, sb, _stream_ptr(stream),
        )
    )
    return out


def _nvfp4_gemv(entry, a, w_packed, w_e4m3, scale2, out, stream, static_weight):
    torch = _torch()
    m, k = a.shape
    n = w_packed.shape[0]
    if out is None:
        out = _empty((m, n), torch.bfloat16, a)
    _check(
        entry(
            _dev(a, torch.bfloat16, (m, k), "a"),
            _dev(w_packed, torch.uint8, (n, k // 2), "w_packed"),
            _dev(w_e4m3, torch.uint8, (n, k // 16), "w_e4m3"),
            ctypes.c_float(float(scale2)),
            _dev(out, torch.bfloat16, (m, n), "out"),
            m,
            n,
            k,
            DECODE_STATIC_WEIGHT if static_weight else 0,
            _stream_ptr(stream),
        )
    )
    return out


def w4a16_decode(a, w_packed, w_e4m3, scale2: float, out=None, stream=None, static_weight=False):
    """NVFP4 W4A16 decode GEMV on the stored weight -> out [M, N] bfloat16.
    ``static_weight=True`` as in :func:`decode`."""
    return _nvfp4_gemv(lib().bsr_w4a16_decode_ex, a, w_packed, w_e4m3, scale2, out, stream, static_weight)


def quant_nvfp4_rows(a, out=None, stream=None):
    """Per-row NVFP4 quantiser of the W4A4 path: a [M, K] bfloat16 ->
    (a_packed [M, K/2] uint8, a_e4m3 [M, K/16] uint8, a_scale2 [M] float32)."""
    torch = _torch()
    m, k = a.shape
    if out is None:
        out = (_empty((m, k // 2), torch.uint8, a), _empty((m, k // 16), torch.uint8, a),
               _empty((m,), torch.float32, a))
    packed, e4, s2 = out
    _check(
        lib().bsr_nvfp4_quant_rows(
            _dev(a, torch.bfloat16, (m, k), "a"),
            _dev(packed, torch.uint8, (m, k // 2), "a_packed"),
            _dev(e4, torch.uint8, (m, k // 16), "a_e4m3"),
            _dev(s2, torch.float32, (m,), "a_scale2"),
            m,
            k,
            _stream_ptr(stream),
        )
    )
    return packed, e4, s2


def w4a4_decode(a, w_packed, w_e4m3, scale2: float, out=None, stream=None, static_weight=False):
    """NVFP4 W4A4 decode GEMV (activation rows quantised to NVFP4 inside the
    kernel) -> out [M, N] bfloat16.  ``static_weight=True`` as in
    :func:`decode`."""
    return _nvfp4_gemv(lib().bsr_w4a4_decode_ex, a, w_packed, w_e4m3, scale2, out, stream, static_weight)


def sf_blocked_bytes(rows: int, k: int) -> int:
    """Bytes of the blocked scale layout of the W4A4 GEMM (0 if invalid)."""
    return int(lib().bsr_nvfp4_sf_blocked_bytes(rows, k))


def sf_blocked(e4m3, out=None, stream=None):
    """Row-major E4M3 scales [rows, K/16] uint8 -> the W4A4 GEMM's blocked
    layout (uint8 [sf_blocked_bytes(rows, K)])."""
    torch = _torch()
    rows, kb = e4m3.shape
    k = kb * 16
    nbytes = sf_blocked_bytes(rows, k)
    if out is None:
        out = _empty((nbytes,), torch.uint8, e4m3)
    _check(
        lib().bsr_nvfp4_sf_blocked(
            _dev(e4m3, torch.uint8, (rows, kb), "e4m3"), _dev(out, torch.uint8, (nbytes,), "blocked"), rows, k,
            _stream_ptr(stream),
        )
    )
    return out


def w4a4_gemm(a_packed, a_sf_blocked, a_scale2, w_packed, w_sf_blocked, scale2: float, out=None, status=None,
              stream=None):
    """W4A4 GEMM on the tensor cores -> out [M, N] bfloat16.  `status` is a
    device int32 tensor of one element into which a timed-out wait ORs its
    bit (a fresh zero one when omitted)."""
    torch = _torch()
    m, kh = a_packed.shape
    n = w_packed.shape[0]
    k = 2 * kh
    if out is None:
        out = _empty((m, n), torch.bfloat16, a_packed)
    if status is None:
        status = torch.zeros((1,), dtype=torch.int32, device=a_packed.device)
    _check(
        lib().bsr_w4a4_gemm(
            _dev(a_packed, torch.uint8, (m, kh), "a_packed"),
            _dev(a_sf_blocked, torch.uint8, (sf_blocked_bytes(m, k),), "a_sf_blocked"),
            _dev(a_scale2, torch.float32, (m,), "a_scale2"),
            _dev(w_packed, torch.uint8, (n, kh), "w_packed"),
            _dev(w_sf_blocked, torch.uint8, (sf_blocked_bytes(n, k),), "w_sf_blocked"),
            ctypes.c_float(float(scale2)),
            _dev(out, torch.bfloat16, (m, n), "out"),
            m,
            n,
            k,
            _dev(status, torch.int32, (1,), "status"),
            _stream_ptr(stream),
        )
    )
    return out


def w4a4_proj_scratch_bytes(m: int, k: int) -> int:
    """Scratch bytes of :func:`w4a4_proj` for M rows (0 if invalid)."""
    return int(lib().bsr_w4a4_proj_scratch_bytes(m, k))


def w4a4_proj(a, w_packed, w_sf_blocked, scale2: float, out=None, scratch=None, stream=None):
    """The W4A4 projection on the tensor cores: a [M, K] bfloat16 quantised to
    NVFP4 rows, scales relaid, FP4 MMA against w_packed [N, K/2] (scales
    w_sf_blocked from :func:`sf_blocked`) -> out [M, N] bfloat16."""
    torch = _torch()
    m, k = a.shape
    n = w_packed.shape[0]
    if out is None:
        out = _empty((m, n), torch.bfloat16, a)
    need = w4a4_proj_scratch_bytes(m, k)
    if scratch is None:
        scratch = _empty((max(need, 1),), torch.uint8, a)
    _check(
        lib().bsr_w4a4_proj(
            _dev(a, torch.bfloat16, (m, k), "a"),
            _dev(w_packed, torch.uint8, (n, k // 2), "w_packed"),
            _dev(w_sf_blocked, torch.uint8, (sf_blocked_bytes(n, k),), "w_sf_blocked"),
            ctypes.c_float(float(scale2)),
            _dev(out, torch.bfloat16, (m, n), "out"),
            m,
            n,
            k,
            ctypes.c_void_p(scratch.data_ptr()),
            scratch.numel() * scratch.element_size(),
            _stream_ptr(stream),
        )
    )
    return out


def gemm_block_m(m: int, n: int) -> int:
    """Activation rows per tile the tensor-core GEMM uses for M x N on the
    current device (128, 192 or 256; 0 without a usable device)."""
    return int(lib().bsr_gemm_block_m(m, n))
