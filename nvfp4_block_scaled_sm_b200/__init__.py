"""Block-scaled low-precision quantization (MXFP8 / MXFP4 / NVFP4) for NVIDIA B200.

Python binding of ``libmxq.so`` (C ABI declared in ``include/mxq.h``). This
module only marshals arguments: it allocates outputs with torch on the input's
device, passes raw pointers and the current CUDA stream, and raises on any
non-zero status. Every step of quantization runs in the library's sm_100a
kernels; there is no fallback of any kind, and importing this package fails
if the library has not been built (``python nvfp4_block_scaled_sm_b200/build.py``).

The call ``qweight, scale = mxfp8_quantize(weight)`` follows "PR #1935 完整报告
-- Use TransformerEngine for MXFP8 quantization" (关键源码片段): compact,
non-swizzled qweight (E4M3 codes, same shape) and scale (E8M0 bytes, last dim
N/32), the scale being the dequantization multiplier ("_scale_inv").
"""
from __future__ import annotations

import ctypes
import functools
import os
from typing import Sequence

import torch

__all__ = [
    "MxqError", "lib", "library_path",
    "mxfp8_quantize", "mxfp8_dequantize", "mxfp8_quantize_grouped", "mxfp8_quantize_columnwise",
    "mxfp4_quantize", "mxfp4_dequantize", "mxfp4_quantize_grouped", "mx_fake_quantize",
    "mxfp8_gemm",
    "nvfp4_amax", "nvfp4_quantize", "nvfp4_dequantize",
    "nvfp4_amax_sliced", "nvfp4_quantize_sliced", "nvfp4_quantize_experts",
    "swizzled_scale_bytes", "nvfp4_workspace_bytes", "set_output_allocator", "swizzle_scales",
    "set_nvtx",
    "as_float8_e4m3", "as_float8_e8m0", "as_float4_e2m1x2",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libmxq.so")

BF16, FP32 = 0, 1
FMT_MXFP8, FMT_MXFP4 = 0, 1
NVFP4_GLOBAL_GIVEN = 1


class MxqError(RuntimeError):
    """A libmxq call returned a non-zero status."""

    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn}: status {status}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is missing: build it with "
            "`python nvfp4_block_scaled_sm_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(library_path)
    vp, i64, i32, u32, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                             ctypes.c_uint32, ctypes.c_size_t)
    L.mxq_abi_version.restype = i32
    L.mxq_status_string.argtypes, L.mxq_status_string.restype = [i32], ctypes.c_char_p
    L.mxq_last_cuda_error.restype = ctypes.c_char_p
    L.mxq_swizzled_scale_bytes.argtypes, L.mxq_swizzled_scale_bytes.restype = [i64, i64], i64
    L.mxq_nvfp4_workspace_bytes.argtypes, L.mxq_nvfp4_workspace_bytes.restype = [i64, i64], sz
    L.mxfp8_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp]
    L.mxfp8_dequantize.argtypes = [vp, vp, i64, i64, vp, i32, vp]
    L.mxfp8_quantize_grouped.argtypes = [vp, i32, i32, vp, i64, i64, vp, vp, vp]
    L.mxfp8_quantize_grouped_swizzled.argtypes = [vp, i32, i32, vp, i64, i64, vp, vp, vp, i64, vp]
    L.mxfp8_quantize_grouped_ptrs.argtypes = [i32, vp, vp, i64, i32, vp, vp, vp]
    L.mxq_swizzle_scales.argtypes = [vp, i64, i64, vp, vp]
    L.mxq_grouped_swizzled_scale_bytes_max.argtypes = [i32, i64, i64]
    L.mxq_grouped_swizzled_scale_bytes_max.restype = i64
    L.mxfp8_quantize_columnwise.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, vp]
    L.mxfp4_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp]
    L.mxfp4_dequantize.argtypes = [vp, vp, i64, i64, vp, i32, vp]
    L.mxfp4_quantize_grouped.argtypes = [vp, i32, i32, vp, i64, i64, vp, vp, vp]
    L.mxfp4_quantize_grouped_swizzled.argtypes = [vp, i32, i32, vp, i64, i64, vp, vp, vp, i64, vp]
    L.mxfp4_quantize_grouped_ptrs.argtypes = [i32, vp, vp, i64, i32, vp, vp, vp]
    L.mx_fake_quantize.argtypes = [i32, vp, i32, i64, i64, i64, vp, i32, vp]
    L.mxfp8_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, i32, vp, vp]
    L.mxq_check_bounded_wait.argtypes = [i64, vp, vp]
    L.nvfp4_amax.argtypes = [vp, i32, i64, i64, i64, vp, vp, sz, vp]
    L.nvfp4_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, u32, vp, sz, vp]
    L.nvfp4_dequantize.argtypes = [vp, vp, vp, i64, i64, vp, i32, vp]
    L.mxq_nvfp4_sliced_workspace_bytes.argtypes = [i32]
    L.mxq_nvfp4_sliced_workspace_bytes.restype = sz
    L.nvfp4_quantize_sliced.argtypes = [vp, i32, i64, i64, i64, i32, vp, vp, vp, vp, vp, u32, vp,
                                        sz, vp]
    L.nvfp4_amax_sliced.argtypes = [vp, i32, i64, i64, i64, i32, vp, vp, vp, sz, vp]
    for f in ("mxfp8_quantize", "mxfp8_dequantize", "mxfp8_quantize_grouped",
              "mxfp8_quantize_grouped_swizzled", "mxfp8_quantize_grouped_ptrs",
              "mxfp8_quantize_columnwise", "mxfp4_quantize", "mxfp4_dequantize",
              "mxfp4_quantize_grouped", "mxfp4_quantize_grouped_swizzled",
              "mxfp4_quantize_grouped_ptrs", "mx_fake_quantize", "mxq_swizzle_scales", "mxfp8_gemm",
              "mxq_check_bounded_wait", "nvfp4_amax",
              "nvfp4_quantize_sliced", "nvfp4_amax_sliced",
              "nvfp4_quantize", "nvfp4_dequantize"):
        getattr(L, f).restype = i32
    return L


lib = _load()


def _check(fn: str, status: int):
    if status != 0:
        msg = lib.mxq_status_string(status).decode()
        if status == 6:
            msg += f" ({lib.mxq_last_cuda_error().decode()})"
        raise MxqError(fn, status, msg)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {dt}: expected torch.bfloat16 or torch.float32")


def _require_cuda(*ts: torch.Tensor):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device (no CPU path exists)")


def _stream(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _rows_view(x: torch.Tensor):
    """(M, N, ld_x) of x seen as M rows of N contiguous elements with row
    stride ld_x; raises if the leading dims do not collapse to one stride."""
    if x.dim() == 0:
        raise ValueError("expected at least one dimension")
    N = x.shape[-1]
    if x.dim() == 1:
        return 1, N, N
    if N > 1 and x.stride(-1) != 1:
        raise ValueError("the last dimension must be contiguous")
    M = 1
    for s in x.shape[:-1]:
        M *= s
    lead = [(s, st) for s, st in zip(x.shape[:-1], x.stride()[:-1]) if s > 1]
    if not lead:
        return M, N, N
    ld = lead[-1][1]
    for (s0, st0), (s1, st1) in zip(lead[:-1], lead[1:]):
        if st0 != st1 * s1:
            raise ValueError("leading dimensions do not collapse to a single row stride")
    return M, N, ld


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_output_allocator = None


def set_output_allocator(fn):
    """Route every output and workspace tensor this module allocates through
    ``fn(shape, dtype, device) -> torch.Tensor`` (for example a memory pool,
    or a checker that places each buffer between guard bytes); ``None``
    restores ``torch.empty``. The tensor returned must be contiguous, have
    the requested shape and dtype and start on a 256-byte boundary. Returns
    the previous allocator."""
    global _output_allocator
    prev, _output_allocator = _output_allocator, fn
    return prev


def _empty(shape, dtype: torch.dtype, device) -> torch.Tensor:
    shape = (int(shape),) if isinstance(shape, int) else tuple(int(d) for d in shape)
    if _output_allocator is None:
        return torch.empty(shape, dtype=dtype, device=device)
    t = _output_allocator(shape, dtype, device)
    if tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous():
        raise RuntimeError("the output allocator returned a tensor of the wrong layout")
    return t


def _zeros(shape, dtype: torch.dtype, device) -> torch.Tensor:
    return _empty(shape, dtype, device).zero_()


def swizzled_scale_bytes(M: int, S: int) -> int:
    return int(lib.mxq_swizzled_scale_bytes(M, S))


def nvfp4_workspace_bytes(M: int = 0, N: int = 0) -> int:
    return int(lib.mxq_nvfp4_workspace_bytes(M, N))


def swizzle_scales(scale: torch.Tensor) -> torch.Tensor:
    """A compact [..., S] uint8 scale tensor (E8M0 scales of the MX
    quantizers, or NVFP4's E4M3 block scales) in the 128x4-tile layout read by
    block-scaled tensor-core MMA, as a flat uint8 tensor of
    ``swizzled_scale_bytes(M, S)`` bytes (M = the product of the leading
    dimensions)."""
    _require_cuda(scale)
    if scale.dtype != torch.uint8 or not scale.is_contiguous() or scale.dim() == 0:
        raise TypeError("scale must be a contiguous uint8 tensor")
    S = scale.shape[-1]
    M = scale.numel() // S if S else 0
    out = _empty((max(swizzled_scale_bytes(M, S), 0),), torch.uint8, scale.device)
    _check("mxq_swizzle_scales", lib.mxq_swizzle_scales(_ptr(scale), M, S, _ptr(out), _stream(scale)))
    return out


# ------------------------------------------------------------------ MXFP8

def _mx_quantize(fn: str, x: torch.Tensor, swizzled: bool, per_byte: int):
    _require_cuda(x)
    dt = _dtype_code(x.dtype)
    M, N, ld = _rows_view(x)
    q = _empty((*x.shape[:-1], N // per_byte), torch.uint8, x.device)
    s = _empty((*x.shape[:-1], N // 32), torch.uint8, x.device)
    swz = None
    if swizzled:
        swz = _empty((max(swizzled_scale_bytes(M, N // 32), 0),), torch.uint8, x.device)
    _check(fn, getattr(lib, fn)(_ptr(x), dt, M, N, ld, _ptr(q), _ptr(s), _ptr(swz), _stream(x)))
    return (q, s, swz) if swizzled else (q, s)


def _mx_dequantize(fn: str, q: torch.Tensor, scale: torch.Tensor, dtype: torch.dtype,
                   per_byte: int) -> torch.Tensor:
    _require_cuda(q, scale)
    if q.dtype != torch.uint8 or scale.dtype != torch.uint8:
        raise TypeError("codes and scale must be uint8")
    if not (q.is_contiguous() and scale.is_contiguous()):
        raise ValueError("codes and scale must be contiguous")
    N = q.shape[-1] * per_byte
    M = q.numel() * per_byte // N if N else 0
    if scale.numel() != M * (N // 32):
        raise ValueError("scale does not match the codes")
    y = _empty((*q.shape[:-1], N), dtype, q.device)
    _check(fn, getattr(lib, fn)(_ptr(q), _ptr(scale), M, N, _ptr(y), _dtype_code(dtype),
                                _stream(q)))
    return y


def _offsets_on(dev, row_offsets, E: int, M: int):
    """(device int64 offsets [E + 1], host row counts or None) from row
    offsets given as a sequence, a CPU tensor or a CUDA tensor."""
    if isinstance(row_offsets, torch.Tensor) and row_offsets.is_cuda:
        if row_offsets.dtype != torch.int64 or row_offsets.numel() != E + 1:
            raise TypeError("row_offsets must be int64 with E + 1 entries")
        return row_offsets.contiguous(), None
    host = [int(v) for v in (row_offsets.tolist() if isinstance(row_offsets, torch.Tensor)
                             else row_offsets)]
    if len(host) != E + 1 or host[0] != 0 or host[-1] != M or \
            any(b < a for a, b in zip(host[:-1], host[1:])):
        raise ValueError(f"row_offsets must rise from 0 to the {M} rows in {E + 1} entries")
    off = torch.tensor(host, dtype=torch.int64).to(dev, non_blocking=False)
    return off, [b - a for a, b in zip(host[:-1], host[1:])]


def _mx_quantize_grouped(fmt: str, xs, per_byte: int, row_offsets=None, swizzled=False):
    if isinstance(xs, torch.Tensor) and (xs.dim() == 3 or row_offsets is not None):
        # one stacked tensor: [E, M, N], or [M_total, N] with row offsets
        _require_cuda(xs)
        if not xs.is_contiguous():
            raise ValueError("the stacked tensor must be contiguous")
        dt = _dtype_code(xs.dtype)
        N = xs.shape[-1]
        M = xs.numel() // N if N else 0
        if row_offsets is None:
            E, R = xs.shape[0], xs.shape[1]
            row_offsets = [e * R for e in range(E + 1)]
        else:
            if xs.dim() != 2:
                raise ValueError("row_offsets go with a 2-D [M_total, N] tensor")
            E = (row_offsets.numel() if isinstance(row_offsets, torch.Tensor)
                 else len(row_offsets)) - 1
        off, counts = _offsets_on(xs.device, row_offsets, E, M)
        q = _empty((*xs.shape[:-1], N // per_byte), torch.uint8, xs.device)
        s = _empty((*xs.shape[:-1], N // 32), torch.uint8, xs.device)
        if not swizzled:
            _check(f"{fmt}_quantize_grouped",
                   getattr(lib, f"{fmt}_quantize_grouped")(_ptr(xs), dt, E, _ptr(off), M, N,
                                                           _ptr(q), _ptr(s), _stream(xs)))
            return q, s
        if counts is not None:
            nswz = sum(swizzled_scale_bytes(m, N // 32) for m in counts)
        else:
            nswz = int(lib.mxq_grouped_swizzled_scale_bytes_max(E, M, N // 32))
        swz = _empty((nswz,), torch.uint8, xs.device)
        _check(f"{fmt}_quantize_grouped_swizzled",
               getattr(lib, f"{fmt}_quantize_grouped_swizzled")(
                   _ptr(xs), dt, E, _ptr(off), M, N, _ptr(q), _ptr(s), _ptr(swz), nswz,
                   _stream(xs)))
        return q, s, swz
    if swizzled:
        raise ValueError("per-expert swizzled scales need one stacked tensor")
    parts = list(xs.unbind(0)) if isinstance(xs, torch.Tensor) else list(xs)
    if not parts:
        raise ValueError("no experts")
    _require_cuda(*parts)
    dt = _dtype_code(parts[0].dtype)
    N = parts[0].shape[-1]
    rows = []
    for p in parts:
        if p.dtype != parts[0].dtype or p.shape[-1] != N or p.device != parts[0].device:
            raise ValueError("experts must share dtype, device and last dimension")
        if not p.is_contiguous():
            raise ValueError("expert tensors must be contiguous")
        rows.append(p.numel() // N if N else 0)
    E = len(parts)
    total = sum(rows)
    dev = parts[0].device
    q = _empty((total, N // per_byte), torch.uint8, dev)
    s = _empty((total, N // 32), torch.uint8, dev)
    ptrs = (ctypes.c_void_p * E)(*[p.data_ptr() for p in parts])
    rws = (ctypes.c_int64 * E)(*rows)
    fn = f"{fmt}_quantize_grouped_ptrs"
    _check(fn, getattr(lib, fn)(E, ctypes.cast(ptrs, ctypes.c_void_p),
                                ctypes.cast(rws, ctypes.c_void_p), N, dt, _ptr(q), _ptr(s),
                                _stream(parts[0])))
    return q, s


def mxfp8_quantize(x: torch.Tensor, *, swizzled: bool = False):
    """MXFP8 rowwise quantize of a bf16/fp32 CUDA tensor.

    Returns ``(qweight, scale)``: uint8 E4M3 codes shaped like ``x`` and uint8
    E8M0 bytes shaped ``x.shape[:-1] + (N // 32,)``; with ``swizzled=True`` a
    third flat uint8 tensor holds the scales in the 128x4-tile layout read by
    block-scaled tensor-core MMA.
    """
    return _mx_quantize("mxfp8_quantize", x, swizzled, 1)


def mxfp8_dequantize(qweight: torch.Tensor, scale: torch.Tensor,
                     dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """decode(q) * 2^(scale - 127), as bf16 (RNE) or fp32 (exact)."""
    return _mx_dequantize("mxfp8_dequantize", qweight, scale, dtype, 1)


def mxfp8_quantize_grouped(xs: torch.Tensor | Sequence[torch.Tensor], *, row_offsets=None,
                           swizzled: bool = False):
    """Grouped MXFP8 of expert weights sharing N, in one launch.

    ``xs`` is one stacked tensor, [E, M, N] (results [E, M, N] and
    [E, M, N/32]) or [M_total, N] with ``row_offsets`` (E + 1 rising row
    offsets from 0 to M_total, as a list or an int64 tensor, on the host or on
    the device); or a sequence of contiguous [M_e, N] tensors in separate
    allocations (results concatenated along rows: [sum M_e, N] and
    [sum M_e, N/32]). With ``swizzled=True`` (stacked tensors only) a third,
    flat uint8 tensor holds each expert's scales in its own 128x4-tile
    layout, expert after expert; when the offsets live on the device it is
    sized by the upper bound of ``mxq_grouped_swizzled_scale_bytes_max``."""
    return _mx_quantize_grouped("mxfp8", xs, 1, row_offsets, swizzled)


def mxfp8_quantize_columnwise(x: torch.Tensor, *, rowwise: bool = False):
    """MXFP8 columnwise quantize (groups of 32 rows per column, rows past M
    counting as zeros) of a bf16/fp32 tensor seen as [M, N].

    Returns ``(qweight_t, scale_t)``: uint8 [N, M] E4M3 codes (the transposed
    layout) and uint8 [N, ceil(M/32)] E8M0 bytes. With ``rowwise=True`` the
    same launch also returns the rowwise ``(qweight, scale)`` of
    ``mxfp8_quantize`` first: ``(qweight, scale, qweight_t, scale_t)``."""
    _require_cuda(x)
    dt = _dtype_code(x.dtype)
    M, N, ld = _rows_view(x)
    dev = x.device
    q_t = _empty((N, M), torch.uint8, dev)
    s_t = _empty((N, (M + 31) // 32), torch.uint8, dev)
    q = s = None
    if rowwise:
        q = _empty((M, N), torch.uint8, dev)
        s = _empty((M, N // 32), torch.uint8, dev)
    _check("mxfp8_quantize_columnwise",
           lib.mxfp8_quantize_columnwise(_ptr(x), dt, M, N, ld, _ptr(q_t), _ptr(s_t), _ptr(q),
                                         _ptr(s), _stream(x)))
    if rowwise:
        return (q.view(*x.shape[:-1], N), s.view(*x.shape[:-1], N // 32), q_t, s_t)
    return q_t, s_t


# ------------------------------------------------------------------ MXFP4

def mxfp4_quantize(x: torch.Tensor, *, swizzled: bool = False):
    """MXFP4 rowwise quantize ("V4 mxfp4 #1372"): E8M0 scale per 32 elements
    (emax 2), E2M1 codes packed two per byte, even element in the low nibble.

    Returns ``(packed, scale)``: uint8 ``x.shape[:-1] + (N // 2,)`` and uint8
    ``x.shape[:-1] + (N // 32,)``; ``swizzled=True`` adds the 128x4-tile
    scale layout as a third, flat tensor."""
    return _mx_quantize("mxfp4_quantize", x, swizzled, 2)


def mxfp4_dequantize(packed: torch.Tensor, scale: torch.Tensor,
                     dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """decode_e2m1(code) * 2^(scale - 127), as bf16 (RNE) or fp32 (exact)."""
    return _mx_dequantize("mxfp4_dequantize", packed, scale, dtype, 2)


def mxfp4_quantize_grouped(xs: torch.Tensor | Sequence[torch.Tensor], *, row_offsets=None,
                           swizzled: bool = False):
    """Grouped MXFP4 of expert weights sharing N, in one launch (arguments
    and layouts as :func:`mxfp8_quantize_grouped`, codes packed [.., N // 2])."""
    return _mx_quantize_grouped("mxfp4", xs, 2, row_offsets, swizzled)


def mx_fake_quantize(x: torch.Tensor, fmt: str = "mxfp4",
                     dtype: torch.dtype | None = None) -> torch.Tensor:
    """QAT simulation: dequantize(quantize(x)) for ``fmt`` "mxfp8" or
    "mxfp4" in one pass (codes never stored), as ``dtype`` (default: the
    dtype of ``x``)."""
    formats = {"mxfp8": FMT_MXFP8, "mxfp4": FMT_MXFP4}
    if fmt not in formats:
        raise ValueError(f"fmt must be one of {sorted(formats)}")
    _require_cuda(x)
    dt = _dtype_code(x.dtype)
    dtype = x.dtype if dtype is None else dtype
    M, N, ld = _rows_view(x)
    y = _empty(x.shape, dtype, x.device)
    _check("mx_fake_quantize", lib.mx_fake_quantize(formats[fmt], _ptr(x), dt, M, N, ld, _ptr(y),
                                                    _dtype_code(dtype), _stream(x)))
    return y


# ------------------------------------------------------------------- GEMM

def mxfp8_gemm(qa: torch.Tensor, sa_swizzled: torch.Tensor, qb: torch.Tensor,
               sb_swizzled: torch.Tensor, dtype: torch.dtype = torch.bfloat16,
               error_flag: torch.Tensor | None = None) -> torch.Tensor:
    """D = A B^T from MXFP8 operands on the tensor cores: ``qa`` [M, K] and
    ``qb`` [N, K] uint8 E4M3 codes (as :func:`mxfp8_quantize` returns them)
    and their swizzled scales (the third output of
    ``mxfp8_quantize(..., swizzled=True)``). Returns D [M, N] as ``dtype``.
    ``error_flag`` (a zeroed int32 CUDA tensor) receives a non-zero code if
    a wait inside the kernel gave up."""
    _require_cuda(qa, sa_swizzled, qb, sb_swizzled)
    for t in (qa, qb, sa_swizzled, sb_swizzled):
        if t.dtype != torch.uint8 or not t.is_contiguous():
            raise TypeError("codes and scales must be contiguous uint8 tensors")
    if qa.dim() != 2 or qb.dim() != 2 or qa.shape[1] != qb.shape[1]:
        raise ValueError("expected qa [M, K] and qb [N, K]")
    M, K = qa.shape
    N = qb.shape[0]
    if sa_swizzled.numel() < swizzled_scale_bytes(M, K // 32) or \
            sb_swizzled.numel() < swizzled_scale_bytes(N, K // 32):
        raise ValueError("swizzled scales are smaller than the operands need")
    if error_flag is not None and (error_flag.dtype != torch.int32 or not error_flag.is_cuda):
        raise TypeError("error_flag must be an int32 CUDA tensor")
    d = _empty((M, N), dtype, qa.device)
    _check("mxfp8_gemm", lib.mxfp8_gemm(_ptr(qa), _ptr(sa_swizzled), _ptr(qb), _ptr(sb_swizzled),
                                        M, N, K, _ptr(d), _dtype_code(dtype), _ptr(error_flag),
                                        _stream(qa)))
    return d


def check_bounded_wait(timeout_ns: int = 2_000_000, device=None) -> dict:
    """Runs the self-check of the GEMM's bounded barrier wait on a CUDA device
    (``mxq_check_bounded_wait``): a wait on a barrier that nothing arrives on
    must give up after ``timeout_ns``, and a wait on a completed phase must
    return. Returns ``{"gave_up": bool, "completed": bool, "waited_ns": int}``
    after synchronizing the stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    result = torch.full((4,), -1, dtype=torch.int64, device=dev)
    _check("mxq_check_bounded_wait",
           lib.mxq_check_bounded_wait(int(timeout_ns), _ptr(result), _stream(result)))
    r = result.cpu().tolist()
    return {"gave_up": r[0] == 1, "completed": r[1] == 1, "waited_ns": r[2]}


# ------------------------------------------------------------------ NVFP4

def nvfp4_amax(x: torch.Tensor, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Tensor amax (non-NaN max |x|) as a 0-d fp32 CUDA tensor."""
    _require_cuda(x)
    dt = _dtype_code(x.dtype)
    M, N, ld = _rows_view(x)
    out = _zeros((), torch.float32, x.device)
    ws = workspace if workspace is not None else _empty(
        nvfp4_workspace_bytes(M, N), torch.uint8, x.device)
    _check("nvfp4_amax", lib.nvfp4_amax(_ptr(x), dt, M, N, ld, _ptr(out), _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(x)))
    return out


def nvfp4_quantize(x: torch.Tensor, global_scale: torch.Tensor | None = None,
                   amax: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """NVFP4 two-level quantize.

    Returns ``(packed, block_scale, global_scale)``: uint8 [..., N/2] with two
    E2M1 codes per byte (even element in the low nibble), uint8 E4M3 block
    scales [..., N/16], and the fp32 global scale as a 0-d CUDA tensor.
    ``global_scale`` (a given g) or ``amax`` (a given tensor amax, e.g. the
    all-reduced amax of a sharded tensor) skip the amax pass."""
    _require_cuda(x)
    dt = _dtype_code(x.dtype)
    M, N, ld = _rows_view(x)
    dev = x.device
    packed = _empty((*x.shape[:-1], N // 2), torch.uint8, dev)
    bs = _empty((*x.shape[:-1], N // 16), torch.uint8, dev)
    flags = 0
    if global_scale is not None:
        if global_scale.dtype != torch.float32 or global_scale.numel() != 1:
            raise TypeError("global_scale must be a single fp32 value")
        g = global_scale.to(dev)
        flags = NVFP4_GLOBAL_GIVEN
    else:
        g = _empty((), torch.float32, dev)
    if amax is not None and (amax.dtype != torch.float32 or amax.numel() != 1):
        raise TypeError("amax must be a single fp32 value")
    ws = None
    if global_scale is None and amax is None:
        ws = workspace if workspace is not None else _empty(
            nvfp4_workspace_bytes(M, N), torch.uint8, dev)
    _check("nvfp4_quantize",
           lib.nvfp4_quantize(_ptr(x), dt, M, N, ld, _ptr(packed), _ptr(bs), _ptr(g), _ptr(amax),
                              flags, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                              _stream(x)))
    return packed, bs, g


def _slice_array(slice_rows, M):
    rows = [int(r) for r in slice_rows]
    if not rows or any(r < 0 for r in rows) or sum(rows) != M:
        raise ValueError(f"slice_rows must be non-negative and sum to the {M} rows")
    return (ctypes.c_int64 * len(rows))(*rows), len(rows)


def _sliced_workspace(n, dev, workspace):
    if workspace is not None:
        return workspace
    return _empty(int(lib.mxq_nvfp4_sliced_workspace_bytes(n)), torch.uint8, dev)


def nvfp4_amax_sliced(x: torch.Tensor, slice_rows: Sequence[int],
                      workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Per-slice amax (non-NaN max |x|) of consecutive row ranges of x seen as
    [M, N], as an fp32 CUDA tensor [len(slice_rows)]."""
    _require_cuda(x)
    dt = _dtype_code(x.dtype)
    M, N, ld = _rows_view(x)
    rows, S = _slice_array(slice_rows, M)
    out = _zeros(S, torch.float32, x.device)
    ws = _sliced_workspace(S, x.device, workspace)
    _check("nvfp4_amax_sliced",
           lib.nvfp4_amax_sliced(_ptr(x), dt, M, N, ld, S, ctypes.cast(rows, ctypes.c_void_p),
                                 _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(x)))
    return out


def nvfp4_quantize_sliced(x: torch.Tensor, slice_rows: Sequence[int],
                          global_scales: torch.Tensor | None = None,
                          amax: torch.Tensor | None = None,
                          workspace: torch.Tensor | None = None):
    """NVFP4 quantize with one global scale per slice of consecutive rows of
    x seen as [M, N] (slice s holds slice_rows[s] rows): each slice is
    quantized as :func:`nvfp4_quantize` would quantize it alone.

    Returns ``(packed, block_scale, global_scales)`` with packed / block_scale
    shaped as for :func:`nvfp4_quantize` and fp32 ``global_scales``
    [len(slice_rows)]. ``global_scales`` (given g per slice) or ``amax``
    (given slice amaxes) skip the amax pass."""
    _require_cuda(x)
    dt = _dtype_code(x.dtype)
    M, N, ld = _rows_view(x)
    rows, S = _slice_array(slice_rows, M)
    dev = x.device
    packed = _empty((*x.shape[:-1], N // 2), torch.uint8, dev)
    bs = _empty((*x.shape[:-1], N // 16), torch.uint8, dev)
    flags = 0
    if global_scales is not None:
        if global_scales.dtype != torch.float32 or global_scales.numel() != S:
            raise TypeError("global_scales must be fp32 with one value per slice")
        g = global_scales.to(dev).contiguous()
        flags = NVFP4_GLOBAL_GIVEN
    else:
        g = _zeros(S, torch.float32, dev)
    if amax is not None:
        if amax.dtype != torch.float32 or amax.numel() != S:
            raise TypeError("amax must be fp32 with one value per slice")
        amax = amax.contiguous()
    ws = None
    if global_scales is None and amax is None:
        ws = _sliced_workspace(S, dev, workspace)
    _check("nvfp4_quantize_sliced",
           lib.nvfp4_quantize_sliced(_ptr(x), dt, M, N, ld, S, ctypes.cast(rows, ctypes.c_void_p),
                                     _ptr(packed), _ptr(bs), _ptr(g), _ptr(amax), flags, _ptr(ws),
                                     0 if ws is None else ws.numel() * ws.element_size(),
                                     _stream(x)))
    return packed, bs, g


def nvfp4_quantize_experts(w: torch.Tensor, *, per_half: bool = False,
                           global_scales: torch.Tensor | None = None):
    """NVFP4 of a stacked expert weight [E, R, N] with one global scale per
    expert, or with ``per_half=True`` one per half of each expert's rows
    (fused gate/up weights: rows [0, R/2) gate, [R/2, R) up).

    Returns ``(packed [E, R, N/2], block_scale [E, R, N/16], global_scales)``
    with global_scales fp32 [E] or [E, 2]."""
    if w.dim() != 3:
        raise ValueError("expected a stacked [E, R, N] weight")
    E, R, _ = w.shape
    if per_half and R % 2:
        raise ValueError("per_half needs an even number of rows per expert")
    rows = [R // 2] * (2 * E) if per_half else [R] * E
    gs = None if global_scales is None else global_scales.reshape(-1)
    p, b, g = nvfp4_quantize_sliced(w, rows, global_scales=gs)
    return p, b, g.view(E, 2) if per_half else g


def nvfp4_dequantize(packed: torch.Tensor, block_scale: torch.Tensor, global_scale: torch.Tensor,
                     dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """E2M1 code * (E4M3 block scale * g), as bf16 (RNE) or fp32."""
    _require_cuda(packed, block_scale, global_scale)
    if not (packed.is_contiguous() and block_scale.is_contiguous()):
        raise ValueError("packed and block_scale must be contiguous")
    N = packed.shape[-1] * 2
    M = packed.numel() * 2 // N if N else 0
    if block_scale.numel() != M * (N // 16):
        raise ValueError("block_scale does not match packed")
    y = _empty((*packed.shape[:-1], N), dtype, packed.device)
    _check("nvfp4_dequantize",
           lib.nvfp4_dequantize(_ptr(packed), _ptr(block_scale), _ptr(global_scale), M, N, _ptr(y),
                                _dtype_code(dtype), _stream(packed)))
    return y


# ------------------------------------------------------------------ views

def as_float8_e4m3(q: torch.Tensor) -> torch.Tensor:
    return q.view(torch.float8_e4m3fn)


def as_float8_e8m0(s: torch.Tensor) -> torch.Tensor:
    return s.view(torch.float8_e8m0fnu)


def as_float4_e2m1x2(p: torch.Tensor) -> torch.Tensor:
    return p.view(torch.float4_e2m1fn_x2)


# ------------------------------------------------------------------ NVTX

_nvtx = False


def set_nvtx(enabled: bool) -> bool:
    """Wrap every quantization call of this module in an NVTX range named
    ``mxq.<function>`` (for a profiler's timeline) when ``enabled``; off by
    default. Returns the previous setting."""
    global _nvtx
    prev, _nvtx = _nvtx, bool(enabled)
    return prev


def _traced(fn):
    name = "mxq." + fn.__name__

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        if not _nvtx:
            return fn(*args, **kwargs)
        torch.cuda.nvtx.range_push(name)
        try:
            return fn(*args, **kwargs)
        finally:
            torch.cuda.nvtx.range_pop()
    return wrapper


for _name in ("mxfp8_quantize", "mxfp8_dequantize", "mxfp8_quantize_grouped",
              "mxfp8_quantize_columnwise", "mxfp4_quantize", "mxfp4_dequantize",
              "mxfp4_quantize_grouped", "mx_fake_quantize", "mxfp8_gemm", "nvfp4_amax",
              "nvfp4_quantize", "nvfp4_dequantize", "nvfp4_amax_sliced", "nvfp4_quantize_sliced",
              "nvfp4_quantize_experts", "swizzle_scales"):
    globals()[_name] = _traced(globals()[_name])
del _name
