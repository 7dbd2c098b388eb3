"""CPU oracle for block-scaled quantization (MXFP8 / NVFP4).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library and
its Python binding never import it, and it imports nothing from them: the two
share no code.

The arithmetic lives in ``mxq_oracle.c`` (plain scalar C, one element at a
time); this module builds it with gcc and exposes numpy-facing wrappers. The
two compositions defined here, the row pad-and-crop adapter and the grouped
quantize, are written out literally from their definitions:

* "PR #1935 完整报告 -- Use TransformerEngine for MXFP8 quantization",
  实现拆解 item 1: flatten the tensor, zero-pad rows to a multiple of 32,
  quantize rowwise with group 32, crop back, return compact (qweight, scale).
* Grouped quantize of a stack of expert weights ("PR #1935 ...", 实现拆解
  item 4, ``mxfp8_group_quantize``): one result per expert, identical to
  quantizing each expert on its own; outputs concatenated along rows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmxq_oracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
           "-fexcess-precision=standard", "-fPIC", "-shared"]

BF16 = 0
FP32 = 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmxq_oracle.so`` (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            u8, i64, vp, i32 = ctypes.c_uint8, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
            f64, f32 = ctypes.c_double, ctypes.c_float
            L.orc_e8m0_from_amax.argtypes, L.orc_e8m0_from_amax.restype = [f64], u8
            L.orc_e8m0_value.argtypes, L.orc_e8m0_value.restype = [u8], f64
            L.orc_e4m3_encode.argtypes, L.orc_e4m3_encode.restype = [f64], u8
            L.orc_e4m3_decode.argtypes, L.orc_e4m3_decode.restype = [u8], f64
            L.orc_e2m1_encode.argtypes, L.orc_e2m1_encode.restype = [f64], u8
            L.orc_e2m1_decode.argtypes, L.orc_e2m1_decode.restype = [u8], f64
            L.orc_bf16_round.argtypes, L.orc_bf16_round.restype = [f64], ctypes.c_uint16
            L.orc_mxfp8_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp]
            L.orc_mxfp8_dequantize.argtypes = [vp, vp, i64, i64, vp, i32]
            L.orc_swizzle_scales.argtypes = [vp, i64, i64, vp]
            L.orc_mxfp8_quantize_colwise.argtypes = [vp, i32, i64, i64, i64, vp, vp]
            L.orc_mxfp4_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp]
            L.orc_mxfp4_dequantize.argtypes = [vp, vp, i64, i64, vp, i32]
            L.orc_e8m0_from_amax_emax.argtypes = [f64, i32]
            L.orc_e8m0_from_amax_emax.restype = u8
            L.orc_nvfp4_global_amax.argtypes = [vp, i32, i64, i64, i64]
            L.orc_nvfp4_global_amax.restype = f32
            L.orc_nvfp4_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, i32]
            L.orc_nvfp4_dequantize.argtypes = [vp, vp, f32, i64, i64, vp, i32]
            L.orc_nvfp4_quantize_sliced.argtypes = [vp, i32, i64, i64, i64, i32, vp, vp, vp, vp, i32]
            for f in ("orc_e4m3_encode_array", "orc_e2m1_encode_array",
                      "orc_e8m0_from_amax_array", "orc_bf16_round_array"):
                getattr(L, f).argtypes = [vp, i64, vp]
                getattr(L, f).restype = None
            for f in ("orc_mxfp8_quantize", "orc_mxfp8_dequantize", "orc_swizzle_scales",
                      "orc_mxfp8_quantize_colwise", "orc_mxfp4_quantize", "orc_mxfp4_dequantize",
                      "orc_nvfp4_quantize", "orc_nvfp4_dequantize", "orc_nvfp4_quantize_sliced"):
                getattr(L, f).restype = i32
            _lib = L
    return _lib


# ----------------------------------------------------------------- helpers

def _as_input(x: np.ndarray):
    """(array, dtype code) for a bf16-bits (uint16) or float32 array."""
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), BF16
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), FP32
    raise TypeError("oracle inputs are bf16 bit patterns (uint16) or float32")


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: status {rc}")


# ------------------------------------------------------------ scalar codecs

def e8m0_from_amax(amax: float) -> int:
    return int(lib().orc_e8m0_from_amax(float(amax)))


def e8m0_value(b: int) -> float:
    return float(lib().orc_e8m0_value(b))


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_decode(c: int) -> float:
    return float(lib().orc_e4m3_decode(c))


def e2m1_encode(u: float) -> int:
    return int(lib().orc_e2m1_encode(float(u)))


def e2m1_decode(c: int) -> float:
    return float(lib().orc_e2m1_decode(c))


def bf16_round(d: float) -> int:
    return int(lib().orc_bf16_round(float(d)))


def _batch(fname, values, out_dtype):
    v = np.ascontiguousarray(values, np.float64).reshape(-1)
    out = np.empty(v.size, out_dtype)
    getattr(lib(), fname)(_ptr(v), v.size, _ptr(out))
    return out.reshape(np.shape(values))


def e4m3_encode_array(v) -> np.ndarray:
    return _batch("orc_e4m3_encode_array", v, np.uint8)


def e2m1_encode_array(u) -> np.ndarray:
    return _batch("orc_e2m1_encode_array", u, np.uint8)


def e8m0_from_amax_array(a) -> np.ndarray:
    return _batch("orc_e8m0_from_amax_array", a, np.uint8)


def bf16_round_array(d) -> np.ndarray:
    return _batch("orc_bf16_round_array", d, np.uint16)


# -------------------------------------------------------------------- MXFP8

def mxfp8_quantize(x: np.ndarray):
    """Rowwise MXFP8 of a 2-D input [M, N] (uint16 bf16 bits or float32).
    Returns (qweight uint8 [M, N], scale uint8 [M, N/32])."""
    a, dt = _as_input(x)
    M, N = a.shape
    q = np.empty((M, N), np.uint8)
    s = np.empty((M, N // 32), np.uint8)
    _check(lib().orc_mxfp8_quantize(_ptr(a), dt, M, N, N, _ptr(q), _ptr(s)), "mxfp8_quantize")
    return q, s


def mxfp8_quantize_strided(buf: np.ndarray, M: int, N: int, ld_x: int):
    """Rowwise MXFP8 of M rows of N elements read from a flat buffer with row
    stride ld_x elements."""
    a, dt = _as_input(buf.reshape(-1))
    if M and a.size < (M - 1) * ld_x + N:
        raise ValueError("buffer too small for M rows of stride ld_x")
    q = np.empty((M, N), np.uint8)
    s = np.empty((M, N // 32), np.uint8)
    _check(lib().orc_mxfp8_quantize(_ptr(a), dt, M, N, ld_x, _ptr(q), _ptr(s)), "mxfp8_quantize")
    return q, s


def mxfp8_quantize_padded(x: np.ndarray, row_align: int = 32):
    """The pages' adapter contract, written out literally: flatten to
    [M, N], zero-pad the rows to a multiple of ``row_align``, quantize, crop
    back to M rows. Returns compact (qweight [*x.shape], scale
    [*x.shape[:-1], N/32])."""
    lead = x.shape[:-1]
    N = x.shape[-1]
    flat = x.reshape(-1, N)
    M = flat.shape[0]
    Mp = (M + row_align - 1) // row_align * row_align
    padded = np.zeros((Mp, N), dtype=x.dtype)
    padded[:M] = flat
    q, s = mxfp8_quantize(padded)
    return q[:M].reshape(*lead, N), s[:M].reshape(*lead, N // 32)


def mxfp8_quantize_colwise(x: np.ndarray):
    """Columnwise MXFP8 of a 2-D input [M, N]: groups of 32 rows per column,
    rows past M counting as zeros. Returns transposed, cropped outputs
    (q_t uint8 [N, M], scale_t uint8 [N, ceil(M/32)])."""
    a, dt = _as_input(x)
    M, N = a.shape
    q_t = np.empty((N, M), np.uint8)
    s_t = np.empty((N, (M + 31) // 32), np.uint8)
    _check(lib().orc_mxfp8_quantize_colwise(_ptr(a), dt, M, N, N, _ptr(q_t), _ptr(s_t)),
           "mxfp8_quantize_colwise")
    return q_t, s_t


def mxfp8_dequantize(q: np.ndarray, s: np.ndarray, out: str = "bf16") -> np.ndarray:
    """Returns uint16 bf16 bits or float32 [M, N]."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    M, N = q.shape
    if out == "bf16":
        y = np.empty((M, N), np.uint16)
        dt = BF16
    else:
        y = np.empty((M, N), np.float32)
        dt = FP32
    _check(lib().orc_mxfp8_dequantize(_ptr(q), _ptr(s), M, N, _ptr(y), dt), "mxfp8_dequantize")
    return y


def swizzle_scales(s: np.ndarray) -> np.ndarray:
    """Flat uint8 array of ceil(M/128)*128 * ceil(S/4)*4 bytes."""
    s = np.ascontiguousarray(s, np.uint8)
    M, S = s.shape
    Mp, Sp = (M + 127) // 128 * 128, (S + 3) // 4 * 4
    out = np.empty(Mp * Sp, np.uint8)
    _check(lib().orc_swizzle_scales(_ptr(s), M, S, _ptr(out)), "swizzle_scales")
    return out


def _grouped(quantize, xs, swizzled):
    qs, ss = [], []
    for x in xs:
        q, s = quantize(x)
        qs.append(q)
        ss.append(s)
    out = (np.concatenate(qs, 0), np.concatenate(ss, 0))
    if swizzled:
        out += (np.concatenate([swizzle_scales(s) for s in ss]),)
    return out


def mxfp8_quantize_grouped(xs, swizzled: bool = False):
    """Grouped MXFP8 of a list of expert inputs [M_e, N] (shared N): each
    expert quantized on its own, results concatenated along rows. With
    ``swizzled``, also each expert's scales in its own 128x4-tile layout
    (``swizzle_scales`` of that expert's compact scales), the experts' blocks
    concatenated in expert order, as a grouped block-scaled GEMM reads one
    scale matrix per expert."""
    return _grouped(mxfp8_quantize, xs, swizzled)


# -------------------------------------------------------------------- MXFP4

def e8m0_from_amax_emax(amax: float, emax: int) -> int:
    return int(lib().orc_e8m0_from_amax_emax(float(amax), emax))


def mxfp4_quantize(x: np.ndarray):
    """Returns (packed uint8 [M, N/2], scale uint8 [M, N/32])."""
    a, dt = _as_input(x)
    M, N = a.shape
    packed = np.empty((M, N // 2), np.uint8)
    s = np.empty((M, N // 32), np.uint8)
    _check(lib().orc_mxfp4_quantize(_ptr(a), dt, M, N, N, _ptr(packed), _ptr(s)), "mxfp4_quantize")
    return packed, s


def mxfp4_quantize_grouped(xs, swizzled: bool = False):
    """Grouped MXFP4: as :func:`mxfp8_quantize_grouped` with MXFP4 codes."""
    return _grouped(mxfp4_quantize, xs, swizzled)


def mxfp4_dequantize(packed: np.ndarray, s: np.ndarray, out: str = "bf16") -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    M, half = packed.shape
    N = half * 2
    y = np.empty((M, N), np.uint16 if out == "bf16" else np.float32)
    _check(lib().orc_mxfp4_dequantize(_ptr(packed), _ptr(s), M, N, _ptr(y), BF16 if out == "bf16" else FP32),
           "mxfp4_dequantize")
    return y


def fake_quantize(x: np.ndarray, fmt: str, out: str = "bf16") -> np.ndarray:
    """QAT simulate ("V4 mxfp4 #1372": mxfp4_simulate_qat(kv, 32)): the
    dequantization of the quantization, for fmt "mxfp8" or "mxfp4"."""
    if fmt == "mxfp8":
        q, s = mxfp8_quantize(x)
        return mxfp8_dequantize(q, s, out=out)
    if fmt == "mxfp4":
        p, s = mxfp4_quantize(x)
        return mxfp4_dequantize(p, s, out=out)
    raise ValueError(fmt)


# --------------------------------------------------------------------- GEMM

def e4m3_decode_table() -> np.ndarray:
    """float64 values of the 256 E4M3 codes (NaN for 0x7F and 0xFF)."""
    return np.array([lib().orc_e4m3_decode(c) for c in range(256)], np.float64)


def mxfp8_gemm(qa: np.ndarray, sa: np.ndarray, qb: np.ndarray, sb: np.ndarray) -> np.ndarray:
    """The block-scaled product written out in float64: D = A B^T with
    A[m, k] = decode(qa[m, k]) * 2^(sa[m, k/32] - 127) and B likewise from
    (qb, sb). qa [M, K], qb [N, K] E4M3 codes; sa [M, K/32], sb [N, K/32]
    compact E8M0 bytes. Products are exact; the float64 sums are exact for
    the test inputs on a coarse grid and within K * 2^-53 of the exact sum
    otherwise."""
    qa = np.ascontiguousarray(qa, np.uint8)
    qb = np.ascontiguousarray(qb, np.uint8)
    t = e4m3_decode_table()
    K = qa.shape[1]
    ea = np.repeat(np.asarray(sa, np.int64) - 127, 32, axis=1)[:, :K]
    eb = np.repeat(np.asarray(sb, np.int64) - 127, 32, axis=1)[:, :K]
    A = np.ldexp(t[qa], ea)
    B = np.ldexp(t[qb], eb)
    return A @ B.T


# -------------------------------------------------------------------- NVFP4

def nvfp4_global_amax(x: np.ndarray) -> np.float32:
    a, dt = _as_input(x)
    M, N = a.shape
    return np.float32(lib().orc_nvfp4_global_amax(_ptr(a), dt, M, N, N))


def nvfp4_quantize(x: np.ndarray, global_scale: float | None = None):
    """Returns (packed uint8 [M, N/2], block_scale uint8 [M, N/16], g float32)."""
    a, dt = _as_input(x)
    M, N = a.shape
    packed = np.empty((M, N // 2), np.uint8)
    bs = np.empty((M, N // 16), np.uint8)
    g = np.zeros(1, np.float32)
    given = 0
    if global_scale is not None:
        g[0] = np.float32(global_scale)
        given = 1
    _check(lib().orc_nvfp4_quantize(_ptr(a), dt, M, N, N, _ptr(packed), _ptr(bs), _ptr(g), given),
           "nvfp4_quantize")
    return packed, bs, np.float32(g[0])


def nvfp4_quantize_sliced(x: np.ndarray, slice_rows, global_scales=None):
    """NVFP4 with one global scale per slice of consecutive rows ("Add FP8,
    NVFP4, and QARL training and export", _nvfp4_block_quantize_per_slice;
    per-half gate/up scales). Returns (packed [M, N/2], block_scale [M, N/16],
    g float32 [n_slices])."""
    a, dt = _as_input(x)
    M, N = a.shape
    rows = np.ascontiguousarray(slice_rows, np.int64)
    S = rows.shape[0]
    packed = np.empty((M, N // 2), np.uint8)
    bs = np.empty((M, N // 16), np.uint8)
    g = np.zeros(S, np.float32)
    given = 0
    if global_scales is not None:
        g[:] = np.asarray(global_scales, np.float32)
        given = 1
    _check(lib().orc_nvfp4_quantize_sliced(_ptr(a), dt, M, N, N, S, _ptr(rows), _ptr(packed),
                                           _ptr(bs), _ptr(g), given), "nvfp4_quantize_sliced")
    return packed, bs, g


def nvfp4_dequantize(packed: np.ndarray, bs: np.ndarray, g: float, out: str = "bf16") -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.uint8)
    bs = np.ascontiguousarray(bs, np.uint8)
    M, half = packed.shape
    N = half * 2
    if out == "bf16":
        y = np.empty((M, N), np.uint16)
        dt = BF16
    else:
        y = np.empty((M, N), np.float32)
        dt = FP32
    _check(lib().orc_nvfp4_dequantize(_ptr(packed), _ptr(bs), float(np.float32(g)), M, N, _ptr(y), dt),
           "nvfp4_dequantize")
    return y
