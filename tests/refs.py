"""Independent formulations used to pin the oracle (test-only).

None of these reuse the oracle's arithmetic: rounding is done by brute-force
nearest-code search over decoded code tables (decoded by torch's float8 casts)
or by torch's own dtype casts, and the E8M0 byte by the fp32 exponent field.
"""
from __future__ import annotations

import numpy as np
import torch


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 values (exact)."""
    u32 = bits.astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return u32.view(np.float32).astype(np.float64)


def f64_to_bf16_bits_torch(d: np.ndarray) -> np.ndarray:
    """RNE to bf16 by torch's fp32 -> bf16 cast (d must be fp32-exact)."""
    t = torch.from_numpy(np.ascontiguousarray(d, np.float64)).to(torch.float32)
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def e4m3_table() -> np.ndarray:
    """Values of the 256 E4M3 codes, decoded by torch's float8_e4m3fn cast."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def nearest_code(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each a >= 0 (grid sorted, finite,
    a within [0, grid[-1]]); ties go to the even index."""
    hi = np.searchsorted(grid, a, side="left")
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    dlo = np.abs(a - grid[lo])
    dhi = np.abs(grid[hi] - a)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo)


def e4m3_brute(v: np.ndarray) -> np.ndarray:
    """E4M3 code of exact values v by nearest-code search, saturating to 448,
    NaN -> 0x7F, zero sign kept."""
    v = np.asarray(v, np.float64)
    grid = e4m3_table()[:127]                 # codes 0x00..0x7E, increasing
    a = np.minimum(np.abs(np.nan_to_num(v, nan=0.0)), 448.0)
    code = nearest_code(a, grid).astype(np.uint8)
    code = code | np.where(np.signbit(v), 0x80, 0).astype(np.uint8)
    return np.where(np.isnan(v), np.uint8(0x7F), code)


def e2m1_brute(u: np.ndarray) -> np.ndarray:
    u = np.asarray(u, np.float64)
    a = np.minimum(np.abs(np.nan_to_num(u, nan=0.0)), 6.0)
    code = nearest_code(a, E2M1_MAGNITUDES).astype(np.uint8)
    code = code | np.where(np.signbit(u), 0x8, 0).astype(np.uint8)
    return np.where(np.isnan(u), np.uint8(0x7), code)


def e8m0_from_bits(a: np.ndarray) -> np.ndarray:
    """Byte from the fp32 exponent field E of amax: clamp(E - 8, 0, 254),
    127 for zero, 254 for infinity."""
    a32 = np.asarray(a, np.float32)
    E = (a32.view(np.uint32) >> 23).astype(np.int64) & 0xFF
    b = np.clip(E - 8, 0, 254)
    b = np.where(a32 == 0, 127, b)
    b = np.where(np.isinf(a32), 254, b)
    return b.astype(np.uint8)


def mxfp8_quantize_torch(xbits: np.ndarray):
    """MXFP8 rowwise quantize written with torch tensor ops: the NaN-ignoring
    group amax, the exponent-field byte, and torch's float8_e4m3fn cast of the
    power-of-two-scaled values (clamped to +-448 first so the cast never sees
    an out-of-range value)."""
    M, N = xbits.shape
    x = torch.from_numpy(bf16_bits_to_f64(xbits)).view(M, N // 32, 32)
    a = torch.where(torch.isnan(x), torch.zeros_like(x), x.abs()).amax(-1)
    b = torch.from_numpy(e8m0_from_bits(a.numpy()).astype(np.int64))
    v = torch.ldexp(x, (127 - b).unsqueeze(-1).to(torch.float64))
    vc = v.clamp(-448.0, 448.0)
    q = vc.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    q[np.isnan(v.numpy())] = 0x7F
    return q.reshape(M, N), b.numpy().astype(np.uint8).reshape(M, N // 32)


def mxfp8_dequantize_torch(q: np.ndarray, s: np.ndarray):
    """(float32 array, bf16 bits) of decode(q) * 2^(s - 127) with torch ops."""
    M, N = q.shape
    qt = torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64)
    e = torch.from_numpy(s.astype(np.int64)).repeat_interleave(32, dim=1) - 127
    d = torch.ldexp(qt, e.to(torch.float64))
    f32 = d.to(torch.float32).numpy().copy()
    nan = np.isnan(f32)
    f32.view(np.uint32)[nan] = 0x7FC00000
    bf = d.to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    bf[nan] = 0x7FC0
    return f32, bf


def swizzle_torch(s: np.ndarray) -> np.ndarray:
    """128x4 scale tiles by a tensor reshape/permute: [Mp, Sp] ->
    (Mp/128, 4, 32, Sp/4, 4) -> (i, j, r%32, r/32 within tile, c%4)."""
    M, S = s.shape
    Mp, Sp = (M + 127) // 128 * 128, (S + 3) // 4 * 4
    p = torch.zeros((Mp, Sp), dtype=torch.uint8)
    p[:M, :S] = torch.from_numpy(np.ascontiguousarray(s))
    t = p.view(Mp // 128, 4, 32, Sp // 4, 4).permute(0, 3, 2, 1, 4).contiguous()
    return t.view(-1).numpy()


def nvfp4_quantize_torch(xbits: np.ndarray, g: float | None = None):
    """NVFP4 two-level quantize with torch fp32 tensor ops, torch's
    float8_e4m3fn cast for the block scale and nearest-code search for E2M1."""
    M, N = xbits.shape
    x = torch.from_numpy(bf16_bits_to_f64(xbits).astype(np.float32)).view(M, N // 16, 16)
    absx = torch.where(torch.isnan(x), torch.zeros_like(x), x.abs())
    if g is None:
        g_t = absx.amax() / torch.tensor(2688.0, dtype=torch.float32)
    else:
        g_t = torch.tensor(g, dtype=torch.float32)
    amax_b = absx.amax(-1)
    if float(g_t) == 0.0:
        sb = torch.zeros_like(amax_b).to(torch.float8_e4m3fn)
        eff = torch.zeros_like(amax_b)
    else:
        t = torch.tensor(6.0, dtype=torch.float32) * g_t
        s = amax_b / t
        sb = s.clamp(max=448.0).to(torch.float8_e4m3fn)
        eff = sb.to(torch.float32) * g_t
    u = x / eff.unsqueeze(-1)
    codes = e2m1_brute(u.numpy().astype(np.float64))
    zero = (eff == 0).unsqueeze(-1).expand_as(x).numpy()
    codes = np.where(zero, np.where(np.signbit(x.numpy()), 0x8, 0x0), codes).astype(np.uint8)
    codes = codes.reshape(M, N)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb.view(torch.uint8).numpy().reshape(M, N // 16), np.float32(g_t)
