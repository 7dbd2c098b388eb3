"""Seeded synthetic inputs for block-scaled quantization.

This module only draws random numbers and lays them out; it holds none of the
quantization arithmetic. Both the CUDA path and the CPU oracle consume the
bytes it returns. Every tensor is produced as float32 from
``numpy.random.default_rng(seed)`` and rounded to bf16 (round-to-nearest-even,
via torch's fp32 -> bf16 cast), and returned as bf16 bit patterns (uint16).

Workloads (one per benchmark configuration; shapes are parameters so the
tests can draw smaller instances of the same recipe):

1. ``planted``      bf16 [256, 1024] N(0,1), seed 0, plus hand-planted groups
                    in group 0 of rows 0-7 (all-zero, one 1e4 outlier, +-448,
                    bf16 subnormals, one NaN, one +Inf, E4M3 rounding ties,
                    largest bf16 magnitudes).
2. ``linear_weight``  bf16 [4096, 4096] N(0, 0.02), 0.1 % of entries replaced
                    by +-U(0.5, 4), seed 1.
3. ``activation``   bf16 [16384, 7168] Student-t(df=3) * 0.5; 1 % of the
                    32-element groups zeroed, a disjoint 0.5 % scaled by
                    2^-120, seed 2.
4. ``experts``      64 expert weights bf16 [2048, 7168], per-expert std from
                    U(0.01, 0.05), values N(0, std), seed 3.
5. ``nvfp4_tensor`` bf16 [8192, 8192] N(0,1) with 0.05 % of entries replaced
                    by +-U(20, 100), seed 4.

``normal_on_device`` is the one generator that draws on the GPU (torch's
seeded CUDA generator): it makes tensors of billions of elements that the host
generator would take minutes to produce. The oracle reads rows of such a
tensor copied back from the device.
"""
from __future__ import annotations

import numpy as np
import torch

BF16_MAX_BITS = 0x7F7F            # largest finite bf16 (about 3.39e38)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 bf16 bit patterns, round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_of(values, dtype=np.float32) -> np.ndarray:
    return to_bf16_bits(np.asarray(values, dtype=dtype))


# -------------------------------------------------------------- workload 1

# E4M3 rounding ties at scale byte 127 (the 448 entry pins the group's scale):
# 1.0625 (between 1 and 1.125), 1.1875 (between 1.125 and 1.25), 17 (between
# 16 and 18), 464 (between 448 and the nonexistent 480), 2^-10 (between 0 and
# the smallest subnormal), 3 * 2^-10 (between 2^-9 and 2^-8).
TIE_VALUES = [448.0, 1.0625, 1.1875, 17.0, 464.0, 2.0 ** -10, 3 * 2.0 ** -10,
              -1.0625, -1.1875, -17.0, -464.0, -(2.0 ** -10), -(3 * 2.0 ** -10)]


def planted(seed: int = 0, M: int = 256, N: int = 1024) -> np.ndarray:
    """Workload 1: N(0,1) with hand-planted groups in group 0 of rows 0-7
    (needs M >= 8, N >= 32)."""
    rng = np.random.default_rng(seed)
    x = to_bf16_bits(rng.standard_normal((M, N), dtype=np.float32))
    # row 0: all-zero group
    x[0, :32] = 0
    # row 1: one outlier 1e4 (bf16 9984)
    x[1, 5] = bits_of([1e4])[0]
    # row 2: +-448
    x[2, 0], x[2, 1] = bits_of([448.0, -448.0])
    # row 3: 32 bf16 subnormals +-k * 2^-133, k in [1, 127]
    k = rng.integers(1, 128, size=32).astype(np.uint16)
    sign = rng.integers(0, 2, size=32).astype(np.uint16) << 15
    x[3, :32] = k | sign
    # row 4: one NaN
    x[4, 7] = 0x7FC0
    # row 5: one +Inf
    x[5, 3] = 0x7F80
    # row 6: E4M3 rounding ties at scale byte 127
    x[6, :len(TIE_VALUES)] = bits_of(TIE_VALUES)
    # row 7: largest finite bf16 magnitudes
    x[7, 0], x[7, 1] = BF16_MAX_BITS, BF16_MAX_BITS | 0x8000
    return x


# -------------------------------------------------------------- workload 2

def linear_weight(seed: int = 1, M: int = 4096, N: int = 4096) -> np.ndarray:
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((M, N), dtype=np.float32) * np.float32(0.02)
    n_out = (M * N) // 1000                      # 0.1 %
    pos = rng.choice(M * N, size=n_out, replace=False)
    mag = rng.uniform(0.5, 4.0, size=n_out).astype(np.float32)
    sgn = np.where(rng.integers(0, 2, size=n_out) == 1, -1.0, 1.0).astype(np.float32)
    w.reshape(-1)[pos] = mag * sgn
    return to_bf16_bits(w)


# -------------------------------------------------------------- workload 3

def activation(seed: int = 2, M: int = 16384, N: int = 7168) -> np.ndarray:
    rng = np.random.default_rng(seed)
    a = (rng.standard_t(3.0, size=(M, N)) * 0.5).astype(np.float32)
    G = M * N // 32
    n_zero = G // 100                            # 1 %
    n_tiny = G // 200                            # 0.5 %
    idx = rng.choice(G, size=n_zero + n_tiny, replace=False)
    groups = a.reshape(G, 32)
    groups[idx[:n_zero]] = 0.0
    groups[idx[n_zero:]] *= np.float32(2.0 ** -120)
    return to_bf16_bits(a)


# -------------------------------------------------------------- workload 4

def experts(seed: int = 3, E: int = 64, M: int = 2048, N: int = 7168) -> np.ndarray:
    """Stacked expert weights, uint16 [E, M, N]."""
    rng = np.random.default_rng(seed)
    std = rng.uniform(0.01, 0.05, size=E).astype(np.float32)
    out = np.empty((E, M, N), np.uint16)
    for e in range(E):
        out[e] = to_bf16_bits(rng.standard_normal((M, N), dtype=np.float32) * std[e])
    return out


# -------------------------------------------------------------- workload 5

def nvfp4_tensor(seed: int = 4, M: int = 8192, N: int = 8192) -> np.ndarray:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, N), dtype=np.float32)
    n_out = (M * N) * 5 // 10000                 # 0.05 %
    pos = rng.choice(M * N, size=n_out, replace=False)
    mag = rng.uniform(20.0, 100.0, size=n_out).astype(np.float32)
    sgn = np.where(rng.integers(0, 2, size=n_out) == 1, -1.0, 1.0).astype(np.float32)
    x.reshape(-1)[pos] = mag * sgn
    return to_bf16_bits(x)


WORKLOADS = {
    "planted": dict(fn=planted, shape=(256, 1024), op="mxfp8 quantize+dequantize"),
    "linear_weight": dict(fn=linear_weight, shape=(4096, 4096), op="mxfp8 quantize"),
    "activation": dict(fn=activation, shape=(16384, 7168),
                       op="mxfp8 quantize (+swizzled scales) + dequantize"),
    "experts": dict(fn=experts, shape=(64, 2048, 7168), op="grouped mxfp8 quantize"),
    "nvfp4_tensor": dict(fn=nvfp4_tensor, shape=(8192, 8192), op="nvfp4 quantize"),
}


# ------------------------------------------------------ structured sweeps

def mxfp8_every_value_every_scale() -> np.ndarray:
    """bf16 [M, 1024] covering every (bf16 value, E8M0 byte) pair that can
    occur together: for each byte b in 0..246 the groups start with
    1.5 * 2^(b - 119) (amax with floor(log2) = b - 119, i.e. byte b) followed
    by every bf16 pattern of magnitude below 2^(b - 118) and every NaN
    pattern; for byte 254 the groups start with +inf and hold every pattern.
    Groups are 1 planted + 31 swept elements; the tail is zero-filled."""
    allp = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mag_e = (allp >> 7) & 0xFF                       # exponent field
    is_nan = ((allp & 0x7FFF) > 0x7F80)
    groups = []
    for b in range(0, 247):
        lead = to_bf16_bits(np.array([1.5 * 2.0 ** (b - 119)], np.float32))[0]
        vals = allp[((mag_e <= b + 8) & ~is_nan) | is_nan]
        n = (len(vals) + 30) // 31
        g = np.zeros((n, 32), np.uint16)
        g[:, 0] = lead
        flat = np.zeros(n * 31, np.uint16)
        flat[:len(vals)] = vals
        g[:, 1:] = flat.reshape(n, 31)
        groups.append(g)
    n = (65536 + 30) // 31
    g = np.zeros((n, 32), np.uint16)
    g[:, 0] = 0x7F80
    flat = np.zeros(n * 31, np.uint16)
    flat[:65536] = allp
    g[:, 1:] = flat.reshape(n, 31)
    groups.append(g)
    allg = np.concatenate(groups, 0)
    per_row = 32
    rows = (allg.shape[0] + per_row - 1) // per_row
    out = np.zeros((rows * per_row, 32), np.uint16)
    out[:allg.shape[0]] = allg
    return out.reshape(rows, per_row * 32)


def mx_every_value_every_exponent() -> np.ndarray:
    """bf16 [M, 1024] pairing every bf16 pattern with every group-amax
    exponent field e in 0..255 that can hold it: for e in 1..254 the groups
    start with 1.5 * 2^(e - 127) (for e == 0 with the largest subnormal,
    for e == 255 with +inf) followed by every pattern whose exponent field is
    at most e, and every NaN pattern. Covers every scale byte of any MX
    element format. Groups are 1 planted + 31 swept elements."""
    allp = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mag_e = (allp >> 7) & 0xFF
    is_nan = ((allp & 0x7FFF) > 0x7F80)
    groups = []
    for e in range(256):
        if e == 0:
            lead = 0x007F
        elif e == 255:
            lead = 0x7F80
        else:
            lead = (e << 7) | 0x40
        vals = allp[((mag_e <= e) & ~is_nan) | is_nan] if e < 255 else allp
        n = (len(vals) + 30) // 31
        g = np.zeros((n, 32), np.uint16)
        g[:, 0] = lead
        flat = np.zeros(n * 31, np.uint16)
        flat[:len(vals)] = vals
        g[:, 1:] = flat.reshape(n, 31)
        groups.append(g)
    allg = np.concatenate(groups, 0)
    rows = (allg.shape[0] + 31) // 32
    out = np.zeros((rows * 32, 32), np.uint16)
    out[:allg.shape[0]] = allg
    return out.reshape(rows, 1024)


def mx_all_packed_scale_pairs():
    """(packed [256, 256], scale [256, 16]): row r carries scale byte r on
    every group of 32 elements and the 256 byte values (every pair of E2M1
    codes) once, so every (code, byte) pair is dequantized."""
    q = np.tile(np.arange(256, dtype=np.uint8), (256, 1))
    s = np.repeat(np.arange(256, dtype=np.uint8)[:, None], 16, axis=1)
    return q, s


def gemm_pow2_operand(seed: int, rows: int, K: int) -> np.ndarray:
    """bf16 [rows, K] for exact GEMM checks: each element is 0 or +-2^g with
    g drawn per 32-element group from {-2, ..., 2} (about a quarter zeros), so
    groups carry different power-of-two magnitudes, every element is exactly
    representable after quantization, and all products and partial sums of
    two such operands lie on the grid 2^-4 within 2^(log2 K + 4)."""
    rng = np.random.default_rng(seed)
    g = rng.integers(-2, 3, (rows, K // 32))
    mag = np.repeat(np.ldexp(1.0, g), 32, axis=1)
    sign = rng.choice(np.array([-1.0, 0.0, 1.0, 1.0]), (rows, K))
    return to_bf16_bits((sign * mag).astype(np.float32))


def mxfp8_all_code_scale_pairs():
    """(qweight [256, 8192], scale [256, 256]): row r carries scale byte r on
    every group and the 256 E4M3 codes repeated, so every (code, byte) pair
    is dequantized."""
    q = np.tile(np.arange(256, dtype=np.uint8), (256, 32))
    s = np.repeat(np.arange(256, dtype=np.uint8)[:, None], 256, axis=1)
    return q, s


def nvfp4_e2m1_sweep_fp32() -> np.ndarray:
    """fp32 [M, 256] blocks of 16 whose first element is 6 (with a global
    scale of 1 every block gets scale 1.0 and eff = 1) and whose other 15
    elements sweep fp32 values in [-6, 6]: every 64th bit pattern in [0, 6]
    plus +-512 ulp around each E2M1 value and midpoint, both signs."""
    top = np.float32(6.0).view(np.int32)
    dense = np.arange(0, top + 1, 64, dtype=np.int32)
    pts = np.array([0, 0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6], np.float32)
    near = (pts.view(np.int32)[:, None] + np.arange(-512, 513, dtype=np.int32)[None, :]).reshape(-1)
    near = near[(near >= 0) & (near <= top)]
    v = np.concatenate([dense, near]).view(np.float32)
    v = np.concatenate([v, -v])
    nb = (v.size + 14) // 15
    blocks = np.zeros((nb, 16), np.float32)
    blocks[:, 0] = 6.0
    flat = np.zeros(nb * 15, np.float32)
    flat[:v.size] = v
    blocks[:, 1:] = flat.reshape(nb, 15)
    rows = (nb + 15) // 16
    out = np.zeros((rows * 16, 16), np.float32)
    out[:nb] = blocks
    return out.reshape(rows, 256)


def nvfp4_block_scale_sweep_fp32(seed: int = 5) -> np.ndarray:
    """fp32 [M, 256] blocks whose amax sweeps the E4M3 block-scale range
    (log-uniform over [2^-14, 2^12] plus values near 6 * every E4M3 value and
    midpoint), the other elements uniform in [-amax, amax]."""
    rng = np.random.default_rng(seed)
    from_log = np.exp2(rng.uniform(-14, 12, 40000)).astype(np.float32)
    codes = np.array([m * 2.0 ** e for e in range(-9, 9) for m in (1, 1.0625, 1.125, 1.1875, 1.25,
                      1.375, 1.5, 1.625, 1.75, 1.875)], np.float32) * np.float32(6.0)
    near = (codes.view(np.int32)[:, None] + np.arange(-3, 4, dtype=np.int32)[None, :]).reshape(-1)
    amax = np.concatenate([from_log, near.view(np.float32)])
    nb = amax.size
    rows = (nb + 15) // 16
    blocks = (rng.uniform(-1, 1, (rows * 16, 16)).astype(np.float32)
              * np.resize(amax, rows * 16)[:, None])
    blocks[:, 0] = np.resize(amax, rows * 16)
    return blocks.reshape(rows, 256)


# ------------------------------------------------------------ large inputs

def normal_on_device(M: int, N: int, seed: int, device="cuda") -> torch.Tensor:
    """bf16 [M, N] N(0,1) drawn on the device by torch's seeded CUDA
    generator, in row chunks (each chunk drawn in fp32 and cast to bf16)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 26) // max(N, 1))
    for r in range(0, M, step):
        x[r:r + step] = torch.randn((min(step, M - r), N), generator=gen, device=device,
                                    dtype=torch.float32).to(torch.bfloat16)
    return x
