"""Pins of the oracle's scalar codecs against independent formulations.

E4M3 / E2M1 rounding: brute-force nearest-code search over the decoded code
tables (ties to the even code, saturation), exhaustive over every bf16 value
times every E8M0 scale, plus torch's float8_e4m3fn cast for in-range values.
E8M0: the fp32 exponent-field formula versus the oracle's floor(log2) one.
bf16 rounding: torch's fp32 -> bf16 cast.
"""
import numpy as np
import pytest
import torch

import refs


def all_bf16_values():
    return refs.bf16_bits_to_f64(np.arange(65536, dtype=np.uint32).astype(np.uint16))


def test_e4m3_decode_matches_torch_table(orc):
    table = refs.e4m3_table()
    mine = np.array([orc.e4m3_decode(c) for c in range(256)])
    assert np.array_equal(np.isnan(mine), np.isnan(table))
    ok = ~np.isnan(table)
    assert np.array_equal(mine[ok], table[ok])
    # signs of zero
    assert np.signbit(mine[0x80]) and not np.signbit(mine[0x00])
    assert sorted(np.flatnonzero(np.isnan(mine)).tolist()) == [0x7F, 0xFF]


def test_e4m3_encode_every_bf16_times_every_scale(orc):
    """Every bf16 value times every power of two 2^(127-b), b = 0..254, the
    exact set of values the MXFP8 cast sees for bf16 inputs."""
    xs = all_bf16_values()
    for b0 in range(0, 255, 51):
        bs = np.arange(b0, min(b0 + 51, 255))
        v = np.ldexp(xs[None, :], (127 - bs)[:, None]).reshape(-1)
        got = orc.e4m3_encode_array(v)
        want = refs.e4m3_brute(v)
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e4m3_encode_fp32_near_rounding_boundaries(orc):
    """fp32 inputs (24-bit significands) within +-64 ulp of every E4M3 value and
    every midpoint between neighbours."""
    grid = refs.e4m3_table()[:127]
    mids = (grid[:-1] + grid[1:]) / 2
    pts = np.concatenate([grid, mids, [464.0, 480.0, 512.0]]).astype(np.float32)
    base = pts.view(np.int32)[:, None] + np.arange(-64, 65, dtype=np.int32)[None, :]
    v = base.reshape(-1)
    v = v[(v >= 0)].view(np.float32).astype(np.float64)
    v = np.concatenate([v, -v])
    got = orc.e4m3_encode_array(v)
    want = refs.e4m3_brute(v)
    assert np.array_equal(got, want)


def test_e4m3_encode_matches_torch_cast_in_range(orc):
    rng = np.random.default_rng(11)
    v = np.concatenate([
        rng.uniform(-448, 448, 200000),
        rng.standard_normal(200000) * 0.01,
        np.ldexp(rng.uniform(-1, 1, 100000), rng.integers(-12, 9, 100000)),
    ]).astype(np.float32).astype(np.float64)
    got = orc.e4m3_encode_array(v)
    lib = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, lib)


def test_e4m3_specials(orc):
    assert orc.e4m3_encode(float("nan")) == 0x7F
    assert orc.e4m3_encode(-float("nan")) == 0x7F
    assert orc.e4m3_encode(float("inf")) == 0x7E
    assert orc.e4m3_encode(-float("inf")) == 0xFE
    assert orc.e4m3_encode(1e30) == 0x7E
    assert orc.e4m3_encode(-0.0) == 0x80
    assert orc.e4m3_encode(-1e-30) == 0x80
    assert orc.e4m3_encode(0.0) == 0x00
    assert orc.e4m3_encode(463.99) == 0x7E and orc.e4m3_encode(464.0) == 0x7E


def test_e2m1_decode_values(orc):
    mags = [orc.e2m1_decode(c) for c in range(8)]
    assert mags == list(refs.E2M1_MAGNITUDES)
    assert [orc.e2m1_decode(c | 8) for c in range(8)] == [-m for m in mags]


def test_e2m1_encode_dense_fp32_sample(orc):
    """Every 32nd fp32 bit pattern in [0, 8], plus +-256 ulp around every
    code value and midpoint, both signs."""
    top = np.float32(8.0).view(np.int32)
    dense = np.arange(0, top + 1, 32, dtype=np.int32)
    pts = np.concatenate([refs.E2M1_MAGNITUDES,
                          (refs.E2M1_MAGNITUDES[:-1] + refs.E2M1_MAGNITUDES[1:]) / 2,
                          [7.0, 8.0]]).astype(np.float32)
    near = (pts.view(np.int32)[:, None] + np.arange(-256, 257, dtype=np.int32)[None, :]).reshape(-1)
    bits = np.concatenate([dense, near[near >= 0]])
    u = bits.view(np.float32).astype(np.float64)
    u = np.concatenate([u, -u])
    got = orc.e2m1_encode_array(u)
    want = refs.e2m1_brute(u)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (u[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e2m1_ties_and_specials(orc):
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for u, c in ties.items():
        assert orc.e2m1_encode(u) == c, u
        assert orc.e2m1_encode(-u) == c | 8, -u
    assert orc.e2m1_encode(6.5) == 7 and orc.e2m1_encode(float("inf")) == 7
    assert orc.e2m1_encode(-float("inf")) == 0xF
    assert orc.e2m1_encode(float("nan")) == 7
    assert orc.e2m1_encode(-0.0) == 8


def test_e8m0_matches_exponent_field_formula(orc):
    rng = np.random.default_rng(12)
    pos_bf16 = refs.bf16_bits_to_f64(np.arange(0, 0x7F81, dtype=np.uint32).astype(np.uint16))
    rnd = rng.integers(0, 0x7F800001, 1_000_000, dtype=np.int64).astype(np.uint32).view(np.float32)
    pw = np.ldexp(1.0, np.arange(-149, 128)).astype(np.float32)
    around = np.concatenate([pw, np.nextafter(pw, np.float32(0)), np.nextafter(pw, np.float32(np.inf))])
    a = np.concatenate([pos_bf16, rnd.astype(np.float64), around.astype(np.float64)])
    got = orc.e8m0_from_amax_array(a)
    want = refs.e8m0_from_bits(a)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (a[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e8m0_closed_form(orc):
    """scale = 2^(floor(log2 amax) - 8): amax/scale lies in [256, 512) for
    every normal amax whose byte is not clamped."""
    rng = np.random.default_rng(13)
    a = np.ldexp(rng.uniform(1, 2, 100000), rng.integers(-118, 127, 100000)).astype(np.float32)
    b = orc.e8m0_from_amax_array(a.astype(np.float64)).astype(int)
    r = a.astype(np.float64) / np.ldexp(1.0, b - 127)
    assert np.all((r >= 256) & (r < 512))
    assert orc.e8m0_value(127) == 1.0 and np.isnan(orc.e8m0_value(255))
    assert orc.e8m0_from_amax(0.0) == 127 and orc.e8m0_from_amax(float("inf")) == 254


def test_bf16_round_matches_torch_on_every_dequant_value(orc):
    """Every E4M3 code times every E8M0 scale (the full set of MXFP8 dequant
    values), rounded to bf16."""
    table = refs.e4m3_table()
    d = (table[:, None] * np.ldexp(1.0, np.arange(0, 255) - 127)[None, :]).reshape(-1)
    d = d[~np.isnan(d)]
    got = orc.bf16_round_array(d)
    want = refs.f64_to_bf16_bits_torch(d)
    assert np.array_equal(got, want)


def test_bf16_round_random_fp32(orc):
    rng = np.random.default_rng(14)
    bits = rng.integers(0, 2**32, 1_000_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[~np.isnan(f)].astype(np.float64)
    assert np.array_equal(orc.bf16_round_array(f), refs.f64_to_bf16_bits_torch(f))
    assert orc.bf16_round(float("nan")) == 0x7FC0
    assert orc.bf16_round(2.0 ** -134) == 0x0000        # tie to even at the bottom
    assert orc.bf16_round(3 * 2.0 ** -135) == 0x0001
