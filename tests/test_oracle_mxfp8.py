"""Pins of the oracle's MXFP8 quantize / dequantize / swizzle / grouped.

* Hand-worked groups (tests/golden/hand_worked.json), computed by hand.
* A torch tensor-op formulation (refs.mxfp8_quantize_torch) on inputs drawn
  by the workload recipes, including the planted special groups.
* Invariants: idempotence of quantize(dequantize(.)), the per-element error
  bound, pad-and-crop equals direct, grouped equals per-expert equals
  flattened, strided equals contiguous.
"""
import json
import os

import numpy as np
import pytest

import refs
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _val(s):
    if isinstance(s, str) and s.startswith("0x"):
        return refs.bf16_bits_to_f64(np.array([int(s, 16)], np.uint16))[0]
    return float(s)


def _group(spec, n=32):
    out = [spec["fill"]] * n
    for k, v in spec["x"].items():
        out[int(k)] = v
    return out


def _to_bits(vals):
    bits = []
    for s in vals:
        if isinstance(s, str) and s.startswith("0x"):
            bits.append(int(s, 16))
        else:
            bits.append(int(W.bits_of([float(s)])[0]))
    return np.array(bits, np.uint16)


def _expand(d, n, conv):
    out = [conv(d["fill"])] * n
    for k, v in d.items():
        if k != "fill":
            out[int(k)] = conv(v)
    return out


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["mxfp8"], ids=lambda c: c["name"])
def test_hand_worked_group(orc, case):
    x = _to_bits(_group(case))[None, :]
    q, s = orc.mxfp8_quantize(x)
    assert int(s[0, 0]) == case["scale"], case["why"]
    assert q[0].tolist() == _expand(case["q"], 32, int), case["why"]
    y = orc.mxfp8_dequantize(q, s, out="f32")[0].astype(np.float64)
    want = np.array(_expand(case["dq_f32"], 32, _val))
    assert np.array_equal(np.isnan(y), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(y[ok], want[ok])
    assert np.array_equal(np.signbit(y[ok]), np.signbit(want[ok]))


def _compare_torch(orc, x):
    q, s = orc.mxfp8_quantize(x)
    qt, st = refs.mxfp8_quantize_torch(x)
    assert np.array_equal(s, st)
    assert np.array_equal(q, qt)
    f32, bf = refs.mxfp8_dequantize_torch(q, s)
    assert np.array_equal(orc.mxfp8_dequantize(q, s, out="f32").view(np.uint32), f32.view(np.uint32))
    assert np.array_equal(orc.mxfp8_dequantize(q, s, out="bf16"), bf)
    return q, s


def test_planted_workload_matches_torch(orc):
    _compare_torch(orc, W.planted())


def test_weight_and_activation_recipes_match_torch(orc):
    _compare_torch(orc, W.linear_weight(M=256, N=512))
    _compare_torch(orc, W.activation(M=192, N=7168))


def test_every_bf16_pattern_through_quantize(orc):
    """All 65536 bf16 patterns laid out as 2048 groups (NaN/Inf included)."""
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(64, 1024)
    _compare_torch(orc, x)
    rng = np.random.default_rng(5)
    _compare_torch(orc, rng.permutation(x.reshape(-1)).reshape(64, 1024))


def test_fp32_input_matches_bf16_widening(orc):
    """An fp32 tensor holding bf16 values quantizes like the bf16 tensor."""
    x = W.planted(M=64, N=256)
    xf = refs.bf16_bits_to_f64(x).astype(np.float32)
    q1, s1 = orc.mxfp8_quantize(x)
    q2, s2 = orc.mxfp8_quantize(xf)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_fp32_input_full_precision(orc):
    """fp32 inputs with 24-bit significands against the torch formulation on
    fp32 values (byte from the exponent field, torch's e4m3 cast)."""
    rng = np.random.default_rng(6)
    xf = (rng.standard_t(3, (64, 512)) * 0.5).astype(np.float32)
    q, s = orc.mxfp8_quantize(xf)
    g = xf.astype(np.float64).reshape(64, 16, 32)
    b = refs.e8m0_from_bits(np.abs(g).max(-1))
    v = np.ldexp(g, (127 - b.astype(np.int64))[..., None])
    assert np.array_equal(s, b)
    assert np.array_equal(q, refs.e4m3_brute(v).reshape(64, 512))


def test_idempotent_requantize(orc):
    for x in (W.planted(), W.activation(M=64, N=1024)):
        q, s = orc.mxfp8_quantize(x)
        y = orc.mxfp8_dequantize(q, s, out="f32")
        q2, s2 = orc.mxfp8_quantize(y)
        assert np.array_equal(q, q2) and np.array_equal(s, s2)


def test_error_bound(orc):
    """|dequant - x| <= 2^-4 |x| wherever the scaled value is a normal,
    unsaturated E4M3 value (3 mantissa bits, RNE)."""
    x = W.linear_weight(M=128, N=1024)
    q, s = orc.mxfp8_quantize(x)
    y = orc.mxfp8_dequantize(q, s, out="f32").astype(np.float64)
    xv = refs.bf16_bits_to_f64(x)
    v = np.abs(xv) / np.ldexp(1.0, s.astype(int).repeat(32, 1) - 127)
    m = (v >= 2.0 ** -6) & (v <= 448)
    assert m.mean() > 0.9
    assert np.all(np.abs(y - xv)[m] <= np.ldexp(np.abs(xv[m]), -4))


def test_scale_byte_closed_form(orc):
    x = W.activation(M=64, N=2048)
    _, s = orc.mxfp8_quantize(x)
    a = np.nanmax(np.abs(refs.bf16_bits_to_f64(x)).reshape(64, 64, 32), -1)
    assert np.array_equal(s, refs.e8m0_from_bits(a))


@pytest.mark.parametrize("M", [1, 31, 33, 95])
def test_pad_and_crop_equals_direct(orc, M):
    x = W.planted(seed=7, M=max(M, 8), N=96)[:M]
    q1, s1 = orc.mxfp8_quantize(x)
    q2, s2 = orc.mxfp8_quantize_padded(x)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_padded_adapter_flattens_leading_dims(orc):
    x = W.linear_weight(seed=8, M=6 * 7, N=64).reshape(6, 7, 64)
    q, s = orc.mxfp8_quantize_padded(x)
    assert q.shape == (6, 7, 64) and s.shape == (6, 7, 2)
    q2, s2 = orc.mxfp8_quantize(x.reshape(42, 64))
    assert np.array_equal(q.reshape(42, 64), q2) and np.array_equal(s.reshape(42, 2), s2)


def test_grouped_equals_per_expert_and_flattened(orc):
    xs = W.experts(seed=9, E=5, M=40, N=128)
    qg, sg = orc.mxfp8_quantize_grouped(list(xs))
    qf, sf = orc.mxfp8_quantize(xs.reshape(-1, 128))
    assert np.array_equal(qg, qf) and np.array_equal(sg, sf)
    ragged = [xs[0][:3], xs[1], xs[2][:17]]
    qr, sr = orc.mxfp8_quantize_grouped(ragged)
    for i, part in enumerate(ragged):
        off = sum(p.shape[0] for p in ragged[:i])
        q1, s1 = orc.mxfp8_quantize(part)
        assert np.array_equal(qr[off:off + part.shape[0]], q1)
        assert np.array_equal(sr[off:off + part.shape[0]], s1)


def test_grouped_swizzled_blocks(orc):
    """Per-expert swizzled scales: for experts of 128-row multiples the blocks
    meet without padding, so they equal the torch permute formulation of the
    stacked scales; for ragged experts each block is the permute formulation
    of that expert's scales, padded on its own to 128 rows, in expert order."""
    xs = W.experts(seed=11, E=3, M=256, N=160)
    q, s, z = orc.mxfp8_quantize_grouped(list(xs), swizzled=True)
    assert np.array_equal(z, refs.swizzle_torch(s))
    rows = [5, 0, 130, 128, 1]
    ragged = [W.linear_weight(seed=20 + i, M=max(r, 1), N=96)[:r] for i, r in enumerate(rows)]
    q, s, z = orc.mxfp8_quantize_grouped(ragged, swizzled=True)
    pos = 0
    for i, r in enumerate(rows):
        off = sum(rows[:i])
        block = refs.swizzle_torch(s[off:off + r]) if r else np.zeros(0, np.uint8)
        assert np.array_equal(z[pos:pos + block.size], block), f"expert {i}"
        pos += block.size
    assert pos == z.size == sum((r + 127) // 128 * 128 for r in rows) * 4
    p4, s4, z4 = orc.mxfp4_quantize_grouped(ragged, swizzled=True)
    assert np.array_equal(s4, np.concatenate([orc.mxfp4_quantize(x)[1] for x in ragged]))
    assert z4.size == z.size


def test_strided_equals_contiguous(orc):
    base = W.activation(seed=10, M=48, N=320)
    q1, s1 = orc.mxfp8_quantize(np.ascontiguousarray(base[:, :256]))
    q2, s2 = orc.mxfp8_quantize_strided(base, 48, 256, 320)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_empty(orc):
    q, s = orc.mxfp8_quantize(np.zeros((0, 64), np.uint16))
    assert q.shape == (0, 64) and s.shape == (0, 2)


def test_bad_shapes_rejected(orc):
    with pytest.raises(ValueError):
        orc.mxfp8_quantize(np.zeros((4, 48), np.uint16))


# ----------------------------------------------------------------- swizzle

@pytest.mark.parametrize("M,S", [(128, 4), (256, 224), (130, 7), (1, 1), (300, 33)])
def test_swizzle_matches_permute_formulation(orc, M, S):
    rng = np.random.default_rng(M * 1000 + S)
    s = rng.integers(0, 256, (M, S), dtype=np.uint8)
    out = orc.swizzle_scales(s)
    assert np.array_equal(out, refs.swizzle_torch(s))


def test_swizzle_inverse_recovers_compact(orc):
    rng = np.random.default_rng(15)
    M, S = 300, 33
    s = rng.integers(0, 256, (M, S), dtype=np.uint8)
    out = orc.swizzle_scales(s)
    Sp = (S + 3) // 4 * 4
    r = np.arange(M)[:, None]
    c = np.arange(S)[None, :]
    off = ((r // 128) * (Sp // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    assert np.array_equal(out[off], s)
    mask = np.ones(out.size, bool)
    mask[off.reshape(-1)] = False
    assert np.all(out[mask] == 0)


# -------------------------------------------------------------- columnwise

@pytest.mark.parametrize("M,N", [(64, 96), (37, 32), (1, 16), (100, 48)])
def test_colwise_is_rowwise_of_padded_transpose(orc, M, N):
    """Columnwise groups of the row-padded tensor are the rowwise groups of
    its transpose: compare with the pinned rowwise oracle and with the torch
    formulation on the transposed, zero-padded input, then crop."""
    x = W.planted(seed=M * 3 + N, M=max(M, 8), N=max(N, 32))[:M, :N]
    Mp = (M + 31) // 32 * 32
    padded = np.zeros((Mp, N), np.uint16)
    padded[:M] = x
    xt = np.ascontiguousarray(padded.T)
    q_t, s_t = orc.mxfp8_quantize_colwise(np.ascontiguousarray(x))
    q_r, s_r = orc.mxfp8_quantize(xt)
    q_torch, s_torch = refs.mxfp8_quantize_torch(xt)
    assert np.array_equal(q_t, q_r[:, :M]) and np.array_equal(s_t, s_r)
    assert np.array_equal(q_t, q_torch[:, :M]) and np.array_equal(s_t, s_torch)


def test_colwise_padding_only_touches_last_group(orc):
    """Zero padding never raises an amax: for M a multiple of 32 the result
    does not depend on padding at all, and cropping a taller tensor with the
    same first rows changes only the last group of each column."""
    x = W.activation(seed=91, M=96, N=64)
    q_full, s_full = orc.mxfp8_quantize_colwise(x)
    q_cut, s_cut = orc.mxfp8_quantize_colwise(np.ascontiguousarray(x[:70]))
    assert np.array_equal(q_cut[:, :64], q_full[:, :64])
    assert np.array_equal(s_cut[:, :2], s_full[:, :2])
