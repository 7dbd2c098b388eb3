"""Pins of the oracle's NVFP4 two-level quantize / dequantize.

* Hand-worked blocks (tests/golden/hand_worked.json) with a given global
  scale of 1 (every operation exact).
* A torch fp32 tensor-op formulation (refs.nvfp4_quantize_torch: torch's
  float8_e4m3fn cast for block scales, nearest-code search for E2M1).
* Invariants: the block that holds the tensor amax gets block scale 448;
  the dequantization error is at most half an E2M1 step times eff (plus
  saturation); a zero tensor gives zero scale and sign-kept zero codes.
"""
import json
import os

import numpy as np
import pytest

import refs
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _codes_of(packed):
    lo = packed & 0x0F
    hi = packed >> 4
    return np.stack([lo, hi], -1).reshape(packed.shape[0], -1)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["nvfp4"], ids=lambda c: c["name"])
def test_hand_worked_block(orc, case):
    vals = [case["fill"]] * 16
    for k, v in case["x"].items():
        vals[int(k)] = v
    x = W.bits_of([float(v) for v in vals])[None, :]
    packed, bs, g = orc.nvfp4_quantize(x, global_scale=float(case["g"]))
    assert int(bs[0, 0]) == case["block_scale"], case["why"]
    want = [case["codes"]["fill"]] * 16
    for k, v in case["codes"].items():
        if k != "fill":
            want[int(k)] = v
    assert _codes_of(packed)[0].tolist() == want, case["why"]
    assert packed[0].tolist() == case["packed"], case["why"]


def test_workload_recipe_matches_torch(orc):
    x = W.nvfp4_tensor(M=256, N=1024)
    p, b, g = orc.nvfp4_quantize(x)
    pt, bt, gt = refs.nvfp4_quantize_torch(x)
    assert np.float32(g).view(np.uint32) == np.float32(gt).view(np.uint32)
    assert np.array_equal(b, bt)
    assert np.array_equal(p, pt)


def test_given_global_scale_matches_torch(orc):
    x = W.activation(seed=21, M=64, N=512)
    for g in (0.01, 0.37, 3.0e-5):
        p, b, g2 = orc.nvfp4_quantize(x, global_scale=g)
        pt, bt, _ = refs.nvfp4_quantize_torch(x, g=g)
        assert g2 == np.float32(g)
        assert np.array_equal(b, bt) and np.array_equal(p, pt)


def test_given_equals_computed(orc):
    x = W.nvfp4_tensor(seed=22, M=64, N=256)
    p1, b1, g1 = orc.nvfp4_quantize(x)
    p2, b2, _ = orc.nvfp4_quantize(x, global_scale=g1)
    assert np.array_equal(p1, p2) and np.array_equal(b1, b2)
    assert g1 == orc.nvfp4_global_amax(x) / np.float32(2688.0)


def test_amax_block_gets_top_scale(orc):
    x = W.nvfp4_tensor(seed=23, M=128, N=512)
    p, b, g = orc.nvfp4_quantize(x)
    a = np.abs(refs.bf16_bits_to_f64(x)).reshape(128, 32, 16).max(-1)
    assert np.all(b[a == a.max()] == 0x7E)


def test_dequant_error_bound(orc):
    x = W.nvfp4_tensor(seed=24, M=64, N=512)
    p, b, g = orc.nvfp4_quantize(x)
    y = orc.nvfp4_dequantize(p, b, g, out="f32").astype(np.float64)
    xv = refs.bf16_bits_to_f64(x)
    eff = (refs.e4m3_table()[b].astype(np.float32) * np.float32(g)).astype(np.float64).repeat(16, 1)
    # E2M1 steps are at most 2 (between 4 and 6): error <= eff, plus the
    # saturation of |x|/eff in (6, 6.x] (block scale rounded down)
    over = np.maximum(np.abs(xv) - 6 * eff, 0)
    assert np.all(np.abs(y - xv) <= eff * (1 + 1e-6) + over)


def test_dequant_matches_definition(orc):
    x = W.nvfp4_tensor(seed=25, M=32, N=256)
    p, b, g = orc.nvfp4_quantize(x)
    codes = _codes_of(p).astype(np.int64)
    mags = refs.E2M1_MAGNITUDES[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    eff = refs.e4m3_table()[b].astype(np.float32) * np.float32(g)
    want = (mags.astype(np.float32) * eff.repeat(16, 1)).astype(np.float32)
    got = orc.nvfp4_dequantize(p, b, g, out="f32")
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    gotb = orc.nvfp4_dequantize(p, b, g, out="bf16")
    assert np.array_equal(gotb, refs.f64_to_bf16_bits_torch(want.astype(np.float64)))


def test_zero_tensor(orc):
    x = np.zeros((4, 32), np.uint16)
    x[1, 3] = 0x8000
    p, b, g = orc.nvfp4_quantize(x)
    assert g == 0.0 and np.all(b == 0)
    codes = _codes_of(p)
    assert codes[1, 3] == 8 and codes.sum() == 8


def test_fp32_input_matches_bf16(orc):
    x = W.nvfp4_tensor(seed=26, M=16, N=128)
    p1, b1, g1 = orc.nvfp4_quantize(x)
    p2, b2, g2 = orc.nvfp4_quantize(refs.bf16_bits_to_f64(x).astype(np.float32))
    assert g1 == g2 and np.array_equal(p1, p2) and np.array_equal(b1, b2)


def test_bad_shape(orc):
    with pytest.raises(ValueError):
        orc.nvfp4_quantize(np.zeros((2, 24), np.uint16))
