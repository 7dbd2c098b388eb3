"""Pins of the oracle's MXFP4 quantize / dequantize and fake quantization.

* Hand-worked groups (tests/golden/hand_worked.json, "mxfp4").
* The E8M0 rule with emax 2 against the fp32 exponent-field formula.
* A formulation with numpy/torch: exponent-field byte, nearest-code search
  over the E2M1 values, packing by array slicing, dequant by torch.ldexp.
* Fake quantization equals dequantize(quantize(x)) and is idempotent.
"""
import json
import os

import numpy as np
import pytest
import torch

import refs
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _bits(vals):
    out = []
    for s in vals:
        out.append(int(s, 16) if isinstance(s, str) and s.startswith("0x") else int(W.bits_of([float(s)])[0]))
    return np.array(out, np.uint16)


def _codes(packed):
    return np.stack([packed & 0xF, packed >> 4], -1).reshape(packed.shape[0], -1)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["mxfp4"], ids=lambda c: c["name"])
def test_hand_worked_group(orc, case):
    vals = [case["fill"]] * 32
    for k, v in case["x"].items():
        vals[int(k)] = v
    x = _bits(vals)[None, :]
    p, s = orc.mxfp4_quantize(x)
    assert int(s[0, 0]) == case["scale"], case["why"]
    want = [case["codes"]["fill"]] * 32
    for k, v in case["codes"].items():
        if k != "fill":
            want[int(k)] = v
    assert _codes(p)[0].tolist() == want, case["why"]
    y = orc.mxfp4_dequantize(p, s, out="f32")[0].astype(np.float64)
    wd = [float(case["dq_f32"]["fill"])] * 32
    for k, v in case["dq_f32"].items():
        if k != "fill":
            wd[int(k)] = float(v)
    assert np.array_equal(y, np.array(wd)) and np.array_equal(np.signbit(y), np.signbit(np.array(wd)))


def test_e8m0_emax2_matches_exponent_field(orc):
    rng = np.random.default_rng(101)
    a = np.concatenate([rng.integers(0, 0x7F800001, 200000, dtype=np.int64).astype(np.uint32).view(np.float32),
                        np.float32([0, np.inf, 1, 6, 7.99, 8, 2 ** -130])])
    for v in a[:2000].tolist() + a[-7:].tolist():
        E = (np.float32(v).view(np.uint32) >> 23) & 0xFF
        want = 127 if v == 0 else 254 if np.isinf(v) else min(max(int(E) - 2, 0), 254)
        assert orc.e8m0_from_amax_emax(v, 2) == want, v
    assert orc.e8m0_from_amax_emax(448.0, 8) == orc.e8m0_from_amax(448.0)


def mxfp4_reference(xbits):
    M, N = xbits.shape
    x = refs.bf16_bits_to_f64(xbits).reshape(M, N // 32, 32)
    a = np.where(np.isnan(x), 0, np.abs(x)).max(-1).astype(np.float32)
    E = (a.view(np.uint32) >> 23).astype(np.int64) & 0xFF
    b = np.clip(E - 2, 0, 254)
    b = np.where(a == 0, 127, np.where(np.isinf(a), 254, b)).astype(np.int64)
    codes = refs.e2m1_brute(np.ldexp(x, (127 - b)[..., None])).reshape(M, N)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, b.astype(np.uint8)


@pytest.mark.parametrize("make", [lambda: W.planted(), lambda: W.activation(M=96, N=2048),
                                  lambda: np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(64, 1024)])
def test_matches_reference_formulation(orc, make):
    x = make()
    p, s = orc.mxfp4_quantize(x)
    pr, sr = mxfp4_reference(x)
    assert np.array_equal(s, sr) and np.array_equal(p, pr)
    codes = _codes(p).astype(np.int64)
    vals = refs.E2M1_MAGNITUDES[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    d = torch.ldexp(torch.from_numpy(vals), torch.from_numpy(s.astype(np.float64).repeat(32, 1) - 127))
    assert np.array_equal(orc.mxfp4_dequantize(p, s, out="f32").view(np.uint32),
                          d.to(torch.float32).numpy().view(np.uint32))


def test_fake_quant_is_round_trip_and_idempotent(orc):
    x = W.activation(seed=102, M=64, N=512)
    for fmt in ("mxfp8", "mxfp4"):
        y = orc.fake_quantize(x, fmt, out="f32")
        if fmt == "mxfp8":
            q, s = orc.mxfp8_quantize(x)
            assert np.array_equal(y.view(np.uint32), orc.mxfp8_dequantize(q, s, out="f32").view(np.uint32))
        y2 = orc.fake_quantize(y, fmt, out="f32")
        assert np.array_equal(y2.view(np.uint32), y.view(np.uint32))
