"""MXFP4 quantize / dequantize / grouped and the fused fake-quantize (MXFP8
and MXFP4) on the GPU against the CPU oracle, bit-exact: identical packed
codes, scale and swizzled-scale bytes, identical bf16 / fp32 output bits.
Inputs follow the workload recipes, plus exhaustive sweeps (every bf16
pattern under every group exponent, every packed byte under every scale
byte) and edge shapes."""
import json
import os

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
OUTS = ((torch.bfloat16, "bf16"), (torch.float32, "f32"))


def check_mxfp4(x: np.ndarray, swizzled=False, dequant=True, what=""):
    got = mxq.mxfp4_quantize(dev(x), swizzled=swizzled)
    N = x.shape[-1]
    po, so = oracle.mxfp4_quantize(x.reshape(-1, N))
    assert_same(host(got[0]).reshape(po.shape), po, f"{what} packed")
    assert_same(host(got[1]).reshape(so.shape), so, f"{what} scale")
    if swizzled:
        assert_same(host(got[2]), oracle.swizzle_scales(so), f"{what} swizzled scale")
    if dequant:
        for dt, name in OUTS:
            y = mxq.mxfp4_dequantize(got[0], got[1], dt)
            assert_same(host(y).reshape(-1, N), oracle.mxfp4_dequantize(po, so, out=name),
                        f"{what} dequant {name}")
    return got


def check_fake(x: np.ndarray, what="", fmts=("mxfp8", "mxfp4")):
    xd = dev(x)
    N = x.shape[-1]
    for fmt in fmts:
        for dt, name in OUTS:
            y = mxq.mx_fake_quantize(xd, fmt, dt)
            want = oracle.fake_quantize(x.reshape(-1, N), fmt, out=name)
            assert_same(host(y).reshape(-1, N), want, f"{what} fake {fmt} -> {name}")


# ------------------------------------------------------------------ MXFP4

@pytest.mark.parametrize("case", json.load(open(GOLDEN))["mxfp4"], ids=lambda c: c["name"])
def test_hand_worked_groups(case):
    vals = [case["fill"]] * 32
    for k, v in case["x"].items():
        vals[int(k)] = v
    bits = [int(s, 16) if isinstance(s, str) and s.startswith("0x") else int(W.bits_of([float(s)])[0])
            for s in vals]
    x = np.array([bits], np.uint16)
    p, s = mxq.mxfp4_quantize(dev(x))
    assert int(host(s)[0, 0]) == case["scale"], case["why"]
    codes = host(p)[0]
    got = np.stack([codes & 0xF, codes >> 4], -1).reshape(-1).tolist()
    want = [case["codes"]["fill"]] * 32
    for k, v in case["codes"].items():
        if k != "fill":
            want[int(k)] = v
    assert got == want, case["why"]


def test_planted_groups():
    check_mxfp4(W.planted(), swizzled=True, what="planted")


def test_linear_weight_full_size():
    check_mxfp4(W.linear_weight(), swizzled=True, what="linear weight 4096x4096")


@pytest.mark.slow
def test_activation_full_size():
    check_mxfp4(W.activation(), swizzled=True, what="activation 16384x7168")


def test_every_bf16_value_under_every_exponent():
    check_mxfp4(W.mx_every_value_every_exponent(), what="exhaustive")


def test_every_packed_byte_under_every_scale_dequant():
    q, s = W.mx_all_packed_scale_pairs()
    for dt, name in OUTS:
        y = mxq.mxfp4_dequantize(dev(q), dev(s), dt)
        assert_same(host(y), oracle.mxfp4_dequantize(q, s, out=name), f"dequant pairs {name}")


def test_random_bit_patterns():
    rng = np.random.default_rng(61)
    x = rng.integers(0, 65536, (512, 2048), dtype=np.uint32).astype(np.uint16)
    check_mxfp4(x, swizzled=True, what="random bf16 bits")


def fp32_specials(seed, M=300, N=1024):
    rng = np.random.default_rng(seed)
    xf = (rng.standard_t(3, (M, N)) * 0.5).astype(np.float32)
    xf[0, :32] = 0
    xf[1, 3] = np.nan
    xf[2, 4] = -np.inf
    xf[3, :32] = np.ldexp(rng.uniform(-1, 1, 32), -135).astype(np.float32)
    xf[4, 0] = np.float32(3.4e38)
    xf[5, :] = rng.integers(0, 2**32, N, dtype=np.uint64).astype(np.uint32).view(np.float32)
    xf[6, :32] = np.float32([6.0, 5.0, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25] * 4)  # E2M1 ties
    return xf


def test_fp32_input():
    check_mxfp4(fp32_specials(62), swizzled=True, what="fp32")


@pytest.mark.parametrize("M", [1, 31, 33, 4095])
@pytest.mark.parametrize("N", [32, 96, 7168])
def test_ragged_shapes(M, N):
    check_mxfp4(W.activation(seed=M * 5 + N, M=M, N=N), swizzled=True, what=f"{M}x{N}")


def test_leading_dims_and_row_stride():
    x = W.activation(seed=63, M=6 * 35, N=256).reshape(6, 35, 256)
    p, s = mxq.mxfp4_quantize(dev(x))
    assert p.shape == (6, 35, 128) and s.shape == (6, 35, 8)
    po, so = oracle.mxfp4_quantize(x.reshape(-1, 256))
    assert_same(host(p).reshape(-1, 128), po, "3-D packed")
    assert_same(host(s).reshape(-1, 8), so, "3-D scale")
    base = W.activation(seed=64, M=300, N=1024)
    p, s, z = mxq.mxfp4_quantize(dev(base)[:, 64:64 + 640], swizzled=True)
    po, so = oracle.mxfp4_quantize(np.ascontiguousarray(base[:, 64:64 + 640]))
    assert_same(host(p), po, "strided packed")
    assert_same(host(s), so, "strided scale")
    assert_same(host(z), oracle.swizzle_scales(so), "strided swizzle")


def test_grouped_ragged_and_stacked():
    rows = [3, 0, 257, 1, 0, 64, 1000]
    xs = [W.linear_weight(seed=300 + i, M=max(r, 1), N=192)[:r] for i, r in enumerate(rows)]
    p, s = mxq.mxfp4_quantize_grouped([dev(x) for x in xs])
    parts = [oracle.mxfp4_quantize(x) for x in xs if x.shape[0]]
    assert_same(host(p), np.concatenate([a for a, _ in parts]), "ragged packed")
    assert_same(host(s), np.concatenate([b for _, b in parts]), "ragged scale")
    st = W.experts(seed=65, E=8, M=96, N=512)
    p, s = mxq.mxfp4_quantize_grouped(dev(st))
    assert p.shape == (8, 96, 256) and s.shape == (8, 96, 16)
    pf, sf = mxq.mxfp4_quantize(dev(st).view(-1, 512))
    assert torch.equal(p.view(-1, 256), pf) and torch.equal(s.view(-1, 16), sf)
    po, so = oracle.mxfp4_quantize(st.reshape(-1, 512))
    assert_same(host(pf), po, "stacked packed")
    assert_same(host(sf), so, "stacked scale")


def test_grouped_many_fp32_experts():
    xs = [(np.random.default_rng(400 + e).standard_normal((e % 5 + 1, 64)) * (e + 1)).astype(np.float32)
          for e in range(100)]
    p, s = mxq.mxfp4_quantize_grouped([dev(x) for x in xs])
    parts = [oracle.mxfp4_quantize(x) for x in xs]
    assert_same(host(p), np.concatenate([a for a, _ in parts]), "100 experts packed")
    assert_same(host(s), np.concatenate([b for _, b in parts]), "100 experts scale")


def test_requantize_is_identity():
    x = dev(W.activation(seed=66, M=256, N=2048))
    p, s = mxq.mxfp4_quantize(x)
    p2, s2 = mxq.mxfp4_quantize(mxq.mxfp4_dequantize(p, s, torch.float32))
    assert torch.equal(p, p2) and torch.equal(s, s2)


def test_empty_and_errors():
    p, s = mxq.mxfp4_quantize(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"))
    assert p.shape == (0, 32) and s.shape == (0, 2)
    with pytest.raises(mxq.MxqError):
        mxq.mxfp4_quantize(torch.zeros(4, 48, dtype=torch.bfloat16, device="cuda"))


# ----------------------------------------------------------- fake quantize

def test_fake_planted_and_exhaustive():
    check_fake(W.planted(), "planted")
    check_fake(W.mx_every_value_every_exponent(), "exhaustive")


def test_fake_fp32_and_random_bits():
    check_fake(fp32_specials(67), "fp32")
    rng = np.random.default_rng(68)
    check_fake(rng.integers(0, 65536, (256, 2048), dtype=np.uint32).astype(np.uint16), "random bits")


@pytest.mark.parametrize("M", [1, 33, 4095])
@pytest.mark.parametrize("N", [32, 7168])
def test_fake_ragged(M, N):
    check_fake(W.activation(seed=M * 11 + N, M=M, N=N), f"{M}x{N}")


def test_fake_equals_quantize_then_dequantize_on_device():
    for x in (dev(W.activation(seed=69, M=1024, N=7168)), dev(fp32_specials(70, M=512, N=2048))):
        for dt, _ in OUTS:
            q, s = mxq.mxfp8_quantize(x)
            assert torch.equal(mxq.mx_fake_quantize(x, "mxfp8", dt).view(torch.uint8),
                               mxq.mxfp8_dequantize(q, s, dt).view(torch.uint8))
            p, s = mxq.mxfp4_quantize(x)
            assert torch.equal(mxq.mx_fake_quantize(x, "mxfp4", dt).view(torch.uint8),
                               mxq.mxfp4_dequantize(p, s, dt).view(torch.uint8))


def test_fake_strided_and_leading_dims():
    base = W.activation(seed=71, M=300, N=1024)
    view = dev(base)[:, 32:32 + 736]
    for fmt in ("mxfp8", "mxfp4"):
        y = mxq.mx_fake_quantize(view, fmt)
        assert y.is_contiguous() and y.shape == (300, 736)
        want = oracle.fake_quantize(np.ascontiguousarray(base[:, 32:32 + 736]), fmt, out="bf16")
        assert_same(host(y), want, f"strided fake {fmt}")
    x = W.planted(seed=72, M=4 * 24, N=128).reshape(4, 24, 128)
    y = mxq.mx_fake_quantize(dev(x), "mxfp4", torch.float32)
    assert y.shape == (4, 24, 128)
    assert_same(host(y).reshape(-1, 128), oracle.fake_quantize(x.reshape(-1, 128), "mxfp4", out="f32"),
                "3-D fake")


def test_fake_is_idempotent():
    x = dev(W.activation(seed=73, M=128, N=4096))
    for fmt in ("mxfp8", "mxfp4"):
        y = mxq.mx_fake_quantize(x, fmt, torch.float32)
        assert torch.equal(mxq.mx_fake_quantize(y, fmt, torch.float32), y)


def test_fake_empty_and_errors():
    y = mxq.mx_fake_quantize(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"), "mxfp4")
    assert y.shape == (0, 64)
    with pytest.raises(ValueError):
        mxq.mx_fake_quantize(torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda"), "nvfp4")
    with pytest.raises(mxq.MxqError):
        mxq.mx_fake_quantize(torch.zeros(4, 40, dtype=torch.bfloat16, device="cuda"), "mxfp8")
