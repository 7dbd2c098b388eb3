"""Seeded random shapes through every operation, each compared with the
oracle byte for byte: ragged M, N from one group up to tens of groups, row
strides wider than N (views of a larger buffer), bf16 and fp32 inputs, bf16
and fp32 outputs, and random bit patterns (NaN, infinities, subnormals) mixed
into normal data. Every output of the binding lies between guard bands."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu

CASES = 24


def _input(rng, M, N, fp32):
    """[M, N] values (normal data with about 1 % random bit patterns) and a
    device view of them with a row stride wider than N."""
    if fp32:
        x = (rng.standard_t(3, (M, N)) * rng.uniform(0.01, 10)).astype(np.float32)
        bits = rng.integers(0, 2**32, (M, N), dtype=np.uint64).astype(np.uint32).view(np.float32)
        pad = 4 * int(rng.integers(0, 3))
    else:
        x = torch.from_numpy((rng.standard_t(3, (M, N)) * rng.uniform(0.01, 10)).astype(np.float32))
        x = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        bits = rng.integers(0, 65536, (M, N)).astype(np.uint16)
        pad = 8 * int(rng.integers(0, 3))
    mask = rng.random((M, N)) < 0.01
    x = np.where(mask, bits, x)
    buf = np.zeros((M, N + pad), x.dtype)
    buf[:, :N] = x
    xd = dev(buf)[:, :N]
    return x, xd


def _shapes(seed, group):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(CASES):
        M = int(rng.choice([1, 2, 31, 33, 127, 128, 129, int(rng.integers(1, 700))]))
        N = group * int(rng.integers(1, 40))
        out.append((M, N, bool(rng.random() < 0.3), int(rng.integers(0, 2**31))))
    return out


@pytest.mark.parametrize("M,N,fp32,seed", _shapes(1, 32))
def test_mxfp8_and_mxfp4(M, N, fp32, seed):
    rng = np.random.default_rng(seed)
    x, xd = _input(rng, M, N, fp32)
    q, s, z = mxq.mxfp8_quantize(xd, swizzled=True)
    qo, so = oracle.mxfp8_quantize(x)
    assert_same(host(q), qo, "mxfp8 codes")
    assert_same(host(s), so, "mxfp8 scales")
    assert_same(host(z), oracle.swizzle_scales(so), "mxfp8 swizzled scales")
    out = "f32" if rng.random() < 0.5 else "bf16"
    y = mxq.mxfp8_dequantize(q, s, torch.float32 if out == "f32" else torch.bfloat16)
    assert_same(host(y), oracle.mxfp8_dequantize(qo, so, out=out), "mxfp8 dequant")
    p4, s4, z4 = mxq.mxfp4_quantize(xd, swizzled=True)
    po, s4o = oracle.mxfp4_quantize(x)
    assert_same(host(p4), po, "mxfp4 codes")
    assert_same(host(s4), s4o, "mxfp4 scales")
    assert_same(host(z4), oracle.swizzle_scales(s4o), "mxfp4 swizzled scales")
    y4 = mxq.mxfp4_dequantize(p4, s4, torch.float32 if out == "f32" else torch.bfloat16)
    assert_same(host(y4), oracle.mxfp4_dequantize(po, s4o, out=out), "mxfp4 dequant")
    for fmt in ("mxfp8", "mxfp4"):
        yf = mxq.mx_fake_quantize(xd, fmt, torch.float32 if out == "f32" else torch.bfloat16)
        assert_same(host(yf), oracle.fake_quantize(x, fmt, out=out), f"{fmt} fake-quantize")


@pytest.mark.parametrize("M,N,fp32,seed", _shapes(2, 16))
def test_nvfp4_and_columnwise(M, N, fp32, seed):
    rng = np.random.default_rng(seed)
    x, xd = _input(rng, M, N, fp32)
    finite = np.isfinite(x.astype(np.float32) if fp32 else
                         (x.astype(np.uint32) << 16).view(np.float32)).all()
    if finite:  # NVFP4 inputs with NaN or infinities are outside the method's contract
        p, b, g = mxq.nvfp4_quantize(xd)
        po, bo, go = oracle.nvfp4_quantize(x)
        assert_same(host(g).reshape(1), np.array([go], np.float32), "nvfp4 global scale")
        assert_same(host(b), bo, "nvfp4 block scales")
        assert_same(host(p), po, "nvfp4 codes")
        y = mxq.nvfp4_dequantize(p, b, g, torch.float32)
        assert_same(host(y), oracle.nvfp4_dequantize(po, bo, go, out="f32"), "nvfp4 dequant")
    qt, st = mxq.mxfp8_quantize_columnwise(xd)
    qto, sto = oracle.mxfp8_quantize_colwise(x)
    assert_same(host(qt), qto, "columnwise codes")
    assert_same(host(st), sto, "columnwise scales")
    if N % 32 == 0:
        q, s, qt2, st2 = mxq.mxfp8_quantize_columnwise(xd, rowwise=True)
        qo, so = oracle.mxfp8_quantize(x)
        assert_same(host(q), qo, "fused rowwise codes")
        assert_same(host(s), so, "fused rowwise scales")
        assert_same(host(qt2), qto, "fused columnwise codes")
        assert_same(host(st2), sto, "fused columnwise scales")


@pytest.mark.parametrize("seed", range(8))
def test_grouped_random_offsets(seed):
    rng = np.random.default_rng(100 + seed)
    E = int(rng.integers(1, 40))
    rows = [int(r) for r in rng.choice([0, 1, 5, 64, 127, 128, 129, 300], E)]
    N = 32 * int(rng.integers(1, 12))
    fp32 = bool(rng.random() < 0.3)
    if sum(rows) == 0:
        rows[0] = 3
    x, _ = _input(rng, sum(rows), N, fp32)
    parts = [x[a:b] for a, b in zip(np.cumsum([0] + rows[:-1]), np.cumsum(rows))]
    offs = torch.tensor(np.concatenate([[0], np.cumsum(rows)]), dtype=torch.int64).cuda()
    q, s, z = mxq.mxfp8_quantize_grouped(dev(x), row_offsets=offs, swizzled=True)
    qo, so, zo = oracle.mxfp8_quantize_grouped(parts, swizzled=True)
    assert_same(host(q), qo, "grouped codes")
    assert_same(host(s), so, "grouped scales")
    assert_same(host(z)[:zo.size], zo, "grouped per-expert swizzled scales")
