"""MXFP8 columnwise quantize on the GPU against the CPU oracle, bit-exact:
transposed codes and scales (with the zero-padded last group of every column
when M % 32 != 0), and the fused mode whose rowwise outputs must equal the
rowwise oracle."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu


def check(x, fused=False, what=""):
    out = mxq.mxfp8_quantize_columnwise(dev(x), rowwise=fused)
    qo_t, so_t = oracle.mxfp8_quantize_colwise(x)
    q_t, s_t = out[-2], out[-1]
    assert_same(host(q_t), qo_t, f"{what} q_t")
    assert_same(host(s_t), so_t, f"{what} scale_t")
    if fused:
        qo, so = oracle.mxfp8_quantize(x)
        assert_same(host(out[0]), qo, f"{what} rowwise q")
        assert_same(host(out[1]), so, f"{what} rowwise scale")


@pytest.mark.slow
def test_activation_full_size_fused():
    check(W.activation(), fused=True, what="activation 16384x7168")


@pytest.mark.parametrize("M", [1, 31, 33, 100, 128, 4095])
@pytest.mark.parametrize("N", [32, 96, 160, 7168])
def test_ragged_shapes(M, N):
    x = W.activation(seed=M * 13 + N, M=M, N=N)
    check(x, fused=True, what=f"{M}x{N}")


def test_n_multiple_of_16_columnwise_only():
    x = W.linear_weight(seed=92, M=77, N=48)
    check(x, fused=False, what="77x48")
    with pytest.raises(mxq.MxqError):
        mxq.mxfp8_quantize_columnwise(dev(x), rowwise=True)     # rowwise needs N % 32


def test_special_values_and_every_bf16_pattern():
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(512, 128)
    check(x, fused=True, what="all bf16 patterns")
    check(np.ascontiguousarray(x.T[:, :96]), fused=True, what="all bf16 patterns transposed")
    check(W.planted(), fused=True, what="planted")


def test_fp32_and_strided():
    rng = np.random.default_rng(93)
    xf = (rng.standard_t(3, (300, 192)) * 0.5).astype(np.float32)
    xf[5, 7] = np.nan
    xf[9, 3] = np.inf
    check(xf, fused=True, what="fp32")
    base = W.activation(seed=94, M=200, N=512)
    out = mxq.mxfp8_quantize_columnwise(dev(base)[:, 128:128 + 256], rowwise=True)
    sub = np.ascontiguousarray(base[:, 128:384])
    qo_t, so_t = oracle.mxfp8_quantize_colwise(sub)
    qo, so = oracle.mxfp8_quantize(sub)
    assert_same(host(out[2]), qo_t, "strided q_t")
    assert_same(host(out[3]), so_t, "strided scale_t")
    assert_same(host(out[0]), qo, "strided q")
    assert_same(host(out[1]), so, "strided scale")


def test_columnwise_dequantizes_to_the_transpose():
    x = W.linear_weight(seed=95, M=256, N=512)
    q_t, s_t = mxq.mxfp8_quantize_columnwise(dev(x))
    y_t = mxq.mxfp8_dequantize(q_t, s_t, torch.float32)
    q2, s2 = mxq.mxfp8_quantize(y_t)
    assert torch.equal(q2, q_t) and torch.equal(s2, s_t)
