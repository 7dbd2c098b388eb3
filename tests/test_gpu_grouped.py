"""Grouped MXFP8 quantize (one launch over a stack or list of expert tensors)
on the GPU: bit-exact against the oracle's per-expert quantize and against the
single-tensor entry point on the flattened stack."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.slow
def test_expert_stack_full_size():
    xs = W.experts()                                  # [64, 2048, 7168] bf16
    xd = dev(xs)
    q, s = mxq.mxfp8_quantize_grouped(xd)
    assert q.shape == (64, 2048, 7168) and s.shape == (64, 2048, 224)
    qf, sf = mxq.mxfp8_quantize(xd.view(-1, 7168))
    assert torch.equal(q.view(-1, 7168), qf) and torch.equal(s.view(-1, 224), sf)
    for e in (0, 17, 63):
        qo, so = oracle.mxfp8_quantize(xs[e])
        assert_same(host(q[e]), qo, f"expert {e} qweight")
        assert_same(host(s[e]), so, f"expert {e} scale")


def test_ragged_list_with_empty_experts():
    rng = np.random.default_rng(51)
    rows = [3, 0, 257, 1, 0, 64, 1000]
    xs = [W.linear_weight(seed=100 + i, M=max(r, 1), N=192)[:r] for i, r in enumerate(rows)]
    q, s = mxq.mxfp8_quantize_grouped([dev(x) for x in xs])
    qo, so = oracle.mxfp8_quantize_grouped(xs)
    assert_same(host(q), qo, "ragged qweight")
    assert_same(host(s), so, "ragged scale")
    del rng


def test_many_experts_and_fp32():
    xs = [(np.random.default_rng(200 + e).standard_normal((e % 7 + 1, 64)) * (e + 1)).astype(np.float32)
          for e in range(100)]
    q, s = mxq.mxfp8_quantize_grouped([dev(x) for x in xs])
    qo, so = oracle.mxfp8_quantize_grouped(xs)
    assert_same(host(q), qo, "100 experts qweight")
    assert_same(host(s), so, "100 experts scale")


def test_single_expert_matches_plain_call():
    x = W.planted()
    qg, sg = mxq.mxfp8_quantize_grouped([dev(x)])
    qo, so = oracle.mxfp8_quantize(x)
    assert_same(host(qg), qo, "E=1 qweight")
    assert_same(host(sg), so, "E=1 scale")


def test_too_many_experts_rejected():
    x = torch.zeros(1, 32, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mxq.MxqError):
        mxq.mxfp8_quantize_grouped([x] * 1025)
