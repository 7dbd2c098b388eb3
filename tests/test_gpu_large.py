"""Tensors of more than 2^32 elements (8.6 GB of bf16 input, 4.3 GB of E4M3
codes): every byte offset of the input, and of the MXFP8 codes, passes 2^32,
so the kernels' 64-bit index arithmetic is exercised. Outputs are compared
with the oracle on sampled rows: the first and last 128 (so the last
swizzled-scale block is whole), and 256 seeded random ones."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

M, N = (1 << 20) + 1024, 4096      # 4,299,161,600 elements
PLANT = (777_777, 65)              # one 100.0: the tensor's absolute maximum


def _rows(seed):
    rng = np.random.default_rng(seed)
    rows = set(range(128)) | set(range(M - 128, M)) | {PLANT[0]}
    rows |= set(int(r) for r in rng.integers(0, M, 256))
    return torch.tensor(sorted(rows), dtype=torch.int64)


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def test_mxfp8_beyond_4gib():
    x = W.normal_on_device(M, N, seed=91)
    rows = _rows(1)
    xr = _bits(x[rows.cuda()])
    q, s, z = mxq.mxfp8_quantize(x, swizzled=True)
    y = mxq.mxfp8_dequantize(q, s)
    del x
    qo, so = oracle.mxfp8_quantize(xr)
    idx = rows.cuda()
    assert_same(host(q[idx]), qo, "codes of sampled rows")
    assert_same(host(s[idx]), so, "scales of sampled rows")
    assert_same(host(y[idx]), oracle.mxfp8_dequantize(qo, so, out="bf16"), "dequantized rows")
    last = oracle.swizzle_scales(so[-128:])
    assert_same(host(z[-last.size:]), last, "last 128-row block of swizzled scales")


def test_nvfp4_two_passes_beyond_4gib():
    x = W.normal_on_device(M, N, seed=92)
    x[PLANT] = 100.0
    rows = _rows(2)
    xr = _bits(x[rows.cuda()])
    p, b, g = mxq.nvfp4_quantize(x)
    amax = mxq.nvfp4_amax(x)
    del x
    # the planted row is in the sample, so the sample's amax is the tensor's
    # and the oracle's global scale on the sample is the tensor's
    po, bo, go = oracle.nvfp4_quantize(xr)
    assert float(amax.item()) == 100.0
    assert_same(host(g).reshape(1), np.array([go], np.float32), "global scale")
    idx = rows.cuda()
    assert_same(host(b[idx]), bo, "block scales of sampled rows")
    assert_same(host(p[idx]), po, "packed codes of sampled rows")
