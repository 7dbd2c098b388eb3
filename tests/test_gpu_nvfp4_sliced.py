"""NVFP4 with one global scale per slice of rows (per expert, per gate/up
half) on the GPU against the CPU oracle, bit-exact: packed codes, block
scales and the fp32 global scales. Slicings cover empty slices, ragged sizes,
more than 64 slices (the large slice table), strided input, given scales and
given amaxes, and the full-size expert stack on sampled experts."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu


def check(x: np.ndarray, rows, what=""):
    N = x.shape[-1]
    p, b, g = mxq.nvfp4_quantize_sliced(dev(x), rows)
    po, bo, go = oracle.nvfp4_quantize_sliced(x.reshape(-1, N), rows)
    assert_same(host(g), go, f"{what} global scales")
    assert_same(host(b).reshape(bo.shape), bo, f"{what} block scales")
    assert_same(host(p).reshape(po.shape), po, f"{what} packed")
    return p, b, g


def test_per_expert_and_per_half():
    w = W.experts(seed=91, E=8, M=96, N=512)
    check(w, [96] * 8, "per expert")
    check(w, [48] * 16, "per half")
    p, b, g = mxq.nvfp4_quantize_experts(dev(w), per_half=True)
    assert p.shape == (8, 96, 256) and b.shape == (8, 96, 32) and g.shape == (8, 2)
    _, _, go = oracle.nvfp4_quantize_sliced(w.reshape(-1, 512), [48] * 16)
    assert_same(host(g).reshape(-1), go, "experts helper scales")


def test_ragged_slices_with_empty_ones():
    rows = [3, 0, 257, 1, 0, 64, 1000, 0]
    x = W.nvfp4_tensor(seed=92, M=sum(rows), N=192)
    _, _, g = check(x, rows, "ragged")
    assert host(g)[1] == 0 and host(g)[4] == 0 and host(g)[7] == 0


def test_many_slices_fp32():
    rng = np.random.default_rng(93)
    rows = [int(r) for r in rng.integers(0, 9, 300)]
    xf = (rng.standard_normal((sum(rows), 64)) * np.repeat(rng.uniform(0.01, 10, len(rows)), rows)[:, None]
          ).astype(np.float32)
    check(xf, rows, "300 slices fp32")


def test_one_slice_equals_single_tensor():
    x = dev(W.nvfp4_tensor(seed=94, M=300, N=1024))
    p, b, g = mxq.nvfp4_quantize_sliced(x, [300])
    p1, b1, g1 = mxq.nvfp4_quantize(x)
    assert torch.equal(p, p1) and torch.equal(b, b1) and torch.equal(g.view(()), g1)


def test_given_scales_and_given_amax():
    w = W.experts(seed=95, E=6, M=40, N=256)
    rows = [40] * 6
    x = dev(w)
    p, b, g = mxq.nvfp4_quantize_sliced(x, rows)
    amax = mxq.nvfp4_amax_sliced(x, rows)
    ao = [oracle.nvfp4_global_amax(w[e]) for e in range(6)]
    assert_same(host(amax), np.array(ao, np.float32), "slice amax")
    p2, b2, g2 = mxq.nvfp4_quantize_sliced(x, rows, amax=amax)
    assert torch.equal(p, p2) and torch.equal(b, b2) and torch.equal(g, g2)
    gs = torch.tensor([0.001, 0.01, 0.1, 1e-5, 3.0, 0.02], dtype=torch.float32)
    p3, b3, g3 = mxq.nvfp4_quantize_sliced(x, rows, global_scales=gs)
    po, bo, _ = oracle.nvfp4_quantize_sliced(w.reshape(-1, 256), rows, global_scales=gs.numpy())
    assert_same(host(p3), po.reshape(6, 40, 128), "given packed")
    assert_same(host(b3), bo.reshape(6, 40, 16), "given block scales")


def test_strided_input():
    base = W.nvfp4_tensor(seed=96, M=200, N=768)
    view = dev(base)[:, 128:128 + 512]
    rows = [50, 0, 150]
    p, b, g = mxq.nvfp4_quantize_sliced(view, rows)
    po, bo, go = oracle.nvfp4_quantize_sliced(np.ascontiguousarray(base[:, 128:640]), rows)
    assert_same(host(g), go, "strided scales")
    assert_same(host(p), po, "strided packed")
    assert_same(host(b), bo, "strided block scales")


def test_errors():
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        mxq.nvfp4_quantize_sliced(x, [4, 5])
    with pytest.raises(mxq.MxqError):
        mxq.nvfp4_quantize_sliced(x, [1] * 8 + [0] * 1020)


@pytest.mark.slow
def test_expert_stack_full_size_sampled():
    """64 experts [2048, 7168], per expert and per gate/up half, in the launch
    configuration the benchmark times; the oracle checks sampled slices (each
    slice is quantized independently of the others)."""
    w = W.experts()
    x = dev(w)
    for per_half in (False, True):
        p, b, g = mxq.nvfp4_quantize_experts(x, per_half=per_half)
        g = host(g).reshape(64, -1)
        for e in (0, 31, 63):
            halves = ((0, 1024), (1024, 2048)) if per_half else ((0, 2048),)
            for h, (r0, r1) in enumerate(halves):
                po, bo, go = oracle.nvfp4_quantize(w[e, r0:r1])
                assert g[e, h] == go.view(np.uint32), (e, h)
                assert_same(host(p[e, r0:r1]), po, f"expert {e} half {h} packed")
                assert_same(host(b[e, r0:r1]), bo, f"expert {e} half {h} block scales")
