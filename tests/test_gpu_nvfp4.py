"""NVFP4 two-level quantize / dequantize on the GPU against the CPU oracle,
bit-exact: identical global scale bits, block-scale bytes, packed nibbles and
dequantized bits. Full-size workload, sweeps of the E2M1 and E4M3 roundings,
the given-scale and given-amax paths, edge shapes and special values."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu


def check(x: np.ndarray, g=None, what="", dequant=True):
    xd = dev(x)
    gd = None if g is None else torch.tensor(np.float32(g), device="cuda")
    p, b, gs = mxq.nvfp4_quantize(xd, global_scale=gd)
    po, bo, go = oracle.nvfp4_quantize(x.reshape(-1, x.shape[-1]), global_scale=g)
    assert_same(np.array([np.float32(gs.item())]).view(np.uint32),
                np.array([go], np.float32).view(np.uint32), f"{what} global scale")
    assert_same(host(b).reshape(bo.shape), bo, f"{what} block scale")
    assert_same(host(p).reshape(po.shape), po, f"{what} packed")
    if dequant:
        for dt, name in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
            y = mxq.nvfp4_dequantize(p, b, gs, dt)
            assert_same(host(y).reshape(x.reshape(-1, x.shape[-1]).shape),
                        oracle.nvfp4_dequantize(po, bo, go, out=name), f"{what} dequant {name}")


@pytest.mark.slow
def test_full_size_tensor():
    check(W.nvfp4_tensor(), what="nvfp4 8192x8192")


def test_recipe_small():
    check(W.nvfp4_tensor(seed=61, M=300, N=1024), what="recipe")


def test_e2m1_rounding_sweep():
    check(W.nvfp4_e2m1_sweep_fp32(), g=1.0, what="e2m1 sweep", dequant=False)


def test_block_scale_sweep():
    x = W.nvfp4_block_scale_sweep_fp32()
    check(x, g=1.0, what="block-scale sweep g=1")
    check(x, what="block-scale sweep computed g")
    check(x, g=0.0173, what="block-scale sweep g=0.0173")


def test_given_amax_and_amax_entry():
    x = W.nvfp4_tensor(seed=62, M=512, N=2048)
    xd = dev(x)
    a = mxq.nvfp4_amax(xd)
    assert np.float32(a.item()) == oracle.nvfp4_global_amax(x)
    p1, b1, g1 = mxq.nvfp4_quantize(xd)
    p2, b2, g2 = mxq.nvfp4_quantize(xd, amax=a)
    assert torch.equal(p1, p2) and torch.equal(b1, b2) and torch.equal(g1, g2)


@pytest.mark.parametrize("M,N", [(1, 16), (3, 48), (33, 4096), (4095, 96), (257, 7168)])
def test_ragged_shapes(M, N):
    check(W.nvfp4_tensor(seed=M + N, M=M, N=N), what=f"{M}x{N}")


def test_fp32_and_strided_input():
    rng = np.random.default_rng(63)
    xf = (rng.standard_t(3, (200, 512)) * 2).astype(np.float32)
    check(xf, what="fp32")
    base = W.nvfp4_tensor(seed=64, M=128, N=1024)
    p, b, g = mxq.nvfp4_quantize(dev(base)[:, 128:128 + 512])
    po, bo, go = oracle.nvfp4_quantize(np.ascontiguousarray(base[:, 128:640]))
    assert np.float32(g.item()) == go
    assert_same(host(b), bo, "strided block scale")
    assert_same(host(p), po, "strided packed")


def test_zero_and_special_values():
    z = np.zeros((4, 64), np.uint16)
    z[1, 3] = 0x8000
    check(z, what="zero tensor")
    x = W.nvfp4_tensor(seed=65, M=16, N=256)
    x[0, :16] = 0                                  # an all-zero block
    x[1, 0] = 0x0001                               # a tiny block (scale rounds to 0)
    x[1, 1:16] = 0x8001
    x[2, 5] = 0x7FC0                               # NaN inside a block
    check(x, what="special blocks")
    y = x.copy()
    y[3, 7] = 0x7F80                               # +inf: outside the contract, still deterministic
    check(y, what="inf input")


def test_errors():
    with pytest.raises(mxq.MxqError):
        mxq.nvfp4_quantize(torch.zeros(4, 24, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("M,S", [(1, 1), (130, 7), (300, 33), (256, 224), (4096, 512)])
def test_swizzle_scales_standalone(M, S):
    """mxq_swizzle_scales on arbitrary bytes equals the oracle's layout."""
    s = np.random.default_rng(M * 7 + S).integers(0, 256, (M, S), dtype=np.uint8)
    z = mxq.swizzle_scales(dev(s))
    assert_same(host(z), oracle.swizzle_scales(s), f"swizzled [{M}, {S}]")


def test_nvfp4_block_scales_swizzled():
    x = W.nvfp4_tensor(seed=44, M=333, N=1024)
    _, b, _ = mxq.nvfp4_quantize(dev(x))
    _, bo, _ = oracle.nvfp4_quantize(x)
    assert_same(host(mxq.swizzle_scales(b)), oracle.swizzle_scales(bo), "NVFP4 swizzled block scales")


def _nvfp4_values(packed, bs):
    """float64 [M, N] of decode_e2m1(code) * decode_e4m3(block scale), from
    the oracle's outputs (the global scale left out)."""
    e2 = np.array([oracle.e2m1_decode(c) for c in range(16)], np.float64)
    e4 = oracle.e4m3_decode_table()
    codes = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(packed.shape[0], -1)
    return e2[codes] * np.repeat(e4[bs], 16, axis=1)


def test_nvfp4_swizzled_block_scales_feed_a_library_gemm():
    """NVIDIA's library block-scaled GEMM (through torch scaled_mm, NVFP4
    operands with E4M3 block scales per 16 in the 128x4-tile layout) reads
    this library's packed codes and swizzled block scales and reproduces the
    oracle's product within fp32 accumulation error: a consumer pin of the
    NVFP4 scale layout. Each E2M1 x E4M3 product pair is exact in fp32."""
    F = torch.nn.functional
    M, N, K = 256, 384, 512
    xa, xb = W.nvfp4_tensor(seed=45, M=M, N=K), W.nvfp4_tensor(seed=46, M=N, N=K)
    pa, ba, _ = mxq.nvfp4_quantize(dev(xa))
    pb, bb, _ = mxq.nvfp4_quantize(dev(xb))
    try:
        d = F.scaled_mm(pa.view(torch.float4_e2m1fn_x2), pb.view(torch.float4_e2m1fn_x2).t(),
                        mxq.swizzle_scales(ba).view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                        mxq.swizzle_scales(bb).view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.float32)
    except (RuntimeError, NotImplementedError, TypeError, AttributeError) as e:
        pytest.skip(f"this torch build runs no NVFP4 scaled_mm: {str(e)[:120]}")
    torch.cuda.synchronize()
    pao, bao, _ = oracle.nvfp4_quantize(xa)
    pbo, bbo, _ = oracle.nvfp4_quantize(xb)
    A, B = _nvfp4_values(pao, bao), _nvfp4_values(pbo, bbo)
    exact = A @ B.T
    tol = K * 2.0 ** -22 * (np.abs(A) @ np.abs(B).T) + 1e-30
    got = d.cpu().numpy().astype(np.float64)
    bad = np.abs(got - exact) > tol
    assert not bad.any(), f"{int(bad.sum())} entries outside the bound, first {np.argwhere(bad)[:4].tolist()}"
