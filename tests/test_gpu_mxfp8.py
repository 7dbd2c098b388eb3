"""MXFP8 quantize / dequantize on the GPU against the CPU oracle, bit-exact:
identical qweight, scale and swizzled-scale bytes, identical dequantized
bf16 / fp32 bits. Inputs follow the workload recipes (full sizes for the
quantize workloads), plus exhaustive sweeps and edge shapes."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu


def check_quant(x: np.ndarray, swizzled=False, dequant=True, what=""):
    got = mxq.mxfp8_quantize(dev(x), swizzled=swizzled)
    qo, so = oracle.mxfp8_quantize(x.reshape(-1, x.shape[-1]))
    assert_same(host(got[0]).reshape(qo.shape), qo, f"{what} qweight")
    assert_same(host(got[1]).reshape(so.shape), so, f"{what} scale")
    if swizzled:
        assert_same(host(got[2]), oracle.swizzle_scales(so), f"{what} swizzled scale")
    if dequant:
        for dt, name in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
            y = mxq.mxfp8_dequantize(got[0], got[1], dt)
            assert_same(host(y).reshape(qo.shape), oracle.mxfp8_dequantize(qo, so, out=name),
                        f"{what} dequant {name}")
    return got


def test_planted_groups():
    check_quant(W.planted(), swizzled=True, what="planted")


def test_linear_weight_full_size():
    check_quant(W.linear_weight(), swizzled=True, what="linear weight 4096x4096")


@pytest.mark.slow
def test_activation_full_size_round_trip():
    check_quant(W.activation(), swizzled=True, what="activation 16384x7168")


def test_every_bf16_value_at_every_scale():
    check_quant(W.mxfp8_every_value_every_scale(), what="exhaustive")


def test_every_code_at_every_scale_dequant():
    q, s = W.mxfp8_all_code_scale_pairs()
    for dt, name in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        y = mxq.mxfp8_dequantize(dev(q), dev(s), dt)
        assert_same(host(y), oracle.mxfp8_dequantize(q, s, out=name), f"dequant pairs {name}")


def test_random_bit_patterns():
    rng = np.random.default_rng(31)
    x = rng.integers(0, 65536, (512, 2048), dtype=np.uint32).astype(np.uint16)
    check_quant(x, swizzled=True, what="random bf16 bits")


def test_fp32_input():
    rng = np.random.default_rng(32)
    xf = (rng.standard_t(3, (300, 1024)) * 0.5).astype(np.float32)
    xf[0, :32] = 0
    xf[1, 3] = np.nan
    xf[2, 4] = -np.inf
    xf[3, :32] = np.ldexp(rng.uniform(-1, 1, 32), -135).astype(np.float32)
    xf[4, 0] = np.float32(3.4e38)
    xf[5, :] = rng.integers(0, 2**32, 1024, dtype=np.uint64).astype(np.uint32).view(np.float32)
    check_quant(xf, swizzled=True, what="fp32")


@pytest.mark.parametrize("M", [1, 31, 33, 4095])
@pytest.mark.parametrize("N", [32, 96, 7168])
def test_ragged_shapes(M, N):
    x = W.activation(seed=M * 7 + N, M=M, N=N)
    check_quant(x, swizzled=True, what=f"{M}x{N}")


def test_swizzle_padding_shapes():
    for M, N in ((130, 224), (1, 32), (257, 96), (128, 128)):
        check_quant(W.linear_weight(seed=M + N, M=M, N=N), swizzled=True, dequant=False,
                    what=f"swizzle {M}x{N}")


def test_leading_dims_and_row_stride():
    x = W.activation(seed=41, M=6 * 35, N=256).reshape(6, 35, 256)
    q, s = mxq.mxfp8_quantize(dev(x))
    qo, so = oracle.mxfp8_quantize(x.reshape(-1, 256))
    assert q.shape == (6, 35, 256) and s.shape == (6, 35, 8)
    assert_same(host(q).reshape(-1, 256), qo, "3-D qweight")
    assert_same(host(s).reshape(-1, 8), so, "3-D scale")
    base = W.activation(seed=42, M=300, N=1024)
    view = dev(base)[:, 64:64 + 640]                 # row stride 1024, N 640
    q, s, z = mxq.mxfp8_quantize(view, swizzled=True)
    qo, so = oracle.mxfp8_quantize_strided(base[:, 64:].copy(), 300, 640, 960)
    assert_same(host(q), qo, "strided qweight")
    assert_same(host(s), so, "strided scale")
    assert_same(host(z), oracle.swizzle_scales(so), "strided swizzle")
    basef = (np.random.default_rng(43).standard_normal((70, 512)) * 3).astype(np.float32)
    q, s = mxq.mxfp8_quantize(dev(basef)[:, :256])
    qo, so = oracle.mxfp8_quantize_strided(basef, 70, 256, 512)
    assert_same(host(q), qo, "strided fp32 qweight")
    assert_same(host(s), so, "strided fp32 scale")


def test_empty_and_errors():
    q, s = mxq.mxfp8_quantize(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"))
    assert q.shape == (0, 64) and s.shape == (0, 2)
    with pytest.raises(mxq.MxqError):
        mxq.mxfp8_quantize(torch.zeros(4, 48, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(TypeError):
        mxq.mxfp8_quantize(torch.zeros(4, 64, dtype=torch.float16, device="cuda"))


def test_deterministic_and_stream():
    x = dev(W.linear_weight(seed=44, M=512, N=1024))
    q1, s1 = mxq.mxfp8_quantize(x)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        q2, s2 = mxq.mxfp8_quantize(x)
    torch.cuda.current_stream().wait_stream(st)
    assert torch.equal(q1, q2) and torch.equal(s1, s2)


def test_requantize_is_identity():
    x = dev(W.activation(seed=45, M=256, N=2048))
    q, s = mxq.mxfp8_quantize(x)
    q2, s2 = mxq.mxfp8_quantize(mxq.mxfp8_dequantize(q, s, torch.float32))
    assert torch.equal(q, q2) and torch.equal(s, s2)


def test_nvtx_ranges_and_a_failing_allocation():
    """With NVTX ranges on, results are unchanged; an output allocation that
    fails (a host-side fault injected through the allocator hook) surfaces as
    the allocator's exception, and the next call works."""
    x = W.activation(seed=5, M=64, N=256)
    q0, s0 = mxq.mxfp8_quantize(dev(x))
    prev = mxq.set_nvtx(True)
    try:
        q1, s1 = mxq.mxfp8_quantize(dev(x))
    finally:
        mxq.set_nvtx(prev)
    assert torch.equal(q0, q1) and torch.equal(s0, s1)

    calls = []

    def failing(shape, dtype, device):
        calls.append(shape)
        if len(calls) == 2:
            raise MemoryError("injected allocation failure")
        return torch.empty(shape, dtype=dtype, device=device)

    old = mxq.set_output_allocator(failing)
    try:
        with pytest.raises(MemoryError, match="injected"):
            mxq.mxfp8_quantize(dev(x))
    finally:
        mxq.set_output_allocator(old)
    q2, s2 = mxq.mxfp8_quantize(dev(x))
    torch.cuda.synchronize()
    assert torch.equal(q0, q2) and torch.equal(s0, s2)
