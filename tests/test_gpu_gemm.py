"""The tensor-core block-scaled MXFP8 GEMM (tcgen05 kind::mxf8f6f4) against
the oracle's product of the oracle-quantized operands, and the swizzled
scale layout against an independent consumer (torch's MX scaled_mm, which
runs NVIDIA's library GEMM on the same codes and swizzled scales).

Both sides start from the same seeded bf16 inputs: the GPU quantizes them
(codes + swizzled scales) and multiplies; the oracle quantizes them (codes +
compact scales) and forms the float64 product.

Tolerance. Each product of two E4M3 values and two powers of two is exact;
the hardware sums K of them in fp32 in an order of its choosing. A sum of K
terms with per-addition relative error u has error at most K * u * sum|ab|;
u is taken as 2^-22 (four times the round-to-nearest unit, so truncating or
partially aligned accumulation is also covered). bf16 output adds half an
ulp of the rounded sum: bf16 keeps 8 significant bits, so at most 2^-8 of
its magnitude. On the power-of-two grid inputs every
partial sum is exactly representable in fp32, so fp32 output must be exact.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


def gpu_operands(xa, xb):
    qa, sa, za = mxq.mxfp8_quantize(dev(xa), swizzled=True)
    qb, sb, zb = mxq.mxfp8_quantize(dev(xb), swizzled=True)
    return qa, za, qb, zb


def oracle_product(xa, xb):
    qa, sa = oracle.mxfp8_quantize(xa)
    qb, sb = oracle.mxfp8_quantize(xb)
    exact = oracle.mxfp8_gemm(qa, sa, qb, sb)
    t = oracle.e4m3_decode_table()
    K = xa.shape[1]
    A = np.abs(np.ldexp(t[qa], np.repeat(sa.astype(np.int64) - 127, 32, axis=1)[:, :K]))
    B = np.abs(np.ldexp(t[qb], np.repeat(sb.astype(np.int64) - 127, 32, axis=1)[:, :K]))
    return exact, A @ B.T


def run(xa, xb, dtype=torch.float32):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qa, za, qb, zb = gpu_operands(xa, xb)
    d = mxq.mxfp8_gemm(qa, za, qb, zb, dtype, error_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, "a wait in the GEMM kernel gave up"
    return d


def check_tol(d, exact, absum, K, bf16, what):
    got = d.float().cpu().numpy() if isinstance(d, torch.Tensor) else np.asarray(d)
    got = got.astype(np.float64)
    acc = K * 2.0 ** -22 * absum
    tol = acc + (2.0 ** -8 * (np.abs(exact) + acc) if bf16 else 0) + 1e-30
    bad = np.abs(got - exact) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} entries outside the bound, first at {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (256, 384, 1024), (33, 48, 96), (1, 16, 32),
                                   (200, 144, 2048), (300, 272, 160),
                                   (2048, 4096, 256), (3000, 3008, 96)])  # more tiles than SMs
def test_power_of_two_grid_is_exact(M, N, K):
    xa = W.gemm_pow2_operand(1000 + M, M, K)
    xb = W.gemm_pow2_operand(2000 + N, N, K)
    d = run(xa, xb)
    exact, _ = oracle_product(xa, xb)
    got = host(d).view(np.float32).astype(np.float64)
    bad = got != exact
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} differ; first {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (33, 48, 96), (1, 16, 32), (300, 272, 160),
                                   (129, 400, 224), (3000, 3008, 96)])
def test_power_of_two_grid_bf16_is_rounded_exact(M, N, K):
    """bf16 output on the power-of-two grid: the fp32 sum is exact there, so
    each output must be that value rounded to nearest even bf16 (the
    epilogue's row and column edges included)."""
    xa = W.gemm_pow2_operand(3000 + M, M, K)
    xb = W.gemm_pow2_operand(4000 + N, N, K)
    d = run(xa, xb, torch.bfloat16)
    exact, _ = oracle_product(xa, xb)
    want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    got = d.view(torch.int16).cpu().numpy()
    bad = got != want
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} differ; first {np.argwhere(bad)[:4].tolist()}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_activation_times_weight(dtype):
    xa = W.activation(seed=105, M=512, N=2048)
    xb = W.linear_weight(seed=106, M=384, N=2048)
    d = run(xa, xb, dtype)
    exact, absum = oracle_product(xa, xb)
    check_tol(d, exact, absum, 2048, dtype == torch.bfloat16, "activation x weight")


def test_ragged_tiles_and_tail_k():
    xa = W.activation(seed=107, M=129, N=224)     # K = 224: one full block of 128 and a tail of 96
    xb = W.linear_weight(seed=108, M=208, N=224)
    d = run(xa, xb)
    exact, absum = oracle_product(xa, xb)
    check_tol(d, exact, absum, 224, False, "ragged")


def test_swizzled_layout_against_library_consumer():
    """torch's MX scaled_mm reads codes and 128x4-tile swizzled E8M0 scales;
    given this library's swizzled scales it must reproduce the oracle's
    product (and so must this library's own GEMM)."""
    F = torch.nn.functional
    xa = W.activation(seed=109, M=256, N=512)
    xb = W.linear_weight(seed=110, M=256, N=512)
    qa, za, qb, zb = gpu_operands(xa, xb)
    y = F.scaled_mm(qa.view(torch.float8_e4m3fn), qb.view(torch.float8_e4m3fn).t(),
                    za.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                    zb.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                    swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                    output_dtype=torch.float32)
    exact, absum = oracle_product(xa, xb)
    check_tol(y, exact, absum, 512, False, "library MX GEMM on our swizzled scales")
    d = mxq.mxfp8_gemm(qa, za, qb, zb, torch.float32)
    check_tol(d, exact, absum, 512, False, "tcgen05 GEMM")


def test_k_zero_and_errors():
    qa = torch.zeros(4, 0, dtype=torch.uint8, device="cuda")
    qb = torch.zeros(16, 0, dtype=torch.uint8, device="cuda")
    z = torch.zeros(1, dtype=torch.uint8, device="cuda")
    d = mxq.mxfp8_gemm(qa, z, qb, z, torch.float32)
    assert d.shape == (4, 16) and not d.any()
    qa = torch.zeros(4, 64, dtype=torch.uint8, device="cuda")
    qb = torch.zeros(24, 64, dtype=torch.uint8, device="cuda")
    zs = torch.zeros(mxq.swizzled_scale_bytes(128, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(mxq.MxqError):
        mxq.mxfp8_gemm(qa, zs, qb, zs)              # N % 16 != 0


@pytest.mark.slow
def test_full_size_sampled():
    """The size the benchmark times: activation 16384x7168 times a
    7168x7168 weight, checked on sampled rows and columns."""
    xa = W.activation()
    xb = W.linear_weight(seed=111, M=7168, N=7168)
    d = run(xa, xb, torch.bfloat16)
    rng = np.random.default_rng(112)
    rows = np.sort(rng.choice(16384, 48, replace=False))
    cols = np.sort(rng.choice(7168, 40, replace=False))
    exact, absum = oracle_product(xa[rows], xb[cols])
    got = d.float().cpu().numpy()[np.ix_(rows, cols)]
    check_tol(got, exact, absum, 7168, True, "full size, sampled")


@pytest.mark.parametrize("fmt_rows", [[128, 200, 64, 0, 1], [256, 300]])
def test_per_expert_swizzled_scales_feed_the_gemm(fmt_rows):
    """The grouped quantize's per-expert swizzled scales, read by the tensor
    cores: expert e's block of the swizzled output is handed to the GEMM as
    that expert's scale layout, and each expert's product must equal the
    oracle's exactly (power-of-two grid inputs). This pins the per-expert
    layout with a hardware consumer, not only with the oracle's composition."""
    rows = fmt_rows
    K = 256
    parts = [W.gemm_pow2_operand(3000 + i, max(r, 1), K)[:r] for i, r in enumerate(rows)]
    x = np.concatenate(parts, 0)
    offs = np.concatenate([[0], np.cumsum(rows)]).tolist()
    q, s, z = mxq.mxfp8_quantize_grouped(dev(x), row_offsets=offs, swizzled=True)
    xb = W.gemm_pow2_operand(4000, 144, K)
    qb, _, zb = mxq.mxfp8_quantize(dev(xb), swizzled=True)
    qbo, sbo = oracle.mxfp8_quantize(xb)
    pos = 0
    for e, r in enumerate(rows):
        nb = mxq.swizzled_scale_bytes(r, K // 32)
        if r:
            d = mxq.mxfp8_gemm(q[offs[e]:offs[e + 1]].contiguous(), z[pos:pos + nb], qb, zb,
                               torch.float32)
            qa_o, sa_o = oracle.mxfp8_quantize(parts[e])
            exact = oracle.mxfp8_gemm(qa_o, sa_o, qbo, sbo)
            got = host(d).view(np.float32).astype(np.float64)
            assert np.array_equal(got, exact), f"expert {e}: {int((got != exact).sum())} entries differ"
        pos += nb
    assert pos == z.numel()
