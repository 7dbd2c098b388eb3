"""The benchmark's algorithmic byte counts (the numerators of every GB/s and
roofline figure it prints) equal the sizes of the buffers each kernel reads
and writes: the input, the codes, the compact scales and, where written, the
swizzled scales as the library sizes them. No GPU needed."""
import pytest

import bench
import nvfp4_block_scaled_sm_b200 as mxq

SHAPES = [(16384, 7168), (4096, 4096), (256, 1024), (33, 96), (131072, 7168), (8192, 8192)]


@pytest.mark.parametrize("M,N", SHAPES)
def test_mxfp8_quantize_and_dequantize_bytes(M, N):
    E = M * N
    codes, scales = E, M * (N // 32)
    swz = mxq.swizzled_scale_bytes(M, N // 32)
    assert bench.mxfp8_quant_bytes(M, N) == 2 * E + codes + scales + swz
    assert bench.mxfp8_quant_bytes(M, N, swizzled=False) == 2 * E + codes + scales
    assert bench.mxfp8_quant_bytes(M, N, in_bytes=4, swizzled=False) == 4 * E + codes + scales
    assert bench.mxfp8_dequant_bytes(M, N) == codes + scales + 2 * E
    assert bench.mxfp8_dequant_bytes(M, N, 4) == codes + scales + 4 * E


@pytest.mark.parametrize("M,N", SHAPES)
def test_mxfp4_fake_and_nvfp4_bytes(M, N):
    E = M * N
    assert bench.mxfp4_quant_bytes(M, N) == 2 * E + E // 2 + M * (N // 32)
    assert bench.mxfp4_dequant_bytes(M, N) == E // 2 + M * (N // 32) + 2 * E
    assert bench.fake_quant_bytes(M, N) == 4 * E
    # two passes read the input twice; outputs: packed codes, E4M3 block
    # scales (one per 16), the fp32 global scale
    assert bench.nvfp4_quant_bytes(M, N) == 4 * E + E // 2 + M * (N // 16) + 4
    assert bench.nvfp4_quant_bytes(M, N, two_pass=False) == 2 * E + E // 2 + M * (N // 16) + 4


def test_headline_step_bytes():
    """The bench step on the 16384 x 7168 activation: 359,661,568 B for the
    quantize with swizzled scales and 355,991,552 B for the dequantize."""
    assert bench.mxfp8_quant_bytes(16384, 7168) == 359_661_568
    assert bench.mxfp8_dequant_bytes(16384, 7168) == 355_991_552
