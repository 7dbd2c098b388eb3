"""The benchmark's algorithmic byte counts (the numerators of every GB/s and
roofline figure it prints) equal the sizes of the buffers each kernel reads
and writes: the input, the codes, the compact scales and, where written, the
swizzled scales as the library sizes them. No GPU needed."""
import os

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


def test_cpu_baseline_chunks_equal_one_call():
    """The benchmark's multi-core oracle leg (row chunks on threads, each a
    single-threaded oracle call) gives the bytes of one call over all rows."""
    import numpy as np

    import oracle
    import workloads as W
    x = W.activation(seed=3, M=300, N=256)
    parts = bench.oracle_rows_parallel(bench.oracle_round_trip, x, 4)
    q, s, z, y = (np.concatenate([p[i] for p in parts]) for i in range(4))
    qo, so = oracle.mxfp8_quantize(x)
    assert np.array_equal(q, qo) and np.array_equal(s, so)
    assert np.array_equal(y, oracle.mxfp8_dequantize(qo, so, out="bf16"))
    # 128-row chunks: each chunk's swizzled block is a slice of the whole layout
    assert np.array_equal(z[:256 * 8], oracle.swizzle_scales(so)[:256 * 8])


@pytest.mark.parametrize("M", [1, 127, 300, 512, 1000, 4096, 16384, 16385])
def test_e2e_chunks_cover_the_rows(M):
    """The end-to-end pipeline's chunks tile [0, M) in order, each starting on
    a 128-row boundary (so its swizzled scales are one slice of the full
    layout), the first at most 512 rows and none above 2048."""
    b = bench.e2e_chunks(M)
    assert b[0] == 0 and b[-1] == M
    sizes = [r1 - r0 for r0, r1 in zip(b[:-1], b[1:])]
    assert all(n > 0 for n in sizes)
    assert all(r0 % 128 == 0 for r0 in b[:-1])
    assert sizes[0] <= 512 and max(sizes) <= 2048


def test_sample_rows():
    import numpy as np
    r = bench.sample_rows(8192, 100, 5)
    assert r[0] == 0 and r[-1] == 8191 and np.all(np.diff(r) > 0)
    assert set(range(64)) <= set(r.tolist()) and set(range(8128, 8192)) <= set(r.tolist())


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores, no GPU)
    prints one JSON line with the keys the driver reads."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    run = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, cwd=root)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [l for l in run.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, run.stdout[-2000:]
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_bench_rejects_short_warmup():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    run = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--warmup", "2"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert run.returncode != 0
    assert "warmup" in (run.stdout + run.stderr)
