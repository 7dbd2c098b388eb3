"""The C ABI from plain C on the GPU: tests/c/gpu_roundtrip.c (no Python and
no torch in its process) quantizes and dequantizes a bf16 tensor to MXFP8 and
NVFP4-quantizes another through libmxq.so; its outputs must equal the
oracle's byte for byte, and the rows built from the hand-worked groups must
give their worked bytes.
"""
import json
import os
import shutil
import subprocess

import numpy as np
import pytest

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "hand_worked.json")


def _golden_rows():
    """One 32-element row per hand-worked MXFP8 group, with its worked scale
    byte and codes."""
    rows, want = [], []
    for case in json.load(open(GOLDEN))["mxfp8"]:
        vals = [case["fill"]] * 32
        for k, v in case["x"].items():
            vals[int(k)] = v
        bits = [int(v, 16) if isinstance(v, str) and v.startswith("0x") else int(W.bits_of([float(v)])[0])
                for v in vals]
        codes = [int(case["q"]["fill"])] * 32
        for k, v in case["q"].items():
            if k != "fill":
                codes[int(k)] = int(v)
        rows.append(bits)
        want.append((case["name"], case["scale"], codes))
    return np.array(rows, np.uint16), want


def _build(tmp_dir):
    cc = shutil.which("gcc") or shutil.which("cc")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if cc is None or not os.path.exists(os.path.join(cuda, "include", "cuda_runtime_api.h")):
        pytest.skip("no C compiler or CUDA toolkit headers")
    libdir = os.path.dirname(mxq.library_path)
    exe = os.path.join(tmp_dir, "gpu_roundtrip")
    build = subprocess.run(
        [cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(os.path.dirname(HERE), "include"),
         "-I", os.path.join(cuda, "include"), os.path.join(HERE, "c", "gpu_roundtrip.c"),
         "-L", libdir, "-lmxq", "-L", os.path.join(cuda, "lib64"), "-lcudart",
         f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", exe],
        capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    return exe


def test_c_program_on_the_gpu():
    out_dir = os.path.join(HERE, "c", "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = _build(out_dir)
    golden, want = _golden_rows()
    G = golden.shape[0]
    # golden groups in columns 0..31 of the first rows, random data elsewhere;
    # 130 rows cross a 128-row swizzle tile and leave a ragged one
    M, N = 130, 96
    x = W.activation(seed=301, M=M, N=N).copy()
    x[:G, :32] = golden
    xn = W.nvfp4_tensor(seed=302, M=M, N=N)       # finite: NVFP4's contract
    src, src_n = os.path.join(out_dir, "x.bin"), os.path.join(out_dir, "xn.bin")
    x.astype("<u2").tofile(src)
    xn.astype("<u2").tofile(src_n)
    prefix = os.path.join(out_dir, "out")
    run = subprocess.run([exe, str(M), str(N), src, src_n, prefix], capture_output=True, text=True,
                         timeout=300)
    assert run.returncode == 0, run.stdout + run.stderr

    def load(ext, dtype, shape):
        return np.fromfile(f"{prefix}.{ext}", dtype=dtype).reshape(shape)

    q = load("q", np.uint8, (M, N))
    s = load("s", np.uint8, (M, N // 32))
    z = load("z", np.uint8, (-1,))
    y = load("y", np.uint16, (M, N))
    for r, (name, scale, codes) in enumerate(want):
        assert int(s[r, 0]) == scale, f"hand-worked group {name}: scale byte"
        assert q[r, :32].tolist() == codes, f"hand-worked group {name}: codes"
    qo, so = oracle.mxfp8_quantize(x)
    assert_same(q, qo, "codes")
    assert_same(s, so, "scales")
    assert_same(z, oracle.swizzle_scales(so), "swizzled scales")
    assert_same(y, oracle.mxfp8_dequantize(qo, so, out="bf16"), "dequantize")
    po, bo, go = oracle.nvfp4_quantize(xn)
    assert_same(load("g4", np.uint32, (1,)), np.array([go], np.float32), "nvfp4 global scale (bits)")
    assert_same(load("b4", np.uint8, (M, N // 16)), bo, "nvfp4 block scales")
    assert_same(load("p4", np.uint8, (M, N // 2)), po, "nvfp4 codes")
