"""The library's calls inside a CUDA graph. Every entry point allocates
nothing itself, never synchronizes and returns its status before any launch,
so a sequence of calls can be captured once and replayed on new data written
into the captured input buffer: MXFP8 rowwise with swizzled scales,
dequantize, columnwise, grouped with device row offsets and per-expert
swizzled scales, NVFP4 with its amax pass (workspace from the binding's
allocator), the no-alloc NVFP4 entry point and the tcgen05 GEMM. Each replay
must give exactly what eager calls give on the same input, and the
quantizers' outputs what the oracle gives."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, host

pytestmark = pytest.mark.gpu

M, N, NW = 1024, 4096, 512
OFFSETS = [0, 100, 100, 700, 1024]          # ragged experts, one of them empty


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc_fn():
    f = ctypes.CDLL(mxq.library_path).nvfp4_quantize_noalloc
    vp, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32
    f.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, u32, vp]
    f.restype = i32
    return f


def _sequence(x, wq, wz, offs, noalloc, noalloc_out):
    """The captured work: one call of each kind on x; returns the outputs."""
    q, s, z = mxq.mxfp8_quantize(x, swizzled=True)
    y = mxq.mxfp8_dequantize(q, s, torch.bfloat16)
    qt, st = mxq.mxfp8_quantize_columnwise(x)
    qg, sg, zg = mxq.mxfp8_quantize_grouped(x, row_offsets=offs, swizzled=True)
    p, b, g = mxq.nvfp4_quantize(x)
    pk, bs, gn = noalloc_out
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = noalloc(ctypes.c_void_p(x.data_ptr()), 0, M, N, N, ctypes.c_void_p(pk.data_ptr()),
                     ctypes.c_void_p(bs.data_ptr()), ctypes.c_void_p(gn.data_ptr()), None, 0, stream)
    assert status == 0, mxq.lib.mxq_status_string(status)
    d = mxq.mxfp8_gemm(q, z, wq, wz)
    return {"q": q, "s": s, "z": z, "y": y, "qt": qt, "st": st, "qg": qg, "sg": sg, "zg": zg,
            "p": p, "b": b, "g": g, "pk": pk, "bs": bs, "gn": gn, "d": d}


def _check_oracle(x: np.ndarray, out: dict, what: str):
    qo, so = oracle.mxfp8_quantize(x)
    assert_same(host(out["q"]), qo, f"{what}: mxfp8 codes")
    assert_same(host(out["s"]), so, f"{what}: mxfp8 scales")
    assert_same(host(out["z"]), oracle.swizzle_scales(so), f"{what}: swizzled scales")
    assert_same(host(out["y"]), oracle.mxfp8_dequantize(qo, so, out="bf16"), f"{what}: dequantize")
    qto, sto = oracle.mxfp8_quantize_colwise(x)
    assert_same(host(out["qt"]), qto, f"{what}: columnwise codes")
    assert_same(host(out["st"]), sto, f"{what}: columnwise scales")
    parts = [x[a:b] for a, b in zip(OFFSETS[:-1], OFFSETS[1:])]
    qgo, sgo, zgo = oracle.mxfp8_quantize_grouped(parts, swizzled=True)
    assert_same(host(out["qg"]), qgo, f"{what}: grouped codes")
    assert_same(host(out["sg"]), sgo, f"{what}: grouped scales")
    assert_same(host(out["zg"])[:zgo.size], zgo, f"{what}: per-expert swizzled scales")
    po, bo, go = oracle.nvfp4_quantize(x)
    for p, b, g, which in (("p", "b", "g", "nvfp4"), ("pk", "bs", "gn", "nvfp4 no-alloc")):
        assert_same(host(out[g]).reshape(1), np.array([go], np.float32), f"{what}: {which} global scale")
        assert_same(host(out[b]), bo, f"{what}: {which} block scales")
        assert_same(host(out[p]), po, f"{what}: {which} codes")


def test_captured_sequence_replays_exactly():
    xs = [W.activation(seed=201, M=M, N=N), W.activation(seed=202, M=M, N=N)]
    wq, _, wz = mxq.mxfp8_quantize(_bf16(W.linear_weight(seed=203, M=NW, N=N)), swizzled=True)
    offs = torch.tensor(OFFSETS, dtype=torch.int64, device="cuda")
    noalloc = _noalloc_fn()
    noalloc_out = (torch.empty((M, N // 2), dtype=torch.uint8, device="cuda"),
                   torch.empty((M, N // 16), dtype=torch.uint8, device="cuda"),
                   torch.empty((), dtype=torch.float32, device="cuda"))

    # eager runs first: the results to compare with, and every first-use
    # set-up (shared-memory limits, the no-alloc scratch address) done
    # outside the capture
    eager = []
    for xin in xs:
        out = _sequence(_bf16(xin), wq, wz, offs, noalloc, noalloc_out)
        eager.append({k: v.clone() for k, v in out.items()})
    torch.cuda.synchronize()

    x_static = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    x_static.copy_(_bf16(xs[0]))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = _sequence(x_static, wq, wz, offs, noalloc, noalloc_out)

    for i in (1, 0, 1):                      # replays on new data, in either order
        x_static.copy_(_bf16(xs[i]))
        for t in out.values():
            t.zero_()                        # nothing left over from the last replay
        graph.replay()
        torch.cuda.synchronize()
        for k, v in out.items():
            assert torch.equal(v, eager[i][k]), f"replay on input {i}: {k} differs from the eager call"
    _check_oracle(xs[1], out, "replay on input 1")
    del graph
