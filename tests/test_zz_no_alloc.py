"""nvfp4_quantize_noalloc, the NVFP4 entry point for callers that cannot
allocate device memory when they quantize (a serving engine or plugin with
pre-planned memory, a C program without a device allocator): it must give
exactly the bytes of nvfp4_quantize with a caller-provided workspace, on two
calls in a row that reuse its fixed internal scratch.

Kept in its own file, collected last, and called through the C ABI.
"""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = ctypes.CDLL(mxq.library_path)
    f = lib.nvfp4_quantize_noalloc
    vp, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32
    f.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, u32, vp]
    f.restype = i32
    return f


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _run_noalloc(f, x):
    M, N = x.shape
    packed = torch.empty((M, N // 2), dtype=torch.uint8, device=x.device)
    bs = torch.empty((M, N // 16), dtype=torch.uint8, device=x.device)
    g = torch.empty((), dtype=torch.float32, device=x.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream)
    st = f(_ptr(x), 0, M, N, N, _ptr(packed), _ptr(bs), _ptr(g), None, 0, stream)
    assert st == 0, mxq.lib.mxq_status_string(st)
    return packed, bs, g


def test_noalloc_matches_workspace_entry_point_twice():
    f = _noalloc_fn()
    for seed, (M, N) in ((81, (1024, 4096)), (82, (777, 2080))):
        x = W.nvfp4_tensor(seed=seed, M=M, N=N)
        xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
        p1, b1, g1 = _run_noalloc(f, xd)
        p2, b2, g2 = mxq.nvfp4_quantize(xd)          # workspace allocated by the caller
        torch.cuda.synchronize()
        assert torch.equal(g1, g2)
        assert torch.equal(b1, b2)
        assert torch.equal(p1, p2)
