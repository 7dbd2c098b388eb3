"""nvfp4_quantize_noalloc, the NVFP4 entry point for callers that cannot
allocate device memory when they quantize (a serving engine or plugin with
pre-planned memory, a C program without a device allocator): it must give
exactly the bytes of nvfp4_quantize with a caller-provided workspace, and of
the CPU oracle, on calls in a row that reuse its fixed internal scratch.

Kept in its own file, collected last, and called through the C ABI. Every
output lives between canary bands that are checked after the calls.
"""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, guarded_empty, host

pytestmark = pytest.mark.gpu

GIVEN = 1


def _noalloc_fn():
    lib = ctypes.CDLL(mxq.library_path)
    f = lib.nvfp4_quantize_noalloc
    vp, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32
    f.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, u32, vp]
    f.restype = i32
    return f


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _launch_noalloc(f, alloc, x, g=None, amax=None, flags=0):
    """Enqueues one noalloc call on the current stream (no synchronize);
    returns its outputs."""
    M, N = x.shape
    packed = guarded_empty(alloc, (M, N // 2), torch.uint8)
    bs = guarded_empty(alloc, (M, N // 16), torch.uint8)
    if g is None:
        g = guarded_empty(alloc, (), torch.float32)
    stream = ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream)
    st = f(_ptr(x), 0, M, N, N, _ptr(packed), _ptr(bs), _ptr(g), _ptr(amax), flags, stream)
    assert st == 0, mxq.lib.mxq_status_string(st)
    return packed, bs, g


def _bf16(x):
    return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()


def _check_oracle(x, out, what, g_given=None):
    po, bo, go = oracle.nvfp4_quantize(x, g_given)
    p, b, g = out
    assert_same(host(g).reshape(1), np.array([go], np.float32), f"{what} global scale")
    assert_same(host(b), bo, f"{what} block scales")
    assert_same(host(p), po, f"{what} packed codes")


def test_noalloc_matches_workspace_entry_point_and_oracle_twice(guard_bands):
    f = _noalloc_fn()
    for seed, (M, N) in ((81, (1024, 4096)), (82, (777, 2080))):
        x = W.nvfp4_tensor(seed=seed, M=M, N=N)
        xd = _bf16(x)
        got = _launch_noalloc(f, guard_bands, xd)
        p2, b2, g2 = mxq.nvfp4_quantize(xd)          # workspace allocated by the caller
        torch.cuda.synchronize()
        assert torch.equal(got[2], g2)
        assert torch.equal(got[1], b2)
        assert torch.equal(got[0], p2)
        _check_oracle(x, got, f"noalloc {M}x{N}")


def test_noalloc_calls_queued_back_to_back(guard_bands):
    """Three calls on one stream with no host synchronize between them: two
    different inputs, then the first again. Each call rewrites every scratch
    slot it reads, so stream order alone keeps them apart."""
    f = _noalloc_fn()
    xa = W.nvfp4_tensor(seed=83, M=2048, N=3072)
    xb = W.nvfp4_tensor(seed=84, M=300, N=8192).copy()
    xb[0, 5] = 0x4700                                 # 32768: a different tensor amax
    da, db = _bf16(xa), _bf16(xb)
    outs = [_launch_noalloc(f, guard_bands, d) for d in (da, db, da)]
    torch.cuda.synchronize()
    _check_oracle(xa, outs[0], "first call")
    _check_oracle(xb, outs[1], "second call")
    _check_oracle(xa, outs[2], "third call (first input again)")


def test_noalloc_given_scale_and_given_amax(guard_bands):
    """The two modes that need no scratch: a given global scale, and a given
    tensor amax; both equal nvfp4_quantize and the oracle."""
    f = _noalloc_fn()
    x = W.nvfp4_tensor(seed=85, M=513, N=1024)
    xd = _bf16(x)
    g = guarded_empty(guard_bands, (), torch.float32)
    g.fill_(0.0371)
    given = _launch_noalloc(f, guard_bands, xd, g=g, flags=GIVEN)
    ref = mxq.nvfp4_quantize(xd, global_scale=g.clone())
    amax = guarded_empty(guard_bands, (), torch.float32)
    amax.fill_(float(oracle.nvfp4_global_amax(x)))
    from_amax = _launch_noalloc(f, guard_bands, xd, amax=amax)
    ref_amax = mxq.nvfp4_quantize(xd, amax=amax)
    torch.cuda.synchronize()
    for a, b in zip(given, ref):
        assert torch.equal(a, b)
    for a, b in zip(from_amax, ref_amax):
        assert torch.equal(a, b)
    _check_oracle(x, given, "given scale", g_given=float(np.float32(0.0371)))
    _check_oracle(x, from_amax, "given amax")
