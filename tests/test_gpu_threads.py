"""Calls from several host threads at once. The library keeps a little
host-side state: per-device caches of shared-memory limits, multiprocessor
and cluster counts, the no-alloc scratch address, and the driver entry
points it fetches once. Four threads, each with its own CUDA stream and
inputs, run mixed sequences concurrently (ctypes releases the interpreter
lock during each call). Every result must equal the same sequence run alone
on one thread."""
import threading

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_sm_b200 as mxq
import workloads as W

pytestmark = pytest.mark.gpu

THREADS, REPEATS = 4, 3


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _work(i: int, x: torch.Tensor, w: tuple):
    """One thread's sequence; a different mix per thread."""
    q, s, z = mxq.mxfp8_quantize(x, swizzled=True)
    out = {"q": q, "s": s, "z": z}
    if i % 2 == 0:
        out["y"] = mxq.mxfp8_dequantize(q, s, torch.float32)
        out["p"], out["b"], out["g"] = mxq.nvfp4_quantize(x)
    else:
        out["qt"], out["st"] = mxq.mxfp8_quantize_columnwise(x)
        out["p4"], out["s4"] = mxq.mxfp4_quantize(x)
    out["d"] = mxq.mxfp8_gemm(q, z, *w)
    return out


def test_threads_on_their_own_streams():
    xs = [_bf16(W.activation(seed=401 + i, M=512 + 128 * i, N=2048)) for i in range(THREADS)]
    wq, _, wz = mxq.mxfp8_quantize(_bf16(W.linear_weight(seed=410, M=384, N=2048)), swizzled=True)
    w = (wq, wz)

    expect = []
    for i in range(THREADS):                     # alone, one after the other
        expect.append({k: v.clone() for k, v in _work(i, xs[i], w).items()})
    torch.cuda.synchronize()

    results = [[] for _ in range(THREADS)]
    errors = []
    start = threading.Barrier(THREADS)

    def run(i):
        try:
            stream = torch.cuda.Stream()
            stream.wait_stream(torch.cuda.default_stream())
            with torch.cuda.stream(stream):
                start.wait()
                for _ in range(REPEATS):
                    out = _work(i, xs[i], w)
                    results[i].append({k: v.clone() for k, v in out.items()})
            stream.synchronize()
        except Exception as e:               # reported on the main thread
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=run, args=(i,)) for i in range(THREADS)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a thread did not finish"
    assert not errors, errors
    torch.cuda.synchronize()
    for i in range(THREADS):
        assert len(results[i]) == REPEATS
        for r, out in enumerate(results[i]):
            for k, v in out.items():
                assert torch.equal(v, expect[i][k]), f"thread {i}, repeat {r}: {k} differs from the lone run"
