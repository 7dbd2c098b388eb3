"""The sharded NVFP4 path with the real kernels: two processes share the one
GPU, each quantizes its row shard with `nvfp4_quantize_sharded` (the GPU
tensor amax of its shard, a MAX all-reduce of that one fp32 over gloo, then
the block pass with the global amax), and the shards together must equal
the whole tensor quantized in one call, byte for byte, with the same global
scale on both ranks. The ranks' kernels never wait on each other; the only
exchange goes through the host. MXFP8 needs no exchange: each rank's rows
must equal the matching rows of the whole-tensor call."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import nvfp4_block_scaled_sm_b200 as mxq
import workloads as W

pytestmark = pytest.mark.gpu

M, N, WORLD = 300, 512, 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _rank(rank, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import nvfp4_block_scaled_sm_b200 as lib
    import workloads as wl
    from nvfp4_block_scaled_sm_b200.distributed import nvfp4_quantize_sharded, shard_rows
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        x = wl.nvfp4_tensor(seed=501, M=M, N=N)
        b, e = shard_rows(M, WORLD, rank)
        xl = torch.from_numpy(np.ascontiguousarray(x[b:e]).view(np.int16)).view(torch.bfloat16).cuda()
        p, s, g = nvfp4_quantize_sharded(xl)
        qm, sm = lib.mxfp8_quantize(xl)
        torch.cuda.synchronize()
        q.put((rank, b, e, p.cpu().numpy(), s.cpu().numpy(), g.cpu().numpy(), qm.cpu().numpy(),
               sm.cpu().numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_on_one_gpu_match_the_whole_tensor():
    x = W.nvfp4_tensor(seed=501, M=M, N=N)
    p, s, g = mxq.nvfp4_quantize(_bf16(x))
    qm, sm = mxq.mxfp8_quantize(_bf16(x))
    p, s, g, qm, sm = (t.cpu().numpy() for t in (p, s, g, qm, sm))

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(WORLD)]
    for pr in procs:
        pr.start()
    got = [q.get(timeout=300) for _ in range(WORLD)]
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0, f"rank process exited with {pr.exitcode}"

    for rank, b, e, pl, sl, gl, qml, sml in sorted(got, key=lambda t: t[0]):
        assert gl.view(np.uint32) == g.view(np.uint32), f"rank {rank}: global scale"
        assert np.array_equal(pl, p[b:e]), f"rank {rank}: NVFP4 codes"
        assert np.array_equal(sl, s[b:e]), f"rank {rank}: NVFP4 block scales"
        assert np.array_equal(qml, qm[b:e]), f"rank {rank}: MXFP8 codes"
        assert np.array_equal(sml, sm[b:e]), f"rank {rank}: MXFP8 scales"
    assert sorted((t[1], t[2]) for t in got) == [(0, 150), (150, 300)]
