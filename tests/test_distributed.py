"""World-size-2 gloo runs (CPU) of the multi-rank host logic: the NVFP4 amax
all-reduce of a row-sharded tensor, the row split, and the benchmark's
max-over-ranks reduction. Local compute uses the oracle (no GPU here)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workloads as W
        from nvfp4_block_scaled_sm_b200.distributed import allreduce_amax_, shard_rows
        import bench
        x = W.nvfp4_tensor(seed=71, M=37, N=256)
        b, e = shard_rows(37, world, rank)
        local = x[b:e]
        amax = torch.tensor(oracle.nvfp4_global_amax(local), dtype=torch.float32)
        allreduce_amax_(amax)
        g = np.float32(amax.item()) / np.float32(2688.0)
        p, s, g2 = oracle.nvfp4_quantize(local, global_scale=g)
        qm, sm = oracle.mxfp8_quantize(local)
        slowest = bench.reduce_max(float(10 + rank), world, torch.device("cpu"))
        q.put((rank, b, e, p, s, np.float32(g2), qm, sm, slowest))
    finally:
        dist.destroy_process_group()


def test_sharded_nvfp4_and_mxfp8_match_whole_tensor(orc):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=180) for _ in range(world)], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import workloads as W
    x = W.nvfp4_tensor(seed=71, M=37, N=256)
    pw, sw, gw = orc.nvfp4_quantize(x)
    qw, smw = orc.mxfp8_quantize(x)
    assert res[0][1] == 0 and res[0][2] == res[1][1] and res[1][2] == 37
    assert res[0][5] == gw and res[1][5] == gw             # same global scale on both ranks
    assert np.array_equal(np.concatenate([r[3] for r in res]), pw)
    assert np.array_equal(np.concatenate([r[4] for r in res]), sw)
    assert np.array_equal(np.concatenate([r[6] for r in res]), qw)
    assert np.array_equal(np.concatenate([r[7] for r in res]), smw)
    assert all(r[8] == 11.0 for r in res)                  # max over ranks


def test_shard_rows_partition():
    from nvfp4_block_scaled_sm_b200.distributed import shard_rows
    for M in (0, 1, 7, 37, 16384):
        for world in (1, 2, 3, 8):
            parts = [shard_rows(M, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == M
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [e - b for b, e in parts]
            assert max(sizes) - min(sizes) <= 1
