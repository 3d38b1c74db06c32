"""The multi-rank host logic of the benchmark on CPU: two gloo ranks.

With N GPUs the benchmark runs one independent replica of the workload per
rank (no collective on the data path); the timed region's length is the
maximum over ranks, and the whole-job rate counts every rank's units.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r pretends its timed region took (r + 1) * 10 ms
        t = bench.max_over_ranks(10.0 * (rank + 1), world, "cpu")
        v = bench.aggregate_rate(1000.0, 5, world, t)
        out[rank] = (t, v)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        t, v = out[r]
        assert t == pytest.approx(20.0)
        # 2 ranks x 1000 units x 5 steps over 20 ms
        assert v == pytest.approx(2 * 1000 * 5 / 0.020)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_rate(10.0, 4, 1, 2.0) == pytest.approx(10 * 4 / 0.002)
