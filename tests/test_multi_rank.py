"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo. Every rank
runs an independent replica; the job time is the slowest rank's and the
throughput counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        mine = 10.0 + 5.0 * rank              # rank 1 is the slow one
        m = bench.max_over_ranks(mine, dist, "cpu")
        thr = bench.job_throughput(2048, world, 4, m)
        dist.barrier()
        out[rank] = (m, thr)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput(repo_root):
    os.environ.setdefault("PYTHONPATH", repo_root)
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for rank in (0, 1):
        m, thr = out[rank]
        assert m == 15.0
        assert thr == pytest.approx(2048 * 2 * 4 / 0.015)


def test_single_rank_without_process_group():
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(100, 1, 10, 1000.0) == pytest.approx(1000.0)
