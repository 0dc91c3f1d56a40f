"""The N>1 bench path on CPU: two gloo ranks, each an independent replica,
take the max of their step times and count the work of both ranks."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 3.0 - rank, 5.0]          # rank 0: 10, 3; rank 1: 11, 2
        got = bench.reduce_max(local, dist, "cpu")
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == [11.0, 3.0, 5.0]
    assert out[1] == [11.0, 3.0, 5.0]


def test_whole_job_value_counts_every_rank():
    import bench
    # 2 ranks x 1e12 FLOP per step in 10 ms (slowest rank) = 2e14 FLOP/s
    assert bench.whole_job_value(1e12, 2, 10.0) == pytest.approx(2e14)
    assert bench.whole_job_value(1e12, 1, 10.0) == pytest.approx(1e14)


def test_reduce_max_without_group_is_identity():
    import bench
    assert bench.reduce_max([1.0, 2.0], None) == [1.0, 2.0]
