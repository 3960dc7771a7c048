"""bench.py's multi-rank plumbing on CPU: two gloo ranks take the max of their
measured times and compute the whole-job throughput the way the GPU run does."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        ms = 100.0 + 50.0 * rank                # rank 1 is the slowest
        mx = bench.max_over_ranks(ms, world, device="cpu")
        out[rank] = (mx, bench.aggregate(200, world, mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        mx, value = out[r]
        assert mx == 150.0
        assert value == pytest.approx(200 * 2 / 0.150)


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate(10, 1, 1000.0) == pytest.approx(10.0)
