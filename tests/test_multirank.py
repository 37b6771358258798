"""The N>1 path of bench.py on CPU: two gloo ranks run independent replicas; the
reported time is the max over ranks and the value counts the work of every rank."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank-dependent fake timings: rank 1 is the slow one for the first value
        mine = [10.0 + 5.0 * rank, 3.0 - rank, 7.0]
        got = bench.max_over_ranks(mine)
        value = bench.whole_job_tflops(world, 2e12, got[0] / 1e3)
        out[rank] = (got, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        got, value = out[r]
        assert got == [15.0, 3.0, 7.0]
        assert value == pytest.approx(2 * 2e12 / 0.015 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.0]) == [1.5, 2.0]
    assert bench.whole_job_tflops(1, 1e12, 0.5) == pytest.approx(2.0)
