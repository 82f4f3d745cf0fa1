"""The multi-rank timing of bench.py on two gloo ranks (CPU): the slowest rank's time
decides, and the whole-job value counts every rank's steps (weak scaling)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 100.0 + 50.0 * rank          # rank 1 is the slow one
    ms = bench.rank_max(local_ms, world)
    out[rank] = (ms, bench.throughput(20, world, ms))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_value():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, value = res[rank]
        assert ms == pytest.approx(150.0)
        assert value == pytest.approx(20 * 2 / 0.150)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.rank_max(3.0, 1) == 3.0
    assert bench.throughput(10, 1, 500.0) == pytest.approx(20.0)
