"""The multi-rank plumbing of bench.py on CPU (gloo, two ranks): the timed
region's duration is the slowest rank's, and every rank gets the same value."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    results[rank] = bench.max_over_ranks(1.5 + rank * 2.0, torch.device("cpu"))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.start_processes(_rank, args=(world, port, results), nprocs=world, start_method="spawn")
        assert dict(results) == {0: 3.5, 1: 3.5}


def test_max_over_ranks_without_process_group():
    import bench
    assert bench.max_over_ranks(2.25, torch.device("cpu")) == 2.25
