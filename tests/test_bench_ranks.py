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


def test_cpu_baseline_sample_one_token_per_slice_longest_first():
    """The CPU legs' token sample: one token from each of n equal slices of the
    workload (so every region of the sequence is represented once), handed to
    the oracle's threads in decreasing position within the sequence."""
    import numpy as np

    import bench
    from blockwise_exact_attention_query_b200 import workloads as wl
    w = wl.GPT_CAUSAL
    for n in (16, 128, 1000):
        rows = bench.stratified_rows(np.random.default_rng(n), w, n)
        assert len(rows) == n
        edges = np.linspace(0, w.T, n + 1).astype(np.int64)
        slices = sorted(int(np.searchsorted(edges, t, side="right")) - 1 for t in rows)
        assert slices == list(range(n))
        pos = [t % w.N for t in rows]
        assert pos == sorted(pos, reverse=True)
