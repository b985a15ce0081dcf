"""The multi-rank path of bench.py on CPU: two gloo ranks, the barrier and the max-over-ranks timing
that bench.py uses (each rank runs an independent replica; no data-path collective exists)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    dist = bench.init_dist(w, "gloo")
    dev = torch.device("cpu")
    bench.barrier(dist, dev)
    local_ms = 10.0 + 5.0 * rank              # per-rank device time of the timed region
    out[rank] = bench.max_over_ranks(local_ms, dist, dev)
    bench.barrier(dist, dev)
    dist.destroy_process_group()


def test_two_rank_max_over_ranks():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork of this (multi-threaded) process
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == out[1] == 15.0


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
