"""The multi-rank host logic of bench.py (replicas, one process per GPU) on two CPU ranks over
gloo: every rank ends with the slowest rank's times, and the job's tokens are the replicas'
sum."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        mine = [10.0 + rank, 5.0 - rank, 20.0 * (rank + 1)]  # per-rank step, decode, e2e ms
        got = bench.max_over_ranks(mine, world, "cpu")
        out[rank] = torch.tensor(got + [float(bench.job_tokens(16, world))], dtype=torch.float64)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_max_and_the_job_size():
    world = 2
    out = torch.zeros(world, 4, dtype=torch.float64).share_memory_()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        assert out[r].tolist() == [11.0, 5.0, 40.0, 32.0]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
    assert bench.job_tokens(16, 1) == 16
