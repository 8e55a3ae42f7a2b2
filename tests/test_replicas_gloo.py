"""The multi-GPU path of bench.py is replicas only: each rank runs its own copy of the
layer and the job's throughput is all ranks' tokens over the slowest rank's time.
Checked here with two gloo ranks on the CPU (no GPU, no NCCL)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]                      # rank 1 is the slow replica
        got = bench.max_over_ranks_dist(ms, world, "cpu")
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        assert dict(out) == {0: 20.0, 1: 20.0}


def test_replica_throughput_counts_all_ranks_over_slowest():
    # 2 ranks x 128 tokens x 10 steps in 20 ms (the slowest rank) -> 128000 tokens/s
    assert bench.replica_throughput(128, 2, 20.0, 10) == pytest.approx(128000.0)
    assert bench.replica_throughput(128, 1, 20.0, 10) == pytest.approx(64000.0)
