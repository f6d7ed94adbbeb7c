"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

Each rank runs an independent shard of the workload (no data-path
collective); the only communication is the max-over-ranks timing.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from tiled_online_softmax_03_b200.inputs import WORKLOADS


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["single_head_128"]
        x = bench.rank_inputs(w, rank)
        # a fake per-rank step time: rank r "takes" 10 + r ms
        slowest = bench.max_over_ranks(10.0 + rank, world)
        digest = float(x["q"].float().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, digest)
        out[rank] = (slowest, gathered)
    finally:
        dist.destroy_process_group()


def test_two_ranks_independent_shards_and_max_timing():
    world = 2
    port = free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        slowest, digests = res[rank]
        assert slowest == 10.0 + world - 1
        assert len(set(digests)) == world  # each rank drew a different shard
    # aggregate throughput counts every rank's FLOP over the slowest time
    assert bench.whole_job_tflops(1e12, 2, 10.0) == pytest.approx(200.0)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    a = bench.rank_inputs(WORKLOADS["single_head_128"], 0)["q"]
    b = bench.rank_inputs(WORKLOADS["single_head_128"], 1)["q"]
    assert not torch.equal(a, b)
