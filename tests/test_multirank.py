"""Multi-rank host logic of the benchmark on CPU: two gloo ranks (127.0.0.1).

The hot path shards over batch items with no data-path exchange; the only
collectives are the barrier and the max-over-ranks reduction of timings.
These run here on `gloo`, world size 2, with the same calls bench.py makes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        local = [1.0 + rank, 10.0 - rank, 5.0 * (rank + 1)]
        got = bench.max_over_ranks(local, world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0, 10.0]


def test_job_throughput_weak_scaling():
    # 2 ranks each processing 1000 units, slowest rank 0.5 s -> 4000 units/s
    assert bench.job_throughput(1000, 2, 0.5) == 4000.0
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]


def test_attention_pair_count_closed_form():
    """The benchmark's algorithmic pair count equals brute-force enumeration."""
    import oracle
    for T, D, W in [(37, 4, 0), (50, 3, 5), (64, 64, 128), (40, 1, 0), (33, 5, 1)]:
        ref = sum(len(oracle.key_set(t, D, W)) for t in range(T))
        assert bench.attention_pairs(T, D, W) == ref, (T, D, W)
