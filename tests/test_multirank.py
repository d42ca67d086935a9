"""Multi-rank host logic of the benchmark on CPU: two gloo ranks (127.0.0.1).

The hot path shards over batch items with no data-path exchange; the only
collectives are the barrier and the max-over-ranks reduction of timings.
These run here on `gloo`, world size 2, with the same calls bench.py makes.
"""
import os
import socket

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


def test_decode_bytes_per_step_matches_key_sets():
    """The decode roofline's algorithmic bytes: every attended cached row once
    (the oracle's key set minus the token itself), K and V, plus the state,
    the step's inputs and output, the ring write and the dilated append."""
    import oracle
    from recurrence_augmented_dilated_chunked_b200 import Workload
    for D, W, dense in [(4, 0, ()), (4, 8, ()), (3, 5, (0,)), (64, 128, (1,)), (1, 0, ())]:
        H, Dh, B = 2, 128, 3
        w = Workload("t", "bf16", B=B, T=0, H=H, Dh=Dh, D=D, W=W, gate_mean=0.0, gate_std=1.0,
                     dense_heads=dense)
        for t in [0, 1, 5, 63, 64, 200, 777]:
            ref = 0
            for h in range(H):
                Dd = 1 if h in dense else D
                rows = len(oracle.key_set(t, Dd, 0 if Dd == 1 else W)) - 1
                per = rows * 2 * Dh * 2 + 2 * Dh * 4 * 2 + 4 * Dh * 2 + Dh * 2
                per += 2 * Dh * 2 if W > 0 else 0
                per += 2 * Dh * 2 if t % Dd == Dd - 1 else 0
                ref += B * per
            assert bench.decode_bytes_per_step(w, t) == ref, (D, W, dense, t)


def test_prefill_pair_count_with_dense_heads():
    import oracle
    from recurrence_augmented_dilated_chunked_b200 import Workload
    w = Workload("t", "bf16", B=2, T=45, H=3, Dh=128, D=4, W=6, gate_mean=0.0, gate_std=1.0,
                 dense_heads=(1,))
    ref = 0
    for h in range(3):
        Dd = 1 if h == 1 else 4
        ref += 2 * sum(len(oracle.key_set(t, Dd, 0 if Dd == 1 else 6)) for t in range(45))
    c = bench.prefill_counts(w)
    assert c["pairs"] == ref
    assert c["attn_flops"] == 4 * 128 * ref
    assert c["scan_bytes"] == 5 * 2 * 45 * 3 * 128 * 2
