"""The N > 1 host logic of bench.py on CPU: two gloo ranks.

Each rank runs its own replica on its own sequences; the job's time is the
slowest rank's (an all-reduce MAX, the only collective besides barriers),
and the job's throughput counts the units of every rank.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    os.environ["RANK"], os.environ["WORLD_SIZE"] = str(rank), str(world)
    os.environ["LOCAL_RANK"] = str(rank)
    import torch.distributed as dist

    import bench
    import workloads as wl
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        r, wsize, local = bench.rank_env()
        ms = bench.max_over_ranks([3.25, 5.5][rank], dist, "cpu")
        dist.barrier()
        # each rank's replica draws its own sequences
        w = wl.WORKLOADS["tiny"]
        q = bench.host_inputs(w, r)[0]
        queue.put((r, wsize, local, ms, float(np.asarray(q, dtype=np.float64).sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time():
    ctx = mp.get_context("spawn")
    queue = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(2, _free_port(), queue), nprocs=2, join=True,
                       start_method="spawn")
    got = sorted(queue.get() for _ in range(2))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 and g[2] == g[0] for g in got)
    assert all(g[3] == 5.5 for g in got)                 # both ranks see the max
    assert got[0][4] != got[1][4]                        # different sequences per rank


def test_job_rate_counts_every_rank():
    import bench
    # 2 ranks x 16,392 tokens per step x 10 steps in 20 ms
    assert bench.job_rate(2, 16392, 10, 20.0) == 2 * 16392 * 10 / 0.020
    assert bench.shard_seed(1001, 0) == 1001
    assert bench.shard_seed(1001, 1) != bench.shard_seed(1001, 0)
