"""The N > 1 host path of bench.py on CPU: two gloo ranks, token sharding and max-over-ranks timing.

The layer partitions by tokens (each rank its own batch, weights replicated, no
collective on the data path), so the only cross-rank step is the timing reduction.
"""
import os
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    rows = bench.rank_rows(rank, 16)
    t_ms = 10.0 + 5.0 * rank                     # rank 1 is the slower one
    slowest = bench.max_over_ranks(t_ms, dist, device="cpu")
    value = bench.job_throughput(16, world, 100, slowest)
    # every rank holds the same reduced value; gather the row sets to check the partition
    gathered = [None] * world
    dist.all_gather_object(gathered, rows.tolist())
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, slowest, value, gathered))


def test_two_gloo_ranks_shard_tokens_and_take_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value, gathered in out:
        assert slowest == 15.0                              # the max over ranks, seen by all
        assert abs(value - 16 * 2 * 100 / 15e-3) < 1e-6     # tokens of all ranks / slowest time
        allrows = np.concatenate([np.array(g) for g in gathered])
        assert np.array_equal(np.sort(allrows), np.arange(32))   # a partition of the global batch


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert list(bench.rank_rows(0, 4)) == [0, 1, 2, 3] and list(bench.rank_rows(2, 4)) == [8, 9, 10, 11]
    assert bench.job_throughput(16, 1, 10, 1.0) == 160000.0
