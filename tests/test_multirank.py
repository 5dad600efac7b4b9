"""The N > 1 bench plumbing on CPU: two gloo ranks, max-over-ranks timing
and distinct per-rank streams of blocks (replicas, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w = bench.dist_init("gloo")
    assert (r, w) == (rank, world)
    got = bench.reduce_max(10.0 + 5 * rank)
    bench.barrier()
    seeds = [None] * world
    dist.all_gather_object(seeds, bench.rank_seed(1100, rank))
    out[rank] = (got, tuple(seeds))
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_seeds():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    seeds = out[0][1]
    assert len(set(seeds)) == world and seeds == out[1][1]


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.dist_env()[1] >= 1
