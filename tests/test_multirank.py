"""The N > 1 plumbing on CPU: two gloo ranks, max-over-ranks timing and
distinct per-rank streams of blocks (replicas, no data-path collective);
and the one exchange a head-sharded selection needs (partial block scores
of each rank's heads, summed across ranks before the top-k)."""
import os
import socket

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
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    seeds = out[0][1]
    assert len(set(seeds)) == world and seeds == out[1][1]


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.dist_env()[1] >= 1


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np

    import oracle
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = synth.WORKLOADS["ragged_c"]
    d = synth.make_layer(wl.replace(pool_blocks=6, planted=2), 21)   # the same inputs on every rank
    H = d["Q"].shape[2]
    per = (H + world - 1) // world
    lo, hi = rank * per, min(H, (rank + 1) * per)
    # this rank's heads only, divided by the total head count
    part = oracle.select_scores(d["Q"], d["mid_K"], heads=(lo, hi), heads_norm=H)
    t = torch.from_numpy(part.copy())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    out[rank] = (t.numpy().tolist(), oracle.select_topk(t.numpy(), 2).tolist(),
                 oracle.select_scores(d["Q"], d["mid_K"]).tolist())
    dist.destroy_process_group()


def test_head_sharded_selection_exchange_on_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    import numpy as np

    import oracle
    summed0, sel0, full = (np.array(x) for x in out[0])
    summed1, sel1, _ = (np.array(x) for x in out[1])
    assert np.array_equal(summed0, summed1) and np.array_equal(sel0, sel1)
    assert np.max(np.abs(summed0 - full)) < 1e-12 * max(1.0, np.max(np.abs(full)))
    assert np.array_equal(sel0, oracle.select_topk(full, 2))
