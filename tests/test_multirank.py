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


class _OracleShardCache:
    """Stands in for a cache that holds heads [lo, hi) of a layer: its
    scores-only selection is the oracle's partial score over those heads, and
    its given-score routing records the oracle's top-k of the scores it gets."""

    def __init__(self, Q, pool_K, lo, hi, n_top):
        self.Q, self.pool_K, self.lo, self.hi, self.n_top = Q, pool_K, lo, hi, n_top
        self.routed = None

    def select_mid_ex(self, layer, Q, policy, heads_total=0, scores_in=None, scores_out=None):
        import oracle
        if policy == 1:                                   # scores only, this rank's heads
            part = oracle.select_scores(self.Q[..., self.lo:self.hi, :], self.pool_K[..., self.lo:self.hi, :],
                                        heads_norm=heads_total)
            scores_out.copy_(torch.from_numpy(part))
        elif policy == 2:                                 # top-k of the given scores
            self.routed = oracle.select_topk(scores_in.numpy(), self.n_top)
        else:
            raise AssertionError(policy)


def _bench_shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import synth
    bench.dist_init("gloo")
    wl = synth.WORKLOADS["ragged_c"]                      # 3 heads over the ranks: 2 + 1
    d = synth.make_layer(wl.replace(pool_blocks=6, planted=2), 21)   # the same layer on every rank
    H = d["Q"].shape[2]
    lo, hi = bench.head_shard(H, world, rank)
    cache = _OracleShardCache(d["Q"], d["mid_K"], lo, hi, 2)
    scores = torch.zeros((wl.batch, 6), dtype=torch.float64)
    bench.select_head_sharded(cache, 0, d["Q"], scores, H, lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM),
                              1, 2)
    out[rank] = ((lo, hi), scores.numpy().tolist(), cache.routed.tolist())
    dist.destroy_process_group()


def test_bench_head_sharded_selection_on_two_gloo_ranks():
    # the bench's own sharded-selection step (scores-only on this rank's heads,
    # the sum across ranks, the top-k of the sum) against the unsharded oracle
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_bench_shard_worker, args=(world, port, out), nprocs=world, join=True)
    import numpy as np

    import oracle
    import synth
    d = synth.make_layer(synth.WORKLOADS["ragged_c"].replace(pool_blocks=6, planted=2), 21)
    full = oracle.select_scores(d["Q"], d["mid_K"])
    assert out[0][0] == (0, 2) and out[1][0] == (2, 3)
    for r in range(world):
        assert np.max(np.abs(np.array(out[r][1]) - full)) < 1e-12 * max(1.0, np.max(np.abs(full)))
        assert np.array_equal(np.array(out[r][2]), oracle.select_topk(full, 2))


def test_head_shard_ranges_cover_every_head_once():
    import bench
    for H in (1, 3, 12, 16):
        for world in range(1, H + 1):
            r = [bench.head_shard(H, world, k) for k in range(world)]
            assert r[0][0] == 0 and r[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [hi - lo for lo, hi in r]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
