"""Multi-rank host logic on CPU (gloo, world size 2).

* The benchmark's batch split: each rank gets its own batch element (distinct seeds, same
  shapes); timings reduce by max and work by sum.
* The head split of one layer: head ranges partition the heads contiguously, and each
  rank's heads (its Q/K/V slice and its rows of a per-head mask) computed on its own give
  the whole layer when gathered -- with the oracle as the compute, so the arithmetic of the
  split is checked without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    w = bench._workload_for_rank(rank)
    times, work = bench.reduce_over_ranks([10.0 + rank, 5.0 * (2 - rank)], 100.0 * (rank + 1), "cpu", True)
    # The data path has no collective: a rank's inputs depend only on its own seed.
    q, _, _ = bench.make_qkv(bench.Workload(**{**w.__dict__, "H": 1, "T": 1}), heads=[0])
    gathered = [torch.zeros_like(q[0, 0, :4, :4].float()) for _ in range(world)]
    dist.all_gather(gathered, q[0, 0, :4, :4].float())
    out[rank] = (w.seed, times, work, not torch.equal(gathered[0], gathered[1]))
    dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    # the manager process is spawned too: forking a process that already runs threads
    # (torch's pools, earlier tests) can deadlock the child
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    seeds = {r: res[r][0] for r in res}
    assert seeds[0] != seeds[1]
    for r in res:
        _, times, work, differ = res[r]
        assert times == [11.0, 10.0]          # max over ranks, per entry
        assert work == 300.0                   # summed work
        assert differ                          # distinct per-rank inputs


def test_head_ranges_partition_the_heads():
    from block_sparse_attention_lva_b200.sharding import head_range
    for H in (1, 2, 3, 7, 12, 40):
        for world in (1, 2, 3, 4, 8, 16):
            ranges = [head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0                                  # contiguous, in rank order
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and sum(sizes) == H


def _shard_worker(rank, world, port, out):
    """Each rank computes its head range of one tiny layer with the oracle (the arithmetic of
    the shard: head range, per-head mask rows, head slices of Q/K/V) and gathers to rank 0."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np
    from block_sparse_attention_lva_b200.sharding import head_range, shard_rows
    from oracle.attention import attention_blocked
    from synthetic import Workload, make_qkv
    w = Workload("shard", B=1, H=5, d=64, T=2, Hg=8, Wg=16, tile=(1, 4, 8), block_size=64, seed=77)
    masks = np.random.default_rng(5).random((w.H, w.nb, w.nb)) < 0.5        # per-head static mask
    h0, h1 = head_range(w.H, world, rank)
    q, k, v = make_qkv(w, heads=range(h0, h1))                              # this rank's heads only
    o, lse = attention_blocked(q, k, v, shard_rows(masks, h0, h1), w.block_size, w.n_valid, w.scale)
    parts = [None] * world
    dist.all_gather_object(parts, (h0, h1, o, lse))
    if rank == 0:
        qa, ka, va = make_qkv(w)
        o_ref, lse_ref = attention_blocked(qa, ka, va, masks, w.block_size, w.n_valid, w.scale)
        o_cat = np.concatenate([p[2] for p in parts], axis=1)
        lse_cat = np.concatenate([p[3] for p in parts], axis=1)
        out["ranges"] = [(p[0], p[1]) for p in parts]
        out["o_equal"] = bool(np.array_equal(o_cat, o_ref))
        out["lse_equal"] = bool(np.array_equal(lse_cat, lse_ref))
    dist.destroy_process_group()


def test_two_ranks_head_shards_make_the_whole_layer():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res["ranges"] == [(0, 3), (3, 5)]
    assert res["o_equal"] and res["lse_equal"]
