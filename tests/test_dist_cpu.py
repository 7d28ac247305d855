"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each rank gets its own
batch element (distinct seeds, same shapes), timings reduce by max and work by sum."""
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
