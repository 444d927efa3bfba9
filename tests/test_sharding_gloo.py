"""Multi-rank plumbing on CPU: two gloo ranks split units and reduce timings."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from compressed_kv_cache_convkv_b200.sharding import max_over_ranks, shard, sum_over_ranks


def test_shard_partitions_units():
    for units in (0, 1, 7, 40, 41):
        for world in (1, 2, 3, 8):
            got = [list(shard(units, world, r)) for r in range(world)]
            assert sum(got, []) == list(range(units))
            sizes = [len(g) for g in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = shard(40, world, rank)                      # heads owned by this rank
        owned = [None] * world
        dist.all_gather_object(owned, list(mine))
        elapsed = 10.0 + rank                              # per-rank device time (ms)
        q.put((rank, owned, max_over_ranks(elapsed, dist), sum_over_ranks(len(mine), dist)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_and_reduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, owned, mx, total in res:
        assert sum(owned, []) == list(range(40))           # every head owned exactly once
        assert mx == 11.0                                  # max over ranks
        assert total == 40.0
