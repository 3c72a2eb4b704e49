"""The multi-rank host logic on CPU: two gloo ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from kv_cache_compression_hkv_b200 import dist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = dist.max_over_ranks(10.0 + rank * 3.5)
        mine = list(dist.shard_sequences(64, world, rank))
        got = [None] * world
        torch.distributed.all_gather_object(got, mine)
        q.put((rank, mx, got, dist.rank_seed(7, rank)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seeds = set()
    for rank, mx, shards, seed in res:
        assert mx == 13.5  # max over both ranks
        flat = sorted(x for s in shards for x in s)
        assert flat == list(range(64))  # every sequence exactly once
        for s in shards:
            assert all(x % 2 == 0 for x in s[::2]) and len(s) % 2 == 0  # CFG pairs intact
        seeds.add(seed)
    assert len(seeds) == 2


def test_shard_sequences_edges():
    assert list(dist.shard_sequences(2, 1, 0)) == [0, 1]
    assert [len(dist.shard_sequences(16, 3, r)) for r in range(3)] == [4, 6, 6]
    assert list(dist.shard_sequences(5, 2, 1, cfg_pairs=False)) == [2, 3, 4]
    with pytest.raises(ValueError):
        dist.shard_sequences(5, 2, 0)
    with pytest.raises(ValueError):
        dist.shard_sequences(8, 2, 2)
    assert dist.max_over_ranks(3.0) == 3.0  # no process group
