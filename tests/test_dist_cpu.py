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
        mine = dist.shard_sequences(64, world, rank)
        halves = dist.shard_sequences(64, world, rank, pairing=1)
        got = [None] * world
        torch.distributed.all_gather_object(got, (mine, halves))
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
        for which in range(2):
            flat = sorted(x for s in shards for x in s[which])
            assert flat == list(range(64))  # every sequence exactly once
        for adj, halves in shards:
            assert all(x % 2 == 0 for x in adj[::2]) and len(adj) % 2 == 0  # pairs intact
            n = len(halves) // 2
            assert all(halves[j] + 32 == halves[j + n] for j in range(n))
        seeds.add(seed)
    assert len(seeds) == 2


def test_shard_sequences_edges():
    assert dist.shard_sequences(2, 1, 0) == [0, 1]
    assert [len(dist.shard_sequences(16, 3, r)) for r in range(3)] == [4, 6, 6]
    assert dist.shard_sequences(5, 2, 1, pairing=0) == [2, 3, 4]
    with pytest.raises(ValueError):
        dist.shard_sequences(5, 2, 0)
    with pytest.raises(ValueError):
        dist.shard_sequences(8, 2, 2)
    with pytest.raises(ValueError):
        dist.shard_sequences(8, 2, 0, pairing=3)
    assert dist.max_over_ranks(3.0) == 3.0  # no process group


@pytest.mark.parametrize("S,world", [(16, 3), (64, 2), (2, 1), (32, 8), (10, 4)])
def test_shard_sequences_keep_cfg_halves_together(S, world):
    """A [conditional | unconditional] batch (s pairs with s + S/2, the
    library's HKV_CFG_HALVES): every pair lands on one rank, and the rank's
    own batch is again [conditional | unconditional], so a context made
    for it with the same pairing ties the same two streams."""
    from oracle import hkv_oracle as O
    owner = {}
    for r in range(world):
        mine = dist.shard_sequences(S, world, r, pairing=1)
        n = len(mine)
        assert n % 2 == 0
        for j, s in enumerate(mine):
            owner[s] = r
            # local partner under the same pairing is the global partner
            jp = O.cfg_partner(j, n, O.CFG_HALVES)
            assert mine[jp] == O.cfg_partner(s, S, O.CFG_HALVES)
    assert sorted(owner) == list(range(S))
    assert all(owner[s] == owner[O.cfg_partner(s, S, O.CFG_HALVES)] for s in range(S))
    for r in range(world):  # adjacent pairing: 2i and 2i+1 together, locally adjacent
        mine = dist.shard_sequences(S, world, r, pairing=2)
        assert all(mine[j] ^ 1 == mine[j ^ 1] for j in range(len(mine)))


class _ShardCache:
    """Stands in for a head-sharded HeadKVCache on CPU: its grouping of the
    heads held here comes from the oracle; it records the calls it gets."""

    def __init__(self, labels_here):
        self.labels_here = labels_here  # [S, heads here], 1 = Local
        self.calls, self.total, self.here = [], None, None

    def prefill_label(self, layer, q, k, v, out=None):
        self.calls.append(("label", layer))
        self.here = torch.tensor((self.labels_here == 1).sum(1), dtype=torch.int32)
        return self.here.clone()

    def prefill_compress(self, layer, k, v, n_local_total):
        self.calls.append(("compress", layer))
        self.total = n_local_total.clone()


def _oracle_labels(seed):
    """[S, H] labels of the llamagen_xl-shaped first layer, 2 sequences."""
    import numpy as np

    from kv_cache_compression_hkv_b200.inputs import WORKLOADS, generate_layer
    from oracle import hkv_oracle as O
    w = WORKLOADS["llamagen_xl"]
    P = w.prefill_len
    q, k, v = (x.double().numpy() for x in generate_layer(w, 0, seed, "cpu", num_seqs=2,
                                                            max_len=P))
    lab = np.zeros((2, w.num_heads), np.uint8)
    for s in range(2):
        for h in range(w.num_heads):
            row = O.class_row(q[s, h], k[s, h], v[s, h], 1)
            lab[s, h] = O.classify(row, w.local_window, 0.9)[1]
    return lab


def _head_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lab = _oracle_labels(seed=3)
        hs = dist.shard_heads(lab.shape[1], world, rank)
        cache = _ShardCache(lab[:, hs.start:hs.stop])
        n = dist.prefill_sharded(cache, 0, None, None, None)
        q.put((rank, list(hs), n.tolist(), (lab == 1).sum(1).tolist(), cache.calls,
               cache.total.tolist(), cache.here.tolist()))
    finally:
        torch.distributed.destroy_process_group()


def test_head_sharded_local_counts_two_gloo_ranks():
    """Each rank groups its own heads; after the all-reduce both ranks hold
    every sequence's Local count over all heads, as one process would."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_head_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    heads = sorted(h for r in res for h in r[1])
    assert heads == list(range(20))  # every head on exactly one rank
    for rank, hs, n, full, calls, total, here in res:
        assert n == full and total == full
        assert calls == [("label", 0), ("compress", 0)]
    full = res[0][3]
    assert [a + b for a, b in zip(res[0][6], res[1][6])] == full
    assert any(r[6] != full for r in res)  # no rank alone knew the totals


def test_shard_heads_edges():
    assert [list(dist.shard_heads(20, 2, r)) for r in range(2)] == [list(range(10)),
                                                                   list(range(10, 20))]
    assert [len(dist.shard_heads(32, 3, r)) for r in range(3)] == [10, 11, 11]
    with pytest.raises(ValueError):
        dist.shard_heads(2, 3, 0)
    with pytest.raises(ValueError):
        dist.shard_heads(8, 2, 2)
    # one rank: the helper is the two phases back to back with its own counts
    c = _ShardCache(torch.tensor([[1, 0, 1], [0, 0, 0]]).numpy())
    assert dist.prefill_sharded(c, 4, None, None, None).tolist() == [2, 0]
    assert c.calls == [("label", 4), ("compress", 4)] and c.total.tolist() == [2, 0]
