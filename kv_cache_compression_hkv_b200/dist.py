"""Multi-process plumbing for running the hot path on several GPUs.

Two ways to shard.  By sequence: sequences (and the CFG pair of each image)
are independent, so each rank owns whole sequences and the data path has no
exchange; the only collective is the timing reduction (max over ranks).  By
head: each rank holds some heads of every (sequence, layer); the heads are
independent except that a sequence's budgets count its Local heads on every
rank, so classification takes one exchange, a sum of the per-sequence Local
counts (S int32 per layer).  One process per GPU, torch.distributed for the
plumbing (NCCL on GPUs, gloo on CPU in tests).
"""
from __future__ import annotations

import torch


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own batch (weak scaling: every rank draws its own)."""
    return seed + 1000 * rank


def shard_sequences(num_seqs: int, world: int, rank: int, cfg_pairs: bool = True) -> range:
    """Contiguous range of the sequences a rank owns.  With cfg_pairs the
    conditional and unconditional halves of an image (sequences 2i, 2i+1)
    stay on one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    unit = 2 if cfg_pairs else 1
    if num_seqs % unit:
        raise ValueError("CFG pairs need an even number of sequences")
    n_units = num_seqs // unit
    lo = n_units * rank // world
    hi = n_units * (rank + 1) // world
    return range(lo * unit, hi * unit)


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank number over all ranks (1 rank: the number itself)."""
    if not torch.distributed.is_available() or not torch.distributed.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def shard_heads(num_heads: int, world: int, rank: int) -> range:
    """Contiguous, balanced range of the heads a rank holds."""
    if world < 1 or not 0 <= rank < world or num_heads < world:
        raise ValueError("bad rank/world or fewer heads than ranks")
    return range(num_heads * rank // world, num_heads * (rank + 1) // world)


def prefill_sharded(cache, layer: int, q, k, v, out=None, group=None):
    """Head-sharded prefill of one layer: grouping of the heads held here,
    a SUM all-reduce of each sequence's Local count over the ranks of
    `group`, then budgets from the total and the compression at
    classification.  Every rank calls it for the same layers in the same
    order.  Returns the summed counts (int32 [S])."""
    n = cache.prefill_label(layer, q, k, v, out=out)
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size(group) > 1:
        torch.distributed.all_reduce(n, op=torch.distributed.ReduceOp.SUM, group=group)
    cache.prefill_compress(layer, k, v, n)
    return n
