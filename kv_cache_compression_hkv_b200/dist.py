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


def shard_sequences(num_seqs: int, world: int, rank: int, pairing: int = 2) -> list[int]:
    """The sequences a rank owns, in the order its own batch should hold
    them.  The images are split into contiguous, balanced ranges, and both
    streams of an image (its conditional and unconditional sequence under
    classifier-free guidance) stay on one rank, laid out as the pairing
    says (the values of hkv_cfg_pairing):
      0 untied:   no pairs; a contiguous range of sequences;
      1 halves:   the batch is [conditional | unconditional], s pairs with
                  s + S/2; the rank gets images [lo, hi) as
                  [lo..hi) + [lo+S/2..hi+S/2), so its own batch is again
                  [conditional | unconditional] (pairing halves locally);
      2 adjacent: streams alternate, 2i pairs with 2i+1; the rank gets the
                  contiguous sequences [2 lo, 2 hi) (pairing adjacent
                  locally)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    if pairing not in (0, 1, 2):
        raise ValueError(f"unknown CFG pairing {pairing}")
    if pairing and num_seqs % 2:
        raise ValueError("CFG pairs need an even number of sequences")
    n_units = num_seqs // 2 if pairing else num_seqs
    lo = n_units * rank // world
    hi = n_units * (rank + 1) // world
    if pairing == 0:
        return list(range(lo, hi))
    if pairing == 2:
        return list(range(2 * lo, 2 * hi))
    half = num_seqs // 2
    return list(range(lo, hi)) + list(range(lo + half, hi + half))


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
