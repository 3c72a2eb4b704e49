"""Multi-process plumbing for running the hot path on several GPUs.

The path shards without any data-path exchange: sequences (and the CFG pair
of each image) are independent, so each rank owns whole sequences.  The only
collective is the timing reduction (max over ranks).  One process per GPU,
torch.distributed for the plumbing (NCCL on GPUs, gloo on CPU in tests).
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
