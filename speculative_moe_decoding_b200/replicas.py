"""Multi-GPU use of the decode step: independent replicas.

The step is a strict chain of dependent passes at batch 1, so it does not
shard; N GPUs run N independent sequences.  The only cross-rank traffic is the
timing reduction here: whole-job tokens/s = (tokens summed over ranks) / (the
slowest rank's timed region).
"""
from __future__ import annotations

from typing import List, Tuple


def shard_sequences(n_sequences: int, rank: int, world: int) -> List[int]:
    """Sequence indices handled by `rank` (round robin)."""
    return list(range(rank, n_sequences, world))


def replica_throughput(tokens: float, ms: float, device=None) -> Tuple[float, float, float]:
    """Returns (tokens/s of the whole job, max ms over ranks, total tokens)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return tokens / (ms / 1000.0), ms, tokens
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    n = torch.tensor([tokens], dtype=torch.float64, device=device)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(n.item()) / (float(t.item()) / 1000.0), float(t.item()), float(n.item())
