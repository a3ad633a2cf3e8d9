"""Row sharding across GPUs, one process per GPU.

Every logit depends on one batch row only (its q, weights and K pages), so a
batch shards by rows with no collective on the data path: each rank runs its
own schedule and logits kernel on its rows, and a caller that needs the full
[B, next_n, L] output gathers the shards afterwards. Across ranks only the
benchmark's timing (max over ranks) and token totals are reduced.
"""
from __future__ import annotations

from typing import Tuple

import torch


def shard_rows(batch: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced row range [start, stop) of `rank` out of `world`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, rem = divmod(batch, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


def reduce_max_sum(elapsed_ms: float, tokens: float, device=None) -> Tuple[float, float]:
    """(max over ranks of elapsed_ms, sum over ranks of tokens). A no-op
    without an initialised process group."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(elapsed_ms), float(tokens)
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    n = torch.tensor([tokens], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(n, op=torch.distributed.ReduceOp.SUM)
    return float(t[0]), float(n[0])
