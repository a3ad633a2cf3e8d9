"""Sharding across GPUs, one process per GPU.

Every logit depends on one batch row only (its q, weights and K pages), so a
batch shards by rows with no collective on the data path: each rank runs its
own schedule and logits kernel on its rows, and a caller that needs the full
[B, next_n, L] output gathers the shards afterwards. Across ranks only the
benchmark's timing (max over ranks) and token totals are reduced.

A very long row can instead be split by token range, each rank holding the K
pages of its range. Its logits then need no exchange either (each is one
token's), but its top-k does: every rank selects its own k best, the lists
are all-gathered (NCCL over NVLink) and merged into the row's top-k
(sharded_topk).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

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


def shard_tokens(length: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced token range [start, stop) of `rank` for a row of
    `length` tokens split by range (lower ranks hold lower tokens)."""
    return shard_rows(length, world, rank)


def sharded_topk(local_logits: torch.Tensor, local_valid: torch.Tensor, k: int,
                 token_offset: int, group=None, by_token: bool = False,
                 topk_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
    """Top-k of rows whose tokens are split by range over the ranks of `group`.

    local_logits: fp32 [rows, L_r], this rank's logits of tokens
    token_offset + t; local_valid: int32 [rows], how many of them are valid
    per row (a prefix). Ranks must hold ascending token ranges in rank order.
    Every rank returns the same int32 [rows, k] global tokens (and fp32
    values): the top-k over the whole rows, listed by value or by token.

    Steps: (1) the local top-k, by token, with values (mqa_logits_topk);
    (2) all-gather of the lists and of the ranks' token ranges; (3) the merge
    (mqa_logits_topk_merge). topk_fn / merge_fn replace (1) / (3), with the
    same signatures as those calls, where the kernels cannot run.
    """
    import paged_mqa_logits_b200 as mq

    dist = torch.distributed
    world = dist.get_world_size(group)
    if world > mq.MQA_TOPK_MERGE_MAX_SHARDS:
        raise ValueError(f"at most {mq.MQA_TOPK_MERGE_MAX_SHARDS} shards")
    if world * k > mq.MQA_TOPK_MERGE_MAX:
        raise ValueError(f"shards * k must be <= {mq.MQA_TOPK_MERGE_MAX}")
    topk_fn = topk_fn or mq.mqa_logits_topk
    merge_fn = merge_fn or mq.mqa_logits_topk_merge
    rows = int(local_logits.shape[0])
    idx, val = topk_fn(local_logits.reshape(rows, 1, -1).contiguous(), local_valid, k,
                       by_token=True, with_values=True)
    idx = idx.reshape(rows, k).contiguous()
    val = val.reshape(rows, k).contiguous()
    # flat buffers: rank r's list lands at [r * rows * k, (r + 1) * rows * k)
    all_idx = torch.empty(world * rows * k, dtype=idx.dtype, device=idx.device)
    all_val = torch.empty(world * rows * k, dtype=val.dtype, device=val.device)
    dist.all_gather_into_tensor(all_idx, idx.reshape(-1), group=group)
    dist.all_gather_into_tensor(all_val, val.reshape(-1), group=group)
    # each rank's token range: its offset and its length (the local row length)
    rng = torch.tensor([int(token_offset), int(local_logits.shape[1])], dtype=torch.int64,
                       device=idx.device)
    all_rng = torch.empty(2 * world, dtype=torch.int64, device=idx.device)
    dist.all_gather_into_tensor(all_rng, rng, group=group)
    pairs = all_rng.view(world, 2).cpu().tolist()
    offsets: List[int] = [int(p[0]) for p in pairs]
    counts: List[int] = [int(p[1]) for p in pairs]
    return merge_fn(all_val.view(world, rows, k), all_idx.view(world, rows, k), offsets, counts,
                    k, by_token=by_token, with_values=True)
