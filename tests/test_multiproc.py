"""The N > 1 path on CPU: world-size-2 gloo ranks. Row shards need no
collective on the data path (the oracle over each rank's rows, gathered,
equals the oracle over the whole batch), and the benchmark's cross-rank
reduction is max of time, sum of tokens. Rows split by token range need one
exchange for their top-k: the sharded top-k's gather and offsets, run with
CPU stand-ins for the two kernels, give the oracle's top-k of the whole
rows."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from paged_mqa_logits_b200.shard import reduce_max_sum, shard_rows, shard_tokens, sharded_topk


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import oracle
    import workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = workloads.make_workload("fp8", 5, 2, 8, 32, 16, 100, [100, 0, 37, 64, 1], seed=3)
        lo, hi = shard_rows(wl.B, world, rank)
        sub = workloads.Workload(**{**wl.__dict__, "B": hi - lo, "q": wl.q[lo:hi].contiguous(),
                                    "block_table": wl.block_table[lo:hi].contiguous(),
                                    "context_lens": wl.context_lens[lo:hi].contiguous(),
                                    "weights": wl.weights[lo:hi].contiguous()})
        out, _ = oracle.logits(sub, with_absw=False)
        parts = [None] * world
        dist.all_gather_object(parts, out)
        ms, tok = reduce_max_sum(1.5 + rank, 10.0 * (rank + 1))
        if rank == 0:
            full, _ = oracle.logits(wl, with_absw=False)
            q.put((np.array_equal(np.concatenate(parts, axis=0), full), ms, tok))
    finally:
        dist.destroy_process_group()


def test_shard_rows_partition():
    for B in (0, 1, 5, 64, 2049):
        for world in (1, 2, 3, 8):
            ranges = [shard_rows(B, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == B
            assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_shard_without_data_collective():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    same, ms, tok = q.get(timeout=10)
    assert same
    assert ms == 2.5 and tok == 30.0


def _cpu_topk(logits, valid, k, by_token=False, with_values=False):
    """Stand-in for mqa_logits_topk on CPU tensors: the oracle's selection,
    plus the selected logits (-inf for -1)."""
    import oracle
    lg = logits.numpy()
    idx = oracle.topk(lg, valid.numpy().astype(np.int32), lg.shape[1], k, by_token)
    val = np.where(idx >= 0, np.take_along_axis(lg, np.maximum(idx, 0), axis=2), -np.inf)
    return torch.from_numpy(idx), torch.from_numpy(val.astype(np.float32))


def _cpu_merge(cand_values, cand_tokens, offsets, counts, k, by_token=False, with_values=False):
    """Stand-in for mqa_logits_topk_merge: (value desc, global token asc) over
    the shards' valid entries; the ranges must ascend without overlap."""
    S, rows, _ = cand_tokens.shape
    assert all(offsets[s] + counts[s] <= offsets[s + 1] for s in range(S - 1))
    idx = np.full((rows, k), -1, np.int32)
    val = np.full((rows, k), -np.inf, np.float32)
    for r in range(rows):
        c = [(float(cand_values[s, r, j]), int(cand_tokens[s, r, j]) + offsets[s])
             for s in range(S) for j in range(cand_tokens.shape[2]) if cand_tokens[s, r, j] >= 0]
        c = sorted(c, key=lambda e: (-e[0], e[1]))[:k]
        if by_token:
            c = sorted(c, key=lambda e: e[1])
        for i, (v, t) in enumerate(c):
            idx[r, i], val[r, i] = t, v
    return torch.from_numpy(idx), torch.from_numpy(val)


def _topk_worker(rank, world, port, q):
    import datetime
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(9)
        rows, L, k = 5, 301, 40
        full = rng.choice(np.array([-1.0, 0.5, 2.0, 3.0], np.float32), size=(rows, L))
        full[1] = rng.standard_normal(L).astype(np.float32)
        valid = np.array([301, 150, 151, 7, 0], np.int32)
        lo, hi = shard_tokens(L, world, rank)
        local = torch.from_numpy(np.ascontiguousarray(full[:, lo:hi]))
        lvalid = torch.from_numpy(np.clip(valid - lo, 0, hi - lo).astype(np.int32))
        ok = True
        for by_token in (False, True):
            idx, val = sharded_topk(local, lvalid, k, lo, by_token=by_token,
                                    topk_fn=_cpu_topk, merge_fn=_cpu_merge)
            want = oracle.topk(full[:, None, :], valid, 1, k, by_token)[:, 0, :]
            ok = ok and np.array_equal(idx.numpy(), want)
            got_v = np.where(want >= 0, np.take_along_axis(full, np.maximum(want, 0), 1), -np.inf)
            ok = ok and np.array_equal(val.numpy(), got_v.astype(np.float32))
        flags = [None] * world
        dist.all_gather_object(flags, ok)
        if rank == 0:
            q.put(all(flags))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_topk_exchange_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_topk_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=5)
