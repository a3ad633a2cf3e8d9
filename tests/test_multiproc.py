"""The N > 1 path on CPU: world-size-2 gloo ranks. Row shards need no
collective on the data path (the oracle over each rank's rows, gathered,
equals the oracle over the whole batch), and the benchmark's cross-rank
reduction is max of time, sum of tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from paged_mqa_logits_b200.shard import reduce_max_sum, shard_rows


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
