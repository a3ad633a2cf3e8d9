"""CUDA-graph capture of the whole path (the page's section 2: the schedule
is computed on the GPU so the call can be captured), and the schedule reuse
rule (valid while every ceil(ctx/256) is unchanged)."""
import numpy as np
import pytest
import torch

import oracle
import paged_mqa_logits_b200 as mq
import workloads
from tests.helpers import compare, to_device

pytestmark = pytest.mark.gpu


def _wl():
    # pages reserved for the longer lengths the tests switch to
    return workloads.make_workload("fp8", 4, 2, 64, 128, 64, 1536, [1000, 0, 513, 1400], seed=77,
                                   reserve_lens=[1024, 300, 640, 1536])


def test_graph_replay_matches_eager_and_follows_new_lengths():
    wl = _wl()
    d = to_device(wl)
    S = mq.mqa_logits_num_ctas()
    sched = torch.empty(S + 1, 2, dtype=torch.int32, device="cuda")
    out = torch.empty(wl.B, wl.next_n, wl.out_len, dtype=torch.float32, device="cuda")

    def step():
        mq.mqa_logits_schedule(d["ctx"], S, sched)
        mq.paged_mqa_logits_fp8(d["q"], d["kv"], d["bt"], d["ctx"], d["w"], sched, out,
                                page_size=wl.page_size)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step()
    s.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)

    # new lengths, some across a 256-token boundary: the graph re-runs the schedule
    new_ctx = torch.tensor([1010, 300, 200, 1536], dtype=torch.int32)
    d["ctx"].copy_(new_ctx)
    g.replay()
    torch.cuda.synchronize()
    wl2 = workloads.Workload(**{**wl.__dict__, "context_lens": new_ctx})
    ref, absw = oracle.logits(wl2)
    compare(out.cpu().numpy(), ref, absw)
    assert np.array_equal(sched.cpu().numpy(), oracle.schedule(new_ctx, S))


def test_schedule_reuse_within_unit_boundaries():
    """A schedule built for lengths L stays correct for L' whenever
    ceil(L'/256) == ceil(L/256) for every row."""
    wl = _wl()
    d = to_device(wl)
    sched = mq.mqa_logits_schedule(d["ctx"])
    new_ctx = torch.tensor([1020, 0, 600, 1300], dtype=torch.int32)  # same unit counts
    assert torch.equal((new_ctx + 255) // 256, (wl.context_lens + 255) // 256)
    d["ctx"].copy_(new_ctx)
    out = mq.paged_mqa_logits_fp8(d["q"], d["kv"], d["bt"], d["ctx"], d["w"], sched,
                                  page_size=wl.page_size, out_len=wl.out_len)
    torch.cuda.synchronize()
    wl2 = workloads.Workload(**{**wl.__dict__, "context_lens": new_ctx})
    ref, absw = oracle.logits(wl2)
    compare(out.cpu().numpy(), ref, absw)
