"""The gather-only diagnostic (include/mqa_logits_diag.h): it runs the FP8
path's data movement on any valid FP8 workload, raises no status bit and
writes nothing to `out`."""
import pytest
import torch

import paged_mqa_logits_b200 as mq
import workloads
from tests.helpers import to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,nn,H,D,ps,L,ctx", [
    (3, 2, 64, 128, 64, 700, [700, 0, 333]),
    (4, 1, 32, 64, 16, 520, [520, 17, 1, 256]),
    (2, 4, 16, 32, 256, 1200, [1200, 900]),
])
def test_gather_diag_moves_the_pages_and_writes_nothing(B, nn, H, D, ps, L, ctx):
    wl = workloads.make_workload("fp8", B, nn, H, D, ps, L, ctx, seed=4000 + D)
    dev = to_device(wl)
    sched = mq.mqa_logits_schedule(dev["ctx"])
    out = torch.full((B, nn, L), 7.0, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(3):
        mq.mqa_diag_fp8_gather(dev["q"], dev["kv"], dev["bt"], dev["ctx"], dev["w"], sched, out,
                               page_size=ps, out_len=L, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert bool(torch.all(out == 7.0))
