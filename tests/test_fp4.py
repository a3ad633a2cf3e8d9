"""FP4 path parity against the fp64 oracle (e2m1 K with e4m3 block scales,
bf16 q). Same bar as FP8: tolerance per element, masking bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.helpers import compare, run

pytestmark = pytest.mark.gpu

CASES = [
    ("B3-H32-D128-ps64", 3, 1, 32, 128, 64, 1100, [1100, 0, 513]),
    ("B3-nn2-H64-D128", 3, 2, 64, 128, 64, 640, [640, 130, 1]),
    ("B2-nn4-H32-D128-ps16", 2, 4, 32, 128, 16, 400, [397, 3]),
    ("B3-H128-D128-ps128", 3, 1, 128, 128, 128, 800, [800, 128, 129]),
    ("B4-H4-D64-ps16", 4, 1, 4, 64, 16, 300, [300, 17, 0, 256]),
    ("B3-nn2-H16-D64-ps256", 3, 2, 16, 64, 256, 900, [899, 512, 255]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fp4_mid_sizes_full(case):
    _, B, nn, H, D, ps, L, ctx = case
    wl = workloads.make_workload("fp4", B, nn, H, D, ps, L, ctx, seed=2000 + CASES.index(case))
    out, _ = run(wl)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl)
    compare(out.cpu().numpy(), ref, absw)


def test_fp4_config_every_element():
    """The FP4 workload at full size: every element against the oracle."""
    wl = workloads.make_config("fp4")
    out, _ = run(wl)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl, threads=None)
    compare(out.cpu().numpy(), ref, absw)


def test_fp4_q_outside_f16_range():
    """q rows whose magnitudes are far outside f16's range (1e-8 .. 1e8) are
    still scored correctly: the per-row power-of-two scale keeps the f16
    conversion exact."""
    wl = workloads.make_workload("fp4", 3, 1, 32, 128, 64, 520, [520, 300, 129], seed=2100)
    q = wl.q.view(torch.bfloat16).float()
    q[0] *= 1e8
    q[1] *= 1e-8
    wl.q = q.to(torch.bfloat16).view(torch.int16).contiguous()
    out, _ = run(wl)
    ref, absw = oracle.logits(wl)
    compare(out.cpu().numpy(), ref, absw)


def test_fp4_page_size_bitwise():
    wl = workloads.make_workload("fp4", 3, 2, 32, 128, 64, 700, [700, 0, 333], seed=2200)
    ref, _ = run(wl)
    ref = ref.cpu()
    for ps, seed in [(16, 1), (32, 2), (128, 3), (256, 4)]:
        out, _ = run(workloads.repage(wl, ps, seed))
        assert torch.equal(out.cpu(), ref), ps


def test_fp4_page_size_bitwise_d64():
    """D = 64: a page is 9 ps / 16 rows of 64 bytes with the 64-byte swizzle;
    every page size gives the same logits bit for bit."""
    wl = workloads.make_workload("fp4", 3, 2, 16, 64, 64, 700, [700, 1, 321], seed=2250)
    ref, _ = run(wl)
    ref = ref.cpu()
    for ps, seed in [(16, 5), (32, 6), (128, 7), (256, 8)]:
        out, _ = run(workloads.repage(wl, ps, seed))
        assert torch.equal(out.cpu(), ref), ps


def test_fp4_q_row_outside_the_f16_scaling_range_is_flagged():
    """A q row whose largest |q| is below 2^-86 cannot be brought into f16's
    normal range by the power-of-two row scale: MQA_STATUS_Q_RANGE is raised
    (rows in range raise nothing)."""
    import paged_mqa_logits_b200 as mq
    wl = workloads.make_workload("fp4", 2, 1, 32, 128, 64, 300, [300, 200], seed=2300)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    run(wl, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    q = wl.q.view(torch.bfloat16).float()
    q[1] *= 2.0 ** -100
    wl.q = q.to(torch.bfloat16).view(torch.int16).contiguous()
    run(wl, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mq.MQA_STATUS_Q_RANGE
