"""Block-scaled FP4 path (q and K both NVFP4, tcgen05 kind::mxf4nvf4) against
the fp64 oracle's NVFP4 definition: every element within the tolerance,
masking bit-exact, on mid sizes with ragged tails and on the full-size FP4
workload with an NVFP4 q."""
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
    ("B4-H8-D128-ps32", 4, 1, 8, 128, 32, 700, [1, 255, 257, 700]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_nvfp4_mid_sizes_full(case):
    _, B, nn, H, D, ps, L, ctx = case
    wl = workloads.make_workload("nvfp4", B, nn, H, D, ps, L, ctx, seed=4000 + CASES.index(case))
    out, _ = run(wl)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl)
    compare(out.cpu().numpy(), ref, absw)


def test_nvfp4_several_chunks_per_cta():
    wl = workloads.make_workload("nvfp4", 2, 1, 8, 64, 16, 12000, [12000, 9999], seed=4100)
    out, _ = run(wl, num_ctas=1)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl)
    compare(out.cpu().numpy(), ref, absw)


def test_nvfp4_config_every_element():
    """The FP4 workload's shapes (B=128, H=32, D=128, page 64, ctx U[512, 16384])
    with q in NVFP4: every element against the oracle."""
    wl = workloads.make_config("nvfp4")
    out, _ = run(wl)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl, threads=None)
    compare(out.cpu().numpy(), ref, absw)


def test_nvfp4_page_size_bitwise():
    wl = workloads.make_workload("nvfp4", 3, 2, 32, 128, 64, 700, [700, 0, 333], seed=4200)
    ref, _ = run(wl)
    ref = ref.cpu()
    for ps, seed in [(16, 1), (32, 2), (128, 3), (256, 4)]:
        out, _ = run(workloads.repage(wl, ps, seed))
        assert torch.equal(out.cpu(), ref), ps
