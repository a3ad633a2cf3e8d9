"""Logits parity: the CUDA path (through the C ABI) against the fp64 oracle,
element by element on the same seeded inputs.

Bar: |gpu - ref| <= 1e-3 * sum_h |w_h * ReLU(s * score_h)| + 1e-5 for every
finite element; -inf exactly where t >= ctx_{b,n} (bit-exact masking)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.helpers import compare, run

pytestmark = pytest.mark.gpu


def full_check(wl, **kw):
    out, _ = run(wl, **kw)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl)
    return compare(out.cpu().numpy(), ref, absw)


def test_tiny_config():
    full_check(workloads.make_config("tiny"))


MID = [
    # (kind, B, next_n, H, D, page, L, ctx)  -- several tiles, ragged tails
    ("fp8", 5, 1, 64, 128, 64, 1504, [1, 127, 128, 129, 1500]),
    ("fp8", 4, 2, 64, 128, 64, 1028, [1, 2, 255, 1027]),
    ("fp8", 3, 3, 32, 128, 16, 700, [700, 0, 257]),
    ("fp8", 3, 4, 16, 64, 32, 520, [513, 4, 300]),
    ("fp8", 3, 1, 128, 128, 128, 900, [899, 384, 1]),
    ("fp8", 2, 2, 128, 128, 256, 1100, [1100, 640]),
    ("fp8", 4, 1, 8, 32, 8, 400, [399, 33, 0, 256]),
    ("fp8", 3, 4, 4, 32, 16, 300, [3, 300, 129]),
    ("fp8", 3, 2, 4, 64, 64, 260, [260, 5, 128]),
]


@pytest.mark.parametrize("case", MID, ids=[f"{c[0]}-B{c[1]}-nn{c[2]}-H{c[3]}-D{c[4]}-ps{c[5]}"
                                           for c in MID])
def test_mid_sizes_full(case):
    kind, B, nn, H, D, ps, L, ctx = case
    wl = workloads.make_workload(kind, B, nn, H, D, ps, L, ctx, seed=1000 + MID.index(case))
    full_check(wl)


# The per-CTA work table holds at most min(32, 512 / (256 / page_size)) units
# per chunk (16 at page size 8, 32 from page size 16 up) and is built 32 rows
# at a time. These cases make one CTA walk several chunks (the builder waits
# for chunk k - 2 to be released before refilling its buffer) and span many
# builder windows of short and empty rows (row sequence numbers and the q
# double buffer across windows).
CHUNKED = [
    # (kind, B, next_n, H, D, page, L, ctx, num_ctas)
    ("fp8", 3, 1, 8, 32, 8, 12800, [12800, 9001, 4097], 2),     # ~50 units per CTA, chunks of 16
    ("fp8", 2, 2, 16, 64, 64, 20000, [20000, 17777], 1),        # 149 units, chunks of 32
    ("fp4", 2, 1, 8, 64, 16, 12000, [12000, 9999], 1),          # 87 units, chunks of 32
]


@pytest.mark.parametrize("case", CHUNKED, ids=[f"{c[0]}-ps{c[5]}-S{c[8]}" for c in CHUNKED])
def test_several_table_chunks_per_cta(case):
    kind, B, nn, H, D, ps, L, ctx, S = case
    wl = workloads.make_workload(kind, B, nn, H, D, ps, L, ctx, seed=2000 + CHUNKED.index(case))
    full_check(wl, num_ctas=S)


def test_many_short_rows_per_cta():
    """150 rows over 3 CTAs: every builder window of 32 rows mixes empty rows,
    one-token rows, rows ending in either half of a unit and multi-unit rows."""
    rng = np.random.default_rng(7)
    ctx = rng.choice([0, 1, 2, 127, 128, 129, 255, 256, 257, 600], size=150).tolist()
    wl = workloads.make_workload("fp8", 150, 2, 8, 32, 16, 608, ctx, seed=2100)
    full_check(wl, num_ctas=3)


@pytest.mark.parametrize("S", [1, 3, 148, 400])
def test_num_ctas_does_not_change_results(S):
    wl = workloads.make_workload("fp8", 6, 2, 64, 128, 64, 2048, [2048, 0, 1, 1000, 513, 77],
                                 seed=3)
    full_check(wl, num_ctas=S)


@pytest.mark.parametrize("name", ["decode", "stress", "mtp"])
def test_full_size_every_element(name):
    """Full-size workload in the benchmark's launch configuration (one CTA per
    SM): every element against the oracle (run on all host cores), masks
    bit-exact, values within the tolerance. This covers every tile, page and
    context edge and every point where one CTA's range ends inside a row."""
    wl = workloads.make_config(name)
    out, _ = run(wl)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl, threads=None)
    compare(out.cpu().numpy(), ref, absw)


def test_page_size_gives_bitwise_identical_output():
    wl = workloads.make_workload("fp8", 4, 2, 64, 128, 64, 1200, [1200, 0, 555, 129], seed=17)
    ref, _ = run(wl)
    ref = ref.cpu()
    for ps, seed in [(8, 1), (16, 2), (32, 3), (128, 4), (256, 5)]:
        out, _ = run(workloads.repage(wl, ps, seed))
        assert torch.equal(out.cpu(), ref), ps


def test_head_permutation_within_tolerance():
    wl = workloads.make_workload("fp8", 3, 1, 64, 128, 64, 600, [600, 300, 1], seed=19)
    ref, absw = oracle.logits(wl)
    perm = torch.randperm(64, generator=torch.Generator().manual_seed(0))
    wl2 = workloads.Workload(**{**wl.__dict__, "q": wl.q[:, :, perm].contiguous(),
                                "weights": wl.weights[:, :, perm].contiguous()})
    out, _ = run(wl2)
    compare(out.cpu().numpy(), ref, absw)


def test_nonneg_weights_give_nonneg_logits():
    wl = workloads.make_workload("fp8", 3, 2, 64, 128, 64, 520, [520, 17, 300], seed=23,
                                 weights_nonneg=True)
    out, _ = run(wl)
    g = out.cpu()
    assert bool((g[torch.isfinite(g)] >= 0).all())


def test_zero_rows_and_empty_batch():
    wl = workloads.make_workload("fp8", 3, 1, 64, 128, 64, 256, [0, 0, 0], seed=29)
    out, _ = run(wl)
    assert bool(torch.isneginf(out).all())
    wl = workloads.make_workload("fp8", 0, 1, 64, 128, 64, 256, [], seed=31)
    out, _ = run(wl)
    assert out.numel() == 0
