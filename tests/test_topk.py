"""Top-k parity: the CUDA selection (through the C ABI) against the oracle's,
on the same fp32 logits, bit-exact (integer output: which tokens, in which
order). Tie-heavy inputs exercise the ordering rule; the context rule and
-1 padding are exercised by short, empty and over-long rows."""
import numpy as np
import pytest
import torch

import oracle
import paged_mqa_logits_b200 as mq
import workloads
from tests.helpers import run

pytestmark = pytest.mark.gpu


def gpu_topk(lg, ctx, k):
    out = mq.mqa_logits_topk(torch.from_numpy(lg).cuda(), torch.from_numpy(ctx).cuda(), k)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def tie_heavy(rng, B, nn, L, distinct=None):
    if distinct is None:
        return rng.standard_normal((B, nn, L)).astype(np.float32)
    palette = np.concatenate([[-0.0, 0.0], rng.standard_normal(distinct - 2)]).astype(np.float32)
    return palette[rng.integers(0, palette.size, size=(B, nn, L))]


@pytest.mark.parametrize("k", [1, 7, 64, 300, 1000, 2048, 4096])
@pytest.mark.parametrize("distinct", [None, 5, 300])
def test_topk_matches_oracle(k, distinct):
    rng = np.random.default_rng(k * 7 + (distinct or 0))
    B, nn, L = 7, 2, 5000
    ctx = np.array([0, 1, 2, k - 1 if k > 1 else 3, k, 4999, 6000], np.int32)
    lg = tie_heavy(rng, B, nn, L, distinct)
    np.testing.assert_array_equal(gpu_topk(lg, ctx, k), oracle.topk(lg, ctx, nn, k))


def test_topk_long_row_and_mtp_rows():
    rng = np.random.default_rng(3)
    lg = tie_heavy(rng, 2, 4, 131072, 1000)
    ctx = np.array([131072, 77777], np.int32)
    for k in (2048, 4096):
        np.testing.assert_array_equal(gpu_topk(lg, ctx, k), oracle.topk(lg, ctx, 4, k))


def test_topk_signed_zero_and_infinities_past_context():
    lg = np.full((1, 1, 64), -np.inf, np.float32)
    lg[0, 0, :40] = np.where(np.arange(40) % 2 == 0, -0.0, 0.0)
    lg[0, 0, 7] = 1.0
    ctx = np.array([40], np.int32)
    for k in (1, 8, 39, 40, 41, 64):
        np.testing.assert_array_equal(gpu_topk(lg, ctx, k), oracle.topk(lg, ctx, 1, k))


def test_topk_of_the_logits_kernel_output():
    """The indexer's pipeline: logits on the GPU, then top-k of those logits,
    compared with the oracle's top-k of the same GPU logits (bit-exact), and
    checked as a valid top-k of the oracle's fp64 logits within the logits
    tolerance."""
    wl = workloads.make_workload("fp8", 4, 2, 64, 128, 64, 3000, [3000, 0, 1500, 257], seed=31)
    out, _ = run(wl)
    torch.cuda.synchronize()
    k = 512
    idx = mq.mqa_logits_topk(out, torch.as_tensor(wl.context_lens).cuda(), k)
    torch.cuda.synchronize()
    g = out.cpu().numpy()
    got = idx.cpu().numpy()
    np.testing.assert_array_equal(got, oracle.topk(g, wl.context_lens.numpy(), wl.next_n, k))
    ref, absw = oracle.logits(wl)
    tol = 1e-3 * absw + 1e-5
    cbn = wl.draft_context_lens().numpy()
    for b in range(wl.B):
        for n in range(wl.next_n):
            m = min(k, int(cbn[b, n]))
            sel = got[b, n, :m]
            assert np.all(got[b, n, m:] == -1)
            if m == 0:
                continue
            rest = np.setdiff1d(np.arange(cbn[b, n]), sel)
            if rest.size:  # nothing left out is clearly larger than anything taken
                lo = (ref[b, n, sel] + tol[b, n, sel]).min()
                hi = (ref[b, n, rest] - tol[b, n, rest]).max()
                assert hi <= lo
