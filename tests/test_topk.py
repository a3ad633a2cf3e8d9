"""Top-k parity: the CUDA selection (through the C ABI) against the oracle's,
on the same fp32 logits, bit-exact (integer output: which tokens, in which
order), in both orders (by value, by token). Tie-heavy inputs exercise the
ordering rule; the context rule and -1 padding are exercised by short, empty
and over-long rows; long rows reach the kernel's three ways of reading a row
(keys cached in shared memory, a candidate list, re-reads from global). The
row-mode cases run with one CTA per row and with every row split over a
cluster of 2 and of 4 CTAs."""
import numpy as np
import pytest
import torch

import oracle
import paged_mqa_logits_b200 as mq
import workloads
from tests.helpers import run

pytestmark = pytest.mark.gpu


def gpu_topk(lg, ctx, k, by_token=False, offset=0):
    """offset > 0 places the logits `offset` floats past an aligned base, so
    no row starts on a 16-byte boundary."""
    flat = torch.zeros(lg.size + offset, dtype=torch.float32, device="cuda")
    flat[offset:] = torch.from_numpy(lg.reshape(-1)).cuda()
    dev = flat[offset:].view(lg.shape)
    out = mq.mqa_logits_topk(dev, torch.from_numpy(ctx).cuda(), k, by_token=by_token)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def keys(v):
    """Order-preserving uint32 keys of fp32 values (-0.0 as +0.0)."""
    u = np.ascontiguousarray(v, np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def top_digit_share(row, k):
    """How many of a row's keys share the first radix digit of its k-th
    largest key: the 11 bits from the highest bit where the row's keys differ."""
    kk = keys(row).astype(np.int64)
    hb = int(kk.min() ^ kk.max()).bit_length() - 1
    sh = max(hb - 10, 0)
    kth = np.sort(kk)[::-1][k - 1]
    return int(((kk >> sh) == (kth >> sh)).sum())


@pytest.fixture(params=["1", "2", "4"], ids=["cta", "cluster2", "cluster4"])
def cluster(request, monkeypatch):
    """Row-mode selection with one CTA per row, or every row split over a
    cluster of 2 or 4 CTAs (the library reads MQA_TOPK_CLUSTER at each call)."""
    monkeypatch.setenv("MQA_TOPK_CLUSTER", request.param)
    return request.param


def tie_heavy(rng, B, nn, L, distinct=None):
    if distinct is None:
        return rng.standard_normal((B, nn, L)).astype(np.float32)
    palette = np.concatenate([[-0.0, 0.0], rng.standard_normal(distinct - 2)]).astype(np.float32)
    return palette[rng.integers(0, palette.size, size=(B, nn, L))]


@pytest.mark.parametrize("by_token", [False, True])
@pytest.mark.parametrize("k", [1, 7, 64, 300, 1000, 2048, 4096])
@pytest.mark.parametrize("distinct", [None, 5, 300])
def test_topk_matches_oracle(k, distinct, by_token, cluster):
    rng = np.random.default_rng(k * 7 + (distinct or 0))
    B, nn, L = 7, 2, 5000
    ctx = np.array([0, 1, 2, k - 1 if k > 1 else 3, k, 4999, 6000], np.int32)
    lg = tie_heavy(rng, B, nn, L, distinct)
    np.testing.assert_array_equal(gpu_topk(lg, ctx, k, by_token),
                                  oracle.topk(lg, ctx, nn, k, by_token))


@pytest.mark.parametrize("by_token", [False, True])
def test_topk_long_rows_candidate_list_and_global_rereads(by_token, cluster):
    """Rows past 16384 valid tokens: spread values, and positive values packed
    into a narrow range like real logits (sums of ReLU terms), keep the keys
    sharing the threshold's first digit under 8192 (candidate list); five
    distinct values do not (every pass re-reads the row)."""
    rng = np.random.default_rng(3)
    spread = tie_heavy(rng, 2, 4, 131072, 1000)
    packed = (20.0 + 2.0 * rng.standard_normal((2, 4, 131072))).astype(np.float32)
    ties = tie_heavy(rng, 2, 4, 131072, 5)
    ctx = np.array([131072, 77777], np.int32)
    for k in (2048, 4096):
        assert top_digit_share(spread[0, 3], k) <= 8192
        assert top_digit_share(packed[0, 3], k) <= 8192
        assert top_digit_share(ties[0, 3], k) > 8192
        for lg in (spread, packed, ties):
            np.testing.assert_array_equal(gpu_topk(lg, ctx, k, by_token),
                                          oracle.topk(lg, ctx, 4, k, by_token))


@pytest.mark.parametrize("by_token", [False, True])
def test_topk_packed_values_and_constant_rows(by_token, cluster):
    """Short rows of positive values in a narrow range (the first digit starts
    low in the key), and rows whose valid logits are all equal."""
    rng = np.random.default_rng(11)
    lg = (20.0 + 2.0 * rng.standard_normal((4, 2, 5000))).astype(np.float32)
    lg[1] = 3.25
    lg[2, :, :2500] = -7.0
    ctx = np.array([5000, 4000, 2500, 300], np.int32)
    for k in (1, 64, 2048):
        np.testing.assert_array_equal(gpu_topk(lg, ctx, k, by_token),
                                      oracle.topk(lg, ctx, 2, k, by_token))


@pytest.mark.parametrize("by_token", [False, True])
def test_topk_cache_boundary_and_unaligned_rows(by_token, cluster):
    """16384 valid tokens (the most kept in shared memory) and one more; rows
    of odd length from a base 4 bytes past alignment."""
    rng = np.random.default_rng(5)
    lg = tie_heavy(rng, 3, 1, 20001, 300)
    ctx = np.array([16384, 16385, 20001], np.int32)
    for k in (100, 2048):
        for offset in (0, 1):
            np.testing.assert_array_equal(gpu_topk(lg, ctx, k, by_token, offset),
                                          oracle.topk(lg, ctx, 1, k, by_token))


def test_topk_signed_zero_and_infinities_past_context(cluster):
    lg = np.full((1, 1, 64), -np.inf, np.float32)
    lg[0, 0, :40] = np.where(np.arange(40) % 2 == 0, -0.0, 0.0)
    lg[0, 0, 7] = 1.0
    ctx = np.array([40], np.int32)
    for k in (1, 8, 39, 40, 41, 64):
        for by_token in (False, True):
            np.testing.assert_array_equal(gpu_topk(lg, ctx, k, by_token),
                                          oracle.topk(lg, ctx, 1, k, by_token))


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
    by_tok = mq.mqa_logits_topk(out, torch.as_tensor(wl.context_lens).cuda(), k, by_token=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(by_tok.cpu().numpy(),
                                  oracle.topk(g, wl.context_lens.numpy(), wl.next_n, k, True))
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


@pytest.mark.parametrize("by_token", [False, True])
def test_topk_values_output(by_token, cluster):
    """values[i] is the logit of indices[i] (-0.0 reported as +0.0), -inf past
    the valid tokens."""
    rng = np.random.default_rng(21)
    lg = tie_heavy(rng, 4, 2, 3000, 300)
    ctx = np.array([3000, 100, 1, 0], np.int32)
    for k in (1, 128, 2048):
        idx, val = mq.mqa_logits_topk(torch.from_numpy(lg).cuda(), torch.from_numpy(ctx).cuda(),
                                      k, by_token=by_token, with_values=True)
        torch.cuda.synchronize()
        idx, val = idx.cpu().numpy(), val.cpu().numpy()
        np.testing.assert_array_equal(idx, oracle.topk(lg, ctx, 2, k, by_token))
        want = np.where(idx >= 0, np.take_along_axis(lg, np.maximum(idx, 0), 2), -np.inf)
        np.testing.assert_array_equal(val, want + np.float32(0.0))  # -0.0 -> +0.0


def emulated_sharded_topk(full, valid, k, shards, by_token):
    """The sharded top-k on one GPU: rows split by token range into `shards`
    ranges, each range's own top-k (by token, with values), the lists stacked
    as an all-gather would, then the merge kernel."""
    from paged_mqa_logits_b200.shard import shard_tokens
    rows, L = full.shape
    vals, toks, offs, cnts = [], [], [], []
    for s in range(shards):
        lo, hi = shard_tokens(L, shards, s)
        local = torch.from_numpy(np.ascontiguousarray(full[:, lo:hi])).cuda().view(rows, 1, hi - lo)
        lv = torch.from_numpy(np.clip(valid - lo, 0, hi - lo).astype(np.int32)).cuda()
        i, v = mq.mqa_logits_topk(local, lv, k, by_token=True, with_values=True)
        toks.append(i.view(rows, k))
        vals.append(v.view(rows, k))
        offs.append(lo)
        cnts.append(hi - lo)
    idx, val = mq.mqa_logits_topk_merge(torch.stack(vals), torch.stack(toks), offs, cnts, k,
                                        by_token=by_token, with_values=True)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy()


@pytest.mark.parametrize("by_token", [False, True])
@pytest.mark.parametrize("shards", [1, 2, 3, 8])
@pytest.mark.parametrize("distinct", [None, 7])
def test_topk_merge_of_token_range_shards(shards, distinct, by_token):
    """The merged top-k equals the oracle's top-k of the whole rows, ties
    across shard boundaries included (the lower global token wins)."""
    rng = np.random.default_rng(shards * 13 + (distinct or 0))
    rows, L = 6, 20000
    full = tie_heavy(rng, rows, 1, L, distinct)[:, 0, :]
    valid = np.array([20000, 12345, 2500, 2047, 3, 0], np.int32)
    for k in (1, 64, 2048):
        if shards * k > mq.MQA_TOPK_MERGE_MAX:
            continue
        idx, val = emulated_sharded_topk(full, valid, k, shards, by_token)
        want = oracle.topk(full[:, None, :], valid, 1, k, by_token)[:, 0, :]
        np.testing.assert_array_equal(idx, want)
        wv = np.where(want >= 0, np.take_along_axis(full, np.maximum(want, 0), 1), -np.inf)
        np.testing.assert_array_equal(val, wv + np.float32(0.0))


def test_topk_merge_empty_and_short_lists():
    """Shards with no valid entries, fewer candidates than k (padding), and
    k_in different from k."""
    vals = torch.full((3, 2, 5), -np.inf, dtype=torch.float32)
    toks = torch.full((3, 2, 5), -1, dtype=torch.int32)
    vals[1, 0, :2] = torch.tensor([1.5, 1.5])
    toks[1, 0, :2] = torch.tensor([0, 4])
    vals[2, 0, :1] = torch.tensor([1.5])
    toks[2, 0, :1] = torch.tensor([2])
    for by_token, want in ((False, [[100, 104, 202, -1, -1, -1, -1], [-1] * 7]),
                           (True, [[100, 104, 202, -1, -1, -1, -1], [-1] * 7])):
        idx = mq.mqa_logits_topk_merge(vals.cuda(), toks.cuda(), [0, 100, 200], [100, 100, 5], 7,
                                       by_token=by_token)
        torch.cuda.synchronize()
        assert idx.cpu().tolist() == want
