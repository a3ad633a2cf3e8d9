"""Pins for the top-k oracle (selection of the k largest logits per row).

A hand-worked example (tests/golden/topk_hand.json) and, on tie-heavy random
inputs, the properties that together determine the answer uniquely: distinct
valid tokens, min(k, ctx_{b,n}) of them then -1, values non-increasing with
ties in token order, nothing left out beats anything taken, and no left-out
token ties the last taken value at a smaller index."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "topk_hand.json")


def test_hand_example():
    spec = json.load(open(GOLDEN))
    for c in spec["cases"]:
        lg = np.array([[[float(v) for v in r] for r in b] for b in c["logits"]], dtype=np.float32)
        got = oracle.topk(lg, np.array(c["ctx"], np.int32), c["next_n"], c["k"])
        assert got.tolist() == c["expect"]
        got = oracle.topk(lg, np.array(c["ctx"], np.int32), c["next_n"], c["k"], by_token=True)
        assert got.tolist() == c["expect_by_token"]


def _draft_ctx(c, L, next_n, n):
    c = min(max(c, 0), L)
    return min(max(c - next_n + 1 + n, 0), c)


@pytest.mark.parametrize("k", [1, 7, 64, 300, 512])
def test_properties_on_tie_heavy_rows(k):
    rng = np.random.default_rng(k)
    B, nn, L = 6, 2, 300
    ctx = np.array([0, 1, 2, 150, 300, 400], np.int32)
    palette = np.array([-3.5, -1.0, -0.0, 0.0, 0.25, 1.0, 2.0, 7.5], np.float32)
    lg = palette[rng.integers(0, palette.size, size=(B, nn, L))]
    out = oracle.topk(lg, ctx, nn, k)
    for b in range(B):
        for n in range(nn):
            cbn = _draft_ctx(int(ctx[b]), L, nn, n)
            row, sel = lg[b, n], out[b, n]
            m = min(k, cbn)
            assert np.all(sel[m:] == -1)
            s = sel[:m]
            assert len(set(s.tolist())) == m and np.all((s >= 0) & (s < cbn))
            v = row[s].astype(np.float64)
            assert np.all(np.diff(v) <= 0)
            eq = np.diff(v) == 0
            assert np.all(np.diff(s)[eq] > 0)          # equal values: token order
            rest = np.setdiff1d(np.arange(cbn), s)
            if m and rest.size:
                assert row[rest].max() <= v[-1]         # nothing left out beats a taken value
                tied = rest[row[rest] == v[-1]]
                if tied.size:                            # ties at the boundary: smallest tokens taken
                    assert tied.min() > s[v == v[-1]].max()


def test_planted_mistakes_are_caught():
    """The property check above rejects a wrong tie order and a wrong boundary."""
    lg = np.array([[[1.0, 3.0, 3.0, 2.0]]], np.float32)
    good = oracle.topk(lg, np.array([4], np.int32), 1, 2)[0, 0]
    assert good.tolist() == [1, 2]
    wrong_ties = [2, 1]        # equal values out of token order
    wrong_boundary = [1, 3]    # skips a larger value
    for bad in (wrong_ties, wrong_boundary):
        v = lg[0, 0, bad]
        ok_order = np.all(np.diff(v) <= 0) and np.all(np.diff(bad)[np.diff(v) == 0] > 0)
        rest = np.setdiff1d(np.arange(4), bad)
        ok_bound = lg[0, 0, rest].max() <= v[-1]
        assert not (ok_order and ok_bound)


@pytest.mark.parametrize("shards", [2, 3, 5])
def test_top_k_of_shard_top_ks_is_top_k_of_row(shards):
    """The property the sharded top-k rests on: with a row split into
    contiguous token ranges, the k best of the union of every range's own k
    best are the row's k best, ties included (equal values keep token order
    because the ranges ascend). Checked with the oracle alone."""
    rng = np.random.default_rng(40 + shards)
    L, k = 997, 50
    palette = np.array([-2.0, -0.0, 0.0, 0.5, 1.0, 3.0], np.float32)
    for trial in range(20):
        row = palette[rng.integers(0, palette.size, size=L)] if trial % 2 else \
            rng.standard_normal(L).astype(np.float32)
        valid = int(rng.integers(0, L + 1))
        want = oracle.topk(row[None, None, :], np.array([valid], np.int32), 1, k)[0, 0]
        # each range's own k best (global tokens), then the k best of their union
        bounds = np.linspace(0, L, shards + 1).astype(int)
        cand = []
        for s in range(shards):
            lo, hi = bounds[s], bounds[s + 1]
            part = oracle.topk(np.ascontiguousarray(row[None, None, lo:hi]),
                               np.array([min(max(valid - lo, 0), hi - lo)], np.int32), 1, k)[0, 0]
            cand += [lo + int(t) for t in part if t >= 0]
        cand = np.array(sorted(cand), np.int64)  # ascending global tokens
        got = oracle.topk(row[cand][None, None, :], np.array([cand.size], np.int32), 1, k)[0, 0]
        got = np.where(got >= 0, cand[np.maximum(got, 0)], -1)
        np.testing.assert_array_equal(got, want)
