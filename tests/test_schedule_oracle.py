"""Pins for the schedule oracle (linear scan), no GPU: hand-worked cases,
a brute force that materialises the flat unit list, and invariants."""
import json
import os

import numpy as np
import pytest

import oracle
import workloads
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def flat_units(ctx):
    """Every (row, unit) pair in order: the brute-force view of the schedule."""
    out = []
    for b, c in enumerate(ctx):
        for j in range((max(int(c), 0) + 255) // 256):
            out.append((b, j))
    return out


def brute(ctx, S):
    units = flat_units(ctx)
    U = len(units)
    res = []
    for i in range(S + 1):
        start = i * (U // S) + min(i, U % S)
        res.append(units[start] if start < U else (len(ctx), 0))
    return np.array(res, dtype=np.int32)


def test_golden_cases():
    g = json.load(open(os.path.join(GOLDEN, "schedule_cases.json")))
    for case in g["cases"]:
        got = oracle.schedule(case["context_lens"], case["num_ctas"])
        assert got.tolist() == case["schedule"], case["why"]


def random_ctx(rng, B):
    kind = rng.integers(0, 4)
    if kind == 0:
        return rng.integers(0, 4097, B)
    if kind == 1:
        c = 256 * rng.integers(0, 9, B) + rng.integers(-1, 2, B)
        return np.clip(c, 0, None)
    if kind == 2:
        c = rng.integers(0, 3000, B)
        c[rng.random(B) < 0.5] = 0
        return c
    return rng.integers(0, 300, B)


@pytest.mark.parametrize("seed", range(40))
def test_matches_brute_force_and_invariants(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 200))
    S = int(rng.choice([1, 2, 7, 148, 300]))
    ctx = random_ctx(rng, B).astype(np.int32)
    got = oracle.schedule(ctx, S)
    assert np.array_equal(got, brute(ctx, S))
    u = (ctx.astype(np.int64) + 255) // 256
    U = int(u.sum())
    P = np.concatenate([[0], np.cumsum(u)])
    starts = np.array([P[r] + o if r < B else U for r, o in got])
    counts = np.diff(starts)
    assert counts.sum() == U
    assert counts.max() - counts.min() <= 1
    assert np.all(np.diff(starts) >= 0)
    for r, o in got:
        if r < B:
            assert u[r] > 0 and 0 <= o < u[r]
        else:
            assert r == B and o == 0


@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_config_schedules_match_brute_force(name):
    ctx = workloads.make_config(name).context_lens.numpy()
    for S in (148, 1, 37):
        assert np.array_equal(oracle.schedule(ctx, S), brute(ctx, S))
