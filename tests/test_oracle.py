"""Pins for the fp64 CPU oracle (no GPU).

The oracle is checked against things other than itself:
  * exact rational brute force on tiny inputs, with torch-decoded values and
    the logical K gathered row by row (not per token through the page table);
  * a hand-worked example (tests/golden/logits_hand.json);
  * closed forms that isolate one term each (gather, sign, scale, ReLU, head
    weights, draft index);
  * a special case that reduces to a numpy matrix-vector product;
  * invariants: head permutation, page size, block-table permutation,
    power-of-two scale, weight negation, masking, non-negativity.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])


def decode_q(wl):
    """q as float64 numpy [B, next_n, H, D], decoded by torch and the OCP e2m1
    value table (independent of the oracle)."""
    if wl.kind == "fp8":
        return wl.q.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    if wl.kind == "fp4":
        return wl.q.view(torch.bfloat16).to(torch.float64).numpy()
    B, nn, H, D = wl.B, wl.next_n, wl.H, wl.D
    raw = wl.q.reshape(B, nn, -1)
    packed = raw[..., :H * D // 2].reshape(B, nn, H, D // 2).numpy()
    codes = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(B, nn, H, D)
    sc = raw[..., H * D // 2:].contiguous().view(torch.float8_e4m3fn).to(torch.float64)
    return E2M1[codes] * np.repeat(sc.numpy().reshape(B, nn, H, D // 16), 16, axis=-1)


def logical_k(wl, b):
    """Row b's K as [ctx_b, D] float64 and its per-token scales [ctx_b],
    gathered by concatenating the row's pages in block-table order."""
    n = int(wl.context_lens[b])
    ps, D = wl.page_size, wl.D
    npg = (n + ps - 1) // ps
    pages = wl.kv_cache[wl.block_table[b, :npg].long()]
    if wl.kind == "fp8":
        k = pages[:, :ps * D].reshape(npg * ps, D)[:n]
        s = pages[:, ps * D:].contiguous().view(torch.float32).reshape(-1)[:n]
        return (k.view(torch.float8_e4m3fn).to(torch.float64).numpy(),
                s.to(torch.float64).numpy())
    packed = pages[:, :ps * D // 2].reshape(npg * ps, D // 2)[:n].numpy()
    codes = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(n, D)
    sc = pages[:, ps * D // 2:].reshape(npg * ps, D // 16)[:n]
    sc = sc.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    k = E2M1[codes] * np.repeat(sc, 16, axis=1)
    return k, np.ones(n)


def brute_force_exact(wl):
    """Exact rational logits, [B][next_n][L] of Fraction or None (masked)."""
    q = decode_q(wl)
    w = wl.weights.to(torch.float64).numpy()
    res = []
    for b in range(wl.B):
        k, s = logical_k(wl, b)
        rows = []
        for n in range(wl.next_n):
            cbn = max(0, min(int(wl.context_lens[b]) - wl.next_n + 1 + n, int(wl.context_lens[b])))
            row = []
            for t in range(wl.out_len):
                if t >= cbn:
                    row.append(None)
                    continue
                tot = Fraction(0)
                for h in range(wl.H):
                    sc = sum(Fraction(float(q[b, n, h, d])) * Fraction(float(k[t, d]))
                             for d in range(wl.D))
                    r = Fraction(float(s[t])) * sc
                    tot += Fraction(float(w[b, n, h])) * max(r, Fraction(0))
                row.append(tot)
            rows.append(row)
        res.append(rows)
    return res


def small(kind="fp8", B=3, next_n=1, H=4, D=32, ps=16, L=72, ctx=(37, 0, 70), seed=5, **kw):
    return workloads.make_workload(kind, B, next_n, H, D, ps, L, list(ctx), seed, **kw)


@pytest.mark.parametrize("wl", [
    workloads.make_config("tiny"),
    small(next_n=2, ctx=(1, 17, 33), seed=9),
    small(B=2, next_n=3, H=2, ps=8, L=24, ctx=(2, 21), seed=11),
    small(kind="fp4", B=2, next_n=1, H=3, D=32, ps=16, L=40, ctx=(33, 5), seed=13),
    small(kind="nvfp4", B=2, next_n=2, H=3, D=32, ps=16, L=40, ctx=(33, 5), seed=15),
], ids=["tiny", "mtp2", "mtp3", "fp4", "nvfp4"])
def test_matches_exact_rational_brute_force(wl):
    out, absw = oracle.logits(wl)
    exact = brute_force_exact(wl)
    for b in range(wl.B):
        for n in range(wl.next_n):
            for t in range(wl.out_len):
                e = exact[b][n][t]
                if e is None:
                    assert out[b, n, t] == -np.inf
                else:
                    # fp64 evaluation of at most H*D dyadic products: tiny relative error
                    assert abs(out[b, n, t] - float(e)) <= 1e-12 * (absw[b, n, t] + 1e-30), (b, n, t)


def _hand_workload():
    g = json.load(open(os.path.join(GOLDEN, "logits_hand.json")))
    sh = g["shape"]
    wl = workloads.make_workload("fp8", sh["B"], sh["next_n"], sh["H"], sh["D"], sh["page_size"],
                                 sh["out_len"], [sh["context_len"]], seed=1)
    q = torch.zeros(1, 1, sh["H"], sh["D"])
    for h, d, v in g["q_nonzero"]:
        q[0, 0, h, d] = v
    wl.q = q.to(torch.float8_e4m3fn).view(torch.uint8)
    kv = wl.kv_cache.clone()
    ps, D = sh["page_size"], sh["D"]
    page = int(wl.block_table[0, 0])
    k = torch.zeros(ps, D)
    for t, d, v in g["k_nonzero"]:
        k[t, d] = v
    kv[page, :ps * D] = k.to(torch.float8_e4m3fn).view(torch.uint8).reshape(-1)
    s = torch.ones(ps)
    s[:3] = torch.tensor(g["scales"])
    kv[page, ps * D:] = s.view(torch.uint8)
    wl.kv_cache = kv
    wl.weights = torch.tensor(g["weights"], dtype=torch.float32).reshape(1, 1, -1)
    return wl, g


def test_hand_worked_example():
    wl, g = _hand_workload()
    out, _ = oracle.logits(wl)
    want = [float("-inf") if e == "-inf" else e for e in g["expected"]]
    assert list(out[0, 0]) == want


def _one_hot_case(next_n=1, seed=3):
    """H heads, head h looks only at feature h of K (q = e_h) with q scale c_h."""
    wl = small(B=2, next_n=next_n, H=3, D=32, ps=16, L=50, ctx=(45, 20), seed=seed)
    q = torch.zeros(wl.B, next_n, wl.H, wl.D)
    c = torch.tensor([1.0, -2.0, 0.5])
    for n in range(next_n):
        for h in range(wl.H):
            q[:, n, h, h + n] = c[h]
    wl.q = q.to(torch.float8_e4m3fn).view(torch.uint8)
    return wl, c


@pytest.mark.parametrize("next_n", [1, 2])
def test_closed_form_one_hot_heads(next_n):
    """out[b,n,t] = sum_h w_h * max(0, s_t * c_h * k_t[h + n]): pins the page
    gather, the per-token scale, the sign, the ReLU, the weights and the draft
    offset of q, each term by itself."""
    wl, c = _one_hot_case(next_n)
    out, _ = oracle.logits(wl)
    w = wl.weights.double().numpy()
    for b in range(wl.B):
        k, s = logical_k(wl, b)
        for n in range(next_n):
            cbn = max(0, int(wl.context_lens[b]) - next_n + 1 + n)
            for t in range(wl.out_len):
                if t >= cbn:
                    assert out[b, n, t] == -np.inf
                    continue
                want = sum(w[b, n, h] * max(0.0, s[t] * float(c[h]) * k[t, h + n])
                           for h in range(wl.H))
                assert out[b, n, t] == pytest.approx(want, rel=1e-15, abs=0)


def test_closed_form_zero_k_and_negative_scores():
    wl = small(seed=21)
    kv = wl.kv_cache.clone()
    kv[:, :16 * 32] = 0  # every K byte zero -> every score 0
    wl.kv_cache = kv
    out, _ = oracle.logits(wl)
    ctx = wl.context_lens
    for b in range(wl.B):
        assert np.all(out[b, 0, :int(ctx[b])] == 0.0)
    # q = -k direction for a single head: all scores <= 0 -> exactly 0
    wl = small(H=1, seed=22)
    wl.q = torch.zeros_like(wl.q)
    qq = torch.zeros(wl.B, 1, 1, 32)
    qq[..., 0] = 1.0
    wl.q = qq.to(torch.float8_e4m3fn).view(torch.uint8)
    kv = wl.kv_cache.clone()
    kk = kv[:, :16 * 32].view(torch.float8_e4m3fn).to(torch.float32).view(-1, 16, 32)
    kk[..., 0] = -kk[..., 0].abs()
    kv[:, :16 * 32] = kk.to(torch.float8_e4m3fn).view(torch.uint8).reshape(kv.shape[0], -1)
    wl.kv_cache = kv
    out, _ = oracle.logits(wl)
    for b in range(wl.B):
        assert np.all(out[b, 0, :int(wl.context_lens[b])] == 0.0)


@pytest.mark.parametrize("kind", ["fp8", "fp4", "nvfp4"])
def test_single_head_reduces_to_matvec(kind):
    """H=1, w=1: out[t] = max(0, s_t * q.k_t), i.e. ReLU of a numpy mat-vec
    product against the row's logical K."""
    wl = small(kind=kind, B=2, H=1, D=64, ps=16, L=90, ctx=(85, 40), seed=31)
    wl.weights = torch.ones_like(wl.weights)
    out, _ = oracle.logits(wl)
    q = decode_q(wl)
    for b in range(wl.B):
        k, s = logical_k(wl, b)
        want = np.maximum(0.0, s * (k @ q[b, 0, 0]))
        n = int(wl.context_lens[b])
        np.testing.assert_allclose(out[b, 0, :n], want, rtol=1e-14, atol=0)
        assert np.all(out[b, 0, n:] == -np.inf)


def test_head_permutation_invariance():
    wl = workloads.make_config("decode")
    wl = workloads.make_workload("fp8", 4, 1, 64, 128, 64, 700, [700, 1, 256, 513], seed=41)
    out, absw = oracle.logits(wl)
    perm = torch.randperm(wl.H, generator=torch.Generator().manual_seed(0))
    wl2 = workloads.Workload(**{**wl.__dict__, "q": wl.q[:, :, perm].contiguous(),
                                "weights": wl.weights[:, :, perm].contiguous()})
    out2, _ = oracle.logits(wl2)
    fin = np.isfinite(out)
    assert np.array_equal(fin, np.isfinite(out2))
    assert np.all(np.abs(out[fin] - out2[fin]) <= 1e-12 * absw[fin] + 1e-300)


@pytest.mark.parametrize("kind", ["fp8", "fp4", "nvfp4"])
def test_page_size_and_block_table_invariance(kind):
    wl = small(kind=kind, B=3, next_n=2, H=4, D=32, ps=16, L=300, ctx=(257, 0, 129), seed=51)
    out, _ = oracle.logits(wl)
    for ps, seed in [(8, 1), (16, 2), (32, 3), (64, 4), (128, 5)]:
        out2, _ = oracle.logits(workloads.repage(wl, ps, seed))
        assert np.array_equal(out, out2), ps


def test_scale_power_of_two_and_weight_negation():
    wl = small(B=2, ctx=(60, 31), L=64, seed=61)
    out, _ = oracle.logits(wl)
    kv = wl.kv_cache.clone()
    s = kv[:, 16 * 32:].contiguous().view(torch.float32) * 4.0
    kv[:, 16 * 32:] = s.view(torch.uint8)
    out4, _ = oracle.logits(workloads.Workload(**{**wl.__dict__, "kv_cache": kv}))
    assert np.array_equal(out4, np.where(np.isfinite(out), out * 4.0, out))
    outn, _ = oracle.logits(workloads.Workload(**{**wl.__dict__, "weights": -wl.weights}))
    assert np.array_equal(outn, np.where(np.isfinite(out), -out, out))


def test_masking_and_nonnegativity():
    wl = small(B=4, next_n=3, ctx=(0, 1, 2, 70), L=72, seed=71, weights_nonneg=True)
    out, _ = oracle.logits(wl)
    cbn = wl.draft_context_lens().numpy()
    t = np.arange(wl.out_len)
    assert np.array_equal(np.isinf(out), t[None, None, :] >= cbn[:, :, None])
    assert np.all(out[np.isfinite(out)] >= 0.0)


def test_draft_rows_equal_single_draft_workloads():
    """Draft n of row b equals a one-draft workload with q[b,n], w[b,n] and
    context ctx_b - next_n + 1 + n over the same pages."""
    wl = small(B=2, next_n=3, ctx=(40, 2), L=48, seed=81)
    out, _ = oracle.logits(wl)
    for n in range(3):
        c = torch.clamp(wl.context_lens - 3 + 1 + n, min=0)
        one = workloads.Workload(**{**wl.__dict__, "next_n": 1,
                                    "q": wl.q[:, n:n + 1].contiguous(),
                                    "weights": wl.weights[:, n:n + 1].contiguous(),
                                    "context_lens": c.to(torch.int32)})
        o1, _ = oracle.logits(one)
        assert np.array_equal(o1[:, 0], out[:, n])


@pytest.mark.parametrize("kind", ["fp8", "fp4", "nvfp4"])
def test_points_agree_with_full(kind):
    wl = small(kind=kind, B=3, next_n=2, ctx=(50, 0, 17), L=64, seed=91)
    out, absw = oracle.logits(wl)
    rng = np.random.default_rng(0)
    idx = np.stack([rng.integers(0, wl.B, 200), rng.integers(0, 2, 200),
                    rng.integers(0, wl.out_len, 200)], axis=1).astype(np.int64)
    p, pa = oracle.points(wl, idx)
    assert np.array_equal(p, out[idx[:, 0], idx[:, 1], idx[:, 2]])
    assert np.array_equal(pa, absw[idx[:, 0], idx[:, 1], idx[:, 2]])


def test_nvfp4_equals_fp4_with_its_q_decoded_to_bf16():
    """An NVFP4 q's values (e2m1 code x e4m3 block scale: at most 5
    significant bits, within [2^-10, 2688]) are exact in bf16, so the
    block-scaled variant must equal the bf16-q FP4 definition on the same
    pages, bit for bit."""
    wl = small(kind="nvfp4", B=3, next_n=2, H=4, D=64, ps=16, L=90, ctx=(85, 0, 40), seed=101)
    qv = decode_q(wl)
    qb = torch.from_numpy(qv).to(torch.bfloat16)
    assert np.array_equal(qb.to(torch.float64).numpy(), qv)  # exact in bf16
    as_fp4 = workloads.Workload(**{**wl.__dict__, "kind": "fp4",
                                   "q": qb.view(torch.int16).contiguous()})
    out, absw = oracle.logits(wl)
    out4, absw4 = oracle.logits(as_fp4)
    assert np.array_equal(out, out4) and np.array_equal(absw, absw4)


def test_nvfp4_closed_form_one_hot_q():
    """q = 1.0 at one (head, element) and 0 elsewhere, weight 1 on that head:
    out[t] = max(0, k_t[d0]) with k_t decoded from the page bytes."""
    wl = small(kind="nvfp4", B=1, next_n=1, H=4, D=64, ps=16, L=50, ctx=(47,), seed=111)
    H, D, h0, d0 = wl.H, wl.D, 2, 37
    q = torch.zeros_like(wl.q)
    code_byte = 0x2 if d0 % 2 == 0 else 0x20         # e2m1 1.0 in d0's nibble
    q[0, 0, h0 * (D // 2) + d0 // 2] = code_byte
    q[0, 0, H * (D // 2) + h0 * (D // 16) + d0 // 16] = 0x38  # e4m3 1.0
    w = torch.zeros_like(wl.weights)
    w[0, 0, h0] = 1.0
    one = workloads.Workload(**{**wl.__dict__, "q": q, "weights": w})
    out, _ = oracle.logits(one)
    k, _ = logical_k(one, 0)
    np.testing.assert_array_equal(out[0, 0, :47], np.maximum(k[:, d0], 0.0))
    assert np.all(out[0, 0, 47:] == -np.inf)


@pytest.mark.parametrize("kind", ["fp8", "fp4", "nvfp4"])
def test_threaded_runner_is_bit_identical(kind):
    """Spreading rows (or points) over threads changes nothing: every element
    comes from the same C call on the same row."""
    H = 32 if kind != "fp8" else 64
    wl = workloads.make_workload(kind, 7, 2, H, 128, 16, 1100, [1100, 0, 513, 1, 700, 256, 999],
                                 seed=41)
    one, a1 = oracle.logits(wl)
    for threads in (3, None):
        many, am = oracle.logits(wl, threads=threads)
        assert np.array_equal(one, many) and np.array_equal(a1, am)
    idx = np.array([(b, n, t) for b in range(7) for n in range(2) for t in (0, 5, 255, 256, 1099)],
                   dtype=np.int64)
    p1, q1 = oracle.points(wl, idx)
    pm, qm = oracle.points(wl, idx, threads=4)
    assert np.array_equal(p1, pm) and np.array_equal(q1, qm)
    assert np.array_equal(p1, one[idx[:, 0], idx[:, 1], idx[:, 2]])
