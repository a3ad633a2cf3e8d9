"""Shared test helpers: moving a workload to the GPU, running the path
through the binding, and the element-wise comparison with the oracle."""
import numpy as np
import torch

import paged_mqa_logits_b200 as mq

# |gpu - ref| <= RTOL * sum_h |w_h * ReLU(s * score_h)| + ATOL per element
RTOL = 1e-3
ATOL = 1e-5


def to_device(wl, device="cuda"):
    return dict(q=wl.q.to(device), kv=wl.kv_cache.to(device), bt=wl.block_table.to(device),
                ctx=wl.context_lens.to(device), w=wl.weights.to(device))


def run(wl, dev=None, num_ctas=None, flags=0, status=None, out=None, schedule=None):
    """Schedule + logits through the C ABI; returns (out, schedule) on the GPU."""
    dev = dev or to_device(wl)
    if schedule is None:
        schedule = mq.mqa_logits_schedule(dev["ctx"], num_ctas)
    kw = dict(page_size=wl.page_size, out_len=wl.out_len, flags=flags, status=status)
    if wl.kind == "nvfp4":
        fn = mq.paged_mqa_logits_nvfp4
        kw["num_heads"] = wl.H
    else:
        fn = mq.paged_mqa_logits_fp8 if wl.kind == "fp8" else mq.paged_mqa_logits_fp4
    out = fn(dev["q"], dev["kv"], dev["bt"], dev["ctx"], dev["w"], schedule, out, **kw)
    return out, schedule


def compare(gpu, ref, absw):
    """Masking bit-exact (-inf exactly where the oracle has -inf, finite
    elsewhere) and values within tolerance. Returns the largest
    |err| / (RTOL * absw + ATOL)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(gpu), ~fin), "masking differs from the oracle"
    assert np.all(np.isfinite(gpu[fin])), "non-finite value where the oracle is finite"
    err = np.abs(gpu[fin] - ref[fin])
    bound = RTOL * absw[fin] + ATOL
    ratio = float((err / bound).max()) if err.size else 0.0
    bad = np.flatnonzero(err > bound)
    assert bad.size == 0, (f"{bad.size} elements out of tolerance, worst ratio {ratio:.3g}; "
                           f"first: gpu={gpu[fin][bad[0]]} ref={ref[fin][bad[0]]}")
    return ratio
